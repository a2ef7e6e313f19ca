"""CPU tests of libpa.so: exported symbols, the host block allocator, and the
capacity arithmetic against the figures the pages print (no GPU needed)."""
import ctypes
import json
import os
import re
import shutil
import subprocess
import sys

import numpy as np
import pytest

import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")

pk = pytest.importorskip("paged_kv_cache_425_b200")
from paged_kv_cache_425_b200 import batch  # noqa: E402


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"\b(pa_\w+)\s*\(", text)
    return sorted(set(names))


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert "pa_decode" in names and "pa_reshape_and_cache" in names and "pa_copy_blocks" in names
    lib = ctypes.CDLL(pk.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_version():
    assert pk.pa_status_string(0) == b"ok"
    assert pk.pa_status_string(pk.PA_ERR_WORKSPACE).startswith(b"workspace")
    assert pk.pa_version() >= 100


def test_workspace_size_rule():
    assert pk.decode_workspace_size(64, 32, 128, 32) == 0            # one partition
    n = pk.decode_workspace_size(64, 32, 128, 128)                  # 4 partitions
    rows = 64 * 32 * 4
    assert n >= rows * 128 * 4 + rows * 8 and n % 256 == 0
    assert pk.decode_workspace_size(64, 32, 128, 128, block_size=32) == 0


def test_workspace_follows_the_partition_rule():
    """Tables spanning 16384 tokens or more use 1024-token partitions: half as
    many partials per row as 512-token ones."""
    def rows_parts(max_blocks):
        n = pk.decode_workspace_size(8, 8, 128, max_blocks)
        return n // (8 * 8 * (128 * 4 + 8))  # lower bound on partitions per row
    assert rows_parts(1023) == 32          # 16368 tokens: 512-token partitions
    assert rows_parts(1024) == 16          # 16384 tokens: 1024-token partitions
    assert rows_parts(2048) == 32


def test_import_fails_loudly_without_the_library(tmp_path):
    dst = tmp_path / "paged_kv_cache_425_b200"
    shutil.copytree(os.path.join(ROOT, "paged_kv_cache_425_b200"), dst,
                    ignore=shutil.ignore_patterns("*.so", "csrc", "__pycache__"))
    code = "import paged_kv_cache_425_b200"
    r = subprocess.run([sys.executable, "-c", code], cwd=tmp_path, capture_output=True, text=True,
                       env={**os.environ, "PYTHONPATH": str(tmp_path)})
    assert r.returncode != 0 and "missing" in r.stderr


# ---------------------------------------------------------------- allocator semantics
def test_fresh_pool_hands_out_in_order_and_frees_to_the_back():
    a = pk.BlockAllocator(8)
    a.add_seq(1, 33)                       # 3 blocks
    assert list(a.block_table(1)) == [0, 1, 2]
    a.add_seq(2, 16)
    assert list(a.block_table(2)) == [3]
    a.free_seq(1)
    a.add_seq(3, 64)                       # 4 blocks: 4..7 first, then the freed ones
    assert list(a.block_table(3)) == [4, 5, 6, 7]
    a.add_seq(4, 1)
    assert list(a.block_table(4)) == [0]


def test_exhaustion_fails_without_side_effects():
    a = pk.BlockAllocator(4)
    a.add_seq(1, 40)                       # 3 blocks
    before = a.stats()
    with pytest.raises(pk.PagedError) as e:
        a.add_seq(2, 17)                   # needs 2, 1 free
    assert e.value.status == pk.PA_ERR_NO_BLOCKS
    assert a.stats() == before
    a.add_seq(2, 16)
    a.append_slot(1)                       # 41st token fits in block 2
    with pytest.raises(pk.PagedError):
        for _ in range(8):
            a.append_slot(1)               # token 49 needs a 5th block
    assert a.num_tokens(1) == 48


def test_append_slot_places_tokens_by_the_table():
    a = pk.BlockAllocator(50)
    rng = np.random.default_rng(0)
    for s in range(5):
        a.add_seq(s, int(rng.integers(0, 40)))
    for _ in range(200):
        s = int(rng.integers(0, 5))
        p = a.num_tokens(s)
        slot, (src, dst) = a.append_slot(s)
        assert (src, dst) == (-1, -1)
        t = a.block_table(s)
        assert slot == t[p // 16] * 16 + p % 16
        assert len(t) == (p + 1 + 15) // 16


def test_fork_shares_and_first_writers_copy_last_writes_in_place():
    a = pk.BlockAllocator(20)
    a.add_seq(0, 40)                       # blocks 0,1,2; block 2 holds 8 tokens
    for c in (1, 2, 3):
        a.fork(0, c)
    assert [a.refcount(b) for b in (0, 1, 2)] == [4, 4, 4]
    copies = []
    for s in (0, 1, 2, 3):
        slot, pair = a.append_slot(s)
        copies.append(pair)
        t = a.block_table(s)
        assert slot == t[2] * 16 + 8
    assert copies[:3] == [(2, 3), (2, 4), (2, 5)]  # first three writers copy block 2
    assert copies[3] == (-1, -1)                   # the last holder writes in place
    assert list(a.block_table(3)) == [0, 1, 2]
    assert [a.refcount(b) for b in (0, 1, 2, 3, 4, 5)] == [4, 4, 1, 1, 1, 1]
    st = a.stats()
    assert st["cow_copies"] == 3 and st["shared_blocks"] == 2
    # a full shared block needs no copy: the next token opens a new block
    b = pk.BlockAllocator(10)
    b.add_seq(0, 32)
    b.fork(0, 1)
    _, pair = b.append_slot(1)
    assert pair == (-1, -1) and b.block_table(1)[2] not in (0, 1)


def test_free_releases_only_unshared_blocks():
    a = pk.BlockAllocator(10)
    a.add_seq(0, 20)
    a.fork(0, 1)
    a.free_seq(0)
    assert a.stats()["free_blocks"] == 8
    a.free_seq(1)
    assert a.stats()["free_blocks"] == 10


def test_random_operations_keep_the_pool_consistent():
    """Refcounts equal the number of tables holding each block; free + used =
    pool; tables have ceil(tokens / 16) entries."""
    rng = np.random.default_rng(1)
    a = pk.BlockAllocator(200)
    live, next_id = set(), 0
    for _ in range(3000):
        op = rng.integers(0, 4)
        try:
            if op == 0 or not live:
                a.add_seq(next_id, int(rng.integers(0, 60)))
                live.add(next_id)
                next_id += 1
            elif op == 1:
                s = int(rng.choice(sorted(live)))
                a.fork(s, next_id)
                live.add(next_id)
                next_id += 1
            elif op == 2:
                a.append_slot(int(rng.choice(sorted(live))))
            else:
                s = int(rng.choice(sorted(live)))
                a.free_seq(s)
                live.discard(s)
        except pk.PagedError as e:
            assert e.status == pk.PA_ERR_NO_BLOCKS
        holders = np.zeros(200, np.int64)
        for s in live:
            t = a.block_table(s)
            assert len(t) == (a.num_tokens(s) + 15) // 16
            assert len(set(t.tolist())) == len(t)
            np.add.at(holders, t, 1)
        rc = np.array([a.refcount(b) for b in range(200)])
        assert np.array_equal(rc, holders)
        st = a.stats()
        assert st["free_blocks"] + st["used_blocks"] == 200
        assert st["used_blocks"] == int((rc > 0).sum())


def test_build_tables_pads_with_minus_one():
    a = pk.BlockAllocator(10)
    a.add_seq(7, 20)
    a.add_seq(9, 0)
    t, lens = a.build_tables([9, 7], 4)
    assert t.tolist() == [[-1, -1, -1, -1], [0, 1, -1, -1]] and lens.tolist() == [0, 20]
    with pytest.raises(pk.PagedError):
        a.build_tables([7], 1)


# ---------------------------------------------------------------- the pages' figures
@pytest.mark.parametrize("name", ["llama7b", "llama13b"])
def test_waste_below_four_percent(name):
    """Paging wastes at most the tail of each sequence's last block: under 4 %
    ('vLLM PagedAttention: reducing KV cache memory waste', opening and 'How
    PagedAttention Works')."""
    w = wl.WORKLOADS[name]
    rng = wl.rng_for(0)
    lens = wl.draw_context_lens(w, rng)
    nb = wl.pool_size(w, lens)
    b = batch.decode_batch(w, lens, wl.draw_block_order(nb, rng), nb, batch.max_blocks_for(w))
    st = b.alloc.stats()
    last_block_tail = sum((-int(L)) % 16 for L in lens)
    assert st["filled_slots"] == int(lens.sum())
    assert st["used_blocks"] * 16 - st["filled_slots"] == last_block_tail
    assert st["waste"] < 0.04
    # the tables really are scattered: few consecutive neighbours
    t = b.tables
    nxt = (t[:, 1:] == t[:, :-1] + 1) & (t[:, 1:] >= 0)
    assert nxt.sum() < 0.01 * (t >= 0).sum()


def test_copy_on_write_step_of_the_sampling_workload():
    w = wl.WORKLOADS["cow"]
    rng = wl.rng_for(0)
    own = wl.draw_branch_tokens(w, rng)
    nb = batch.cow_pool_blocks(w)
    fb = batch.ForkedBatch(w, own, wl.draw_block_order(nb, rng), nb)
    b = fb.step()
    assert len(b.pairs) == w.prompts * (w.branches - 1)
    assert np.all(b.context_lens == w.prompt_len + 1)
    st = fb.alloc.stats()
    assert st["shared_blocks"] == w.prompts * (w.prompt_len // 16)
    assert st["sharing_saving"] > 0.5


def test_kv_size_formula_reproduces_printed_13b_figure():
    with open(os.path.join(GOLDEN, "kv_size_13b.json")) as f:
        g = json.load(f)
    per_token = pk.kv_bytes_per_token(g["layers"], g["kv_heads"], g["head_dim"], g["dtype_bytes"])
    assert per_token == 2 * 40 * 5120 * 2
    gb = per_token * g["tokens"] / 1e9
    assert abs(gb - g["printed_gb"]) <= g["printed_gb_tolerance"]
    assert abs(gb - g["rough_gb"]) <= g["rough_gb_tolerance"]


def test_pool_budget_reproduces_printed_figure():
    with open(os.path.join(GOLDEN, "pool_budget.json")) as f:
        g = json.load(f)
    got = pk.pool_bytes(g["gpu_gb"] * 1e9, g["weights_gb"] * 1e9, g["utilization"]) / 1e9
    assert abs(got - g["printed_pool_gb"]) < 1e-9
    assert pk.pool_bytes(8e9, 16e9, 0.9) == 0.0
    blocks = pk.pool_num_blocks(got * 1e9, 32, 8, 128, 16, 2)  # Llama-3.1-8B shape
    assert blocks == int(7.2e9 // (16 * 2 * 32 * 8 * 128 * 2))


# ---------------------------------------------------------------- automatic prefix caching
def _tokens(rng, n):
    return rng.integers(0, 32000, size=n).astype(np.int32)


def test_prefix_cache_shares_matching_full_blocks():
    rng = np.random.default_rng(3)
    a = pk.BlockAllocator(32)
    a.enable_prefix_caching()
    system = _tokens(rng, 40)                       # 2 full blocks + 8 tokens
    p1 = np.concatenate([system, _tokens(rng, 5)])
    p2 = np.concatenate([system, _tokens(rng, 30)])
    assert a.add_seq_tokens(1, p1) == 0
    assert a.add_seq_tokens(2, p2) == 32            # the two full blocks are reused
    t1, t2 = a.block_table(1), a.block_table(2)
    assert list(t1[:2]) == list(t2[:2]) and t1[2] != t2[2]
    assert [a.refcount(b) for b in t1[:2]] == [2, 2]
    st = a.stats()
    assert st["prefix_hit_blocks"] == 2 and st["prefix_query_blocks"] == 2 + 4
    assert st["cached_blocks"] == 2 + 2             # p2's own third and fourth full blocks


def test_prefix_cache_matches_only_whole_prefixes():
    rng = np.random.default_rng(4)
    a = pk.BlockAllocator(32)
    a.enable_prefix_caching()
    base = _tokens(rng, 48)
    a.add_seq_tokens(1, base)
    other = base.copy()
    other[20] += 1                                  # differs inside block 1
    assert a.add_seq_tokens(2, other) == 16          # only block 0 matches
    shifted = np.concatenate([_tokens(rng, 16), base[16:32]])
    assert a.add_seq_tokens(3, shifted) == 0         # same block content, other prefix
    assert a.add_seq_tokens(4, base[:47]) == 32      # partial last block is never shared


def test_freed_cached_blocks_stay_findable_until_reused():
    rng = np.random.default_rng(5)
    a = pk.BlockAllocator(6)
    a.enable_prefix_caching()
    p = _tokens(rng, 48)                            # 3 full blocks
    a.add_seq_tokens(1, p)
    a.free_seq(1)
    assert a.stats()["free_blocks"] == 6 and a.stats()["cached_blocks"] == 3
    assert a.add_seq_tokens(2, p) == 48             # revived from the free list
    assert a.stats()["free_blocks"] == 3
    a.free_seq(2)
    a.add_seq(3, 16 * 4)                            # 4 blocks: 3 never-used, then evicts one
    assert a.stats()["cached_blocks"] == 2
    a.free_seq(3)
    assert a.add_seq_tokens(4, p) == 0              # the first cached block was evicted


def test_prefix_cache_off_behaves_like_add_seq():
    rng = np.random.default_rng(6)
    a = pk.BlockAllocator(8)
    p = _tokens(rng, 40)
    assert a.add_seq_tokens(1, p) == 0
    assert a.add_seq_tokens(2, p) == 0
    assert list(a.block_table(1)) == [0, 1, 2] and list(a.block_table(2)) == [3, 4, 5]
    assert a.stats()["cached_blocks"] == 0


def test_prefix_cache_exhaustion_leaves_state_unchanged():
    rng = np.random.default_rng(7)
    a = pk.BlockAllocator(5)
    a.enable_prefix_caching()
    p = _tokens(rng, 32)
    a.add_seq_tokens(1, p)                          # 2 blocks
    a.add_seq(2, 48)                                # 3 blocks: pool full
    before = a.stats()
    with pytest.raises(pk.PagedError) as e:
        a.add_seq_tokens(3, np.concatenate([p, _tokens(rng, 1)]))  # 2 hits + 1 new: none free
    assert e.value.status == pk.PA_ERR_NO_BLOCKS and a.stats() == before
    a.free_seq(2)
    assert a.add_seq_tokens(3, np.concatenate([p, _tokens(rng, 1)])) == 32


def test_prefix_cache_hit_rate_on_shared_system_prompt():
    """Requests that share a 512-token system prompt reuse its 32 blocks:
    every request after the first hits all of them."""
    rng = np.random.default_rng(8)
    a = pk.BlockAllocator(4096)
    a.enable_prefix_caching()
    system = _tokens(rng, 512)
    for r in range(50):
        user = _tokens(rng, int(rng.integers(1, 300)))
        cached = a.add_seq_tokens(r, np.concatenate([system, user]))
        assert cached >= (0 if r == 0 else 512)
    st = a.stats()
    assert st["prefix_hit_blocks"] == 49 * 32
    assert st["prefix_hit_blocks"] / st["prefix_query_blocks"] > 0.5


def test_random_operations_with_prefix_cache_keep_the_pool_consistent():
    rng = np.random.default_rng(9)
    a = pk.BlockAllocator(120)
    a.enable_prefix_caching()
    prompts = [_tokens(rng, int(rng.integers(1, 80))) for _ in range(6)]
    live, next_id = set(), 0
    for _ in range(2000):
        op = rng.integers(0, 4)
        try:
            if op == 0 or not live:
                base = prompts[int(rng.integers(0, 6))]
                p = np.concatenate([base, _tokens(rng, int(rng.integers(0, 20)))])
                cached = a.add_seq_tokens(next_id, p)
                assert cached % 16 == 0 and cached <= len(p)
                live.add(next_id)
                next_id += 1
            elif op == 1:
                a.append_slot(int(rng.choice(sorted(live))))
            elif op == 2:
                s = int(rng.choice(sorted(live)))
                a.fork(s, next_id)
                live.add(next_id)
                next_id += 1
            else:
                s = int(rng.choice(sorted(live)))
                a.free_seq(s)
                live.discard(s)
        except pk.PagedError as e:
            assert e.status == pk.PA_ERR_NO_BLOCKS
        holders = np.zeros(120, np.int64)
        for s in live:
            np.add.at(holders, a.block_table(s), 1)
        rc = np.array([a.refcount(b) for b in range(120)])
        assert np.array_equal(rc, holders)
        st = a.stats()
        assert st["free_blocks"] + st["used_blocks"] == 120


def test_swap_rejects_bad_ids_before_any_copy():
    """Host-side check: no CUDA call happens for an out-of-range pair."""
    buf = np.zeros(4 * 2 * 16 * 64, np.uint16)
    pairs = np.array([[0, 1], [5, 2]], np.int32)  # source 5 of a 4-block pool
    rc = pk.pa_swap_blocks(buf.ctypes.data, buf.ctypes.data, 4, buf.ctypes.data, buf.ctypes.data,
                           4, pairs.ctypes.data, 2, 2, 64, 16, pk.F16, None)
    assert rc == pk.PA_ERR_OUT_OF_RANGE
    assert pk.pa_swap_blocks(buf.ctypes.data, buf.ctypes.data, 4, buf.ctypes.data,
                             buf.ctypes.data, 4, pairs.ctypes.data, 2, 2, 96, 16, pk.F16,
                             None) == pk.PA_ERR_UNSUPPORTED


# ---------------------------------------------------------------- continuous batching simulation
def _requests(seed=0, n=200):
    rng = np.random.default_rng(seed)
    return rng.integers(50, 500, n).astype(np.int32), rng.integers(1, 300, n).astype(np.int32)


def test_simulation_finishes_everything_and_counts_each_token_once():
    pl, ol = _requests()
    for nb, m in ((20000, 64), (600, 64), (300, 256)):
        st = pk.simulate_continuous_batching(nb, m, pl, ol)
        assert st["finished"] == len(pl) and st["rejected"] == 0
        assert st["tokens_generated"] == int(ol.sum())
        assert st["admitted"] == len(pl) + st["preemptions"]
        assert 0 < st["mean_usage"] <= st["max_usage"] <= 1.0


def test_ample_pool_never_preempts_and_one_slot_is_sequential():
    pl, ol = _requests(1, 50)
    assert pk.simulate_continuous_batching(100000, 64, pl, ol)["preemptions"] == 0
    st = pk.simulate_continuous_batching(100000, 1, pl, ol)
    assert st["steps"] == int(ol.sum()) and st["mean_running"] <= 1.0


def test_too_few_sequences_starve_and_too_many_preempt():
    """'PagedAttention in vLLM: a throughput settings guide', 'Continuous
    Batching Keeps the GPU Busy': too low a max_num_seqs starves the GPU
    (more steps for the same tokens), too high with a fixed KV budget
    increases preemption."""
    pl, ol = _requests(2)
    low = pk.simulate_continuous_batching(600, 4, pl, ol)
    mid = pk.simulate_continuous_batching(600, 16, pl, ol)
    high = pk.simulate_continuous_batching(600, 256, pl, ol)
    assert low["steps"] > mid["steps"]
    assert low["preemptions"] == 0 and high["preemptions"] > mid["preemptions"]
    assert high["max_usage"] == 1.0


def test_requests_larger_than_the_pool_are_rejected():
    st = pk.simulate_continuous_batching(10, 4, np.array([100, 400], np.int32),
                                         np.array([10, 10], np.int32))
    assert st["rejected"] == 1 and st["finished"] == 1


def test_prefill_select_accepts_the_three_kernels_only():
    assert pk.pa_prefill_select(7) == pk.PA_ERR_INVALID_ARG
    assert pk.pa_prefill_select(-1) == pk.PA_ERR_INVALID_ARG
    for name in ("mma_sync", "tcgen05", "auto"):
        pk.prefill_select(name)
    with pytest.raises(ValueError):
        pk.prefill_select("wgmma")


def test_build_rebuilds_on_any_source_or_header_change():
    """The staleness check covers every file the library is compiled from."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "pa_build", os.path.join(ROOT, "paged_kv_cache_425_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    csrc = os.path.join(ROOT, "paged_kv_cache_425_b200", "csrc")
    want = {os.path.join(csrc, f) for f in os.listdir(csrc)}
    want |= {os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))}
    assert want <= set(b.DEPS)


def test_static_workspace_decode_checks_arguments_like_pa_decode():
    """pa_decode_static_workspace applies pa_decode's argument checks before
    its own size limit, so both return the same status for the same bad
    arguments, even at sizes far beyond the static array (host checks only:
    nothing reaches a device)."""
    huge_s, d, maxb, nb = 1 << 20, 128, 4096, 1024
    cases = [
        (64, 2),            # a query group of 32 heads: unsupported
        (30, 4),            # 30 q heads over 4 kv heads: invalid
    ]
    for hq, hkv in cases:
        a = pk.pa_decode(None, None, None, None, None, None, hkv, 0.1, huge_s, hq, d, 16, maxb,
                         nb, pk.F16, None, 0, None)
        b = pk.pa_decode_static_workspace(None, None, None, None, None, None, hkv, 0.1, huge_s,
                                          hq, d, 16, maxb, nb, pk.F16, None)
        assert a == b and a in (pk.PA_ERR_UNSUPPORTED, pk.PA_ERR_INVALID_ARG), (hq, hkv, a, b)
    # more than 8192 partitions per sequence: unsupported on both.  The
    # pointers are aligned placeholders: the call returns before any launch
    # and never dereferences them.
    wide = 8193 * 64
    fake = [4096 * (i + 1) for i in range(6)]
    a = pk.pa_decode(*fake, 8, 0.1, 4, 32, d, 16, wide, nb, pk.BF16, None, 0, None)
    b = pk.pa_decode_static_workspace(*fake, 8, 0.1, 4, 32, d, 16, wide, nb, pk.BF16, None)
    assert a == b == pk.PA_ERR_UNSUPPORTED


def test_decode_append_checks_arguments_like_pa_decode():
    """pa_decode_append applies pa_decode's checks first, then its own on
    the new rows (present, 16-byte aligned).  Host checks only: every case
    returns before a launch, and the pointers (aligned placeholders, or
    none) are never dereferenced."""
    huge_s, d, maxb, nb = 1 << 20, 128, 4096, 1024
    for hq, hkv in ((64, 2), (30, 4)):
        a = pk.pa_decode(None, None, None, None, None, None, hkv, 0.1, huge_s, hq, d, 16, maxb,
                         nb, pk.F16, None, 0, None)
        b = pk.pa_decode_append(None, None, None, None, None, None, None, None, hkv, 0.1, huge_s,
                                hq, d, 16, maxb, nb, pk.F16, None, 0, None)
        assert a == b and a in (pk.PA_ERR_UNSUPPORTED, pk.PA_ERR_INVALID_ARG), (hq, hkv, a, b)
    fake = [4096 * (i + 1) for i in range(8)]
    out, q, kn, vn, kc, vc, tb, ln = fake
    # no sequences: nothing to do, whatever the new rows are
    assert pk.pa_decode_append(out, q, None, None, kc, vc, tb, ln, 8, 0.1, 0, 32, d, 16, 64,
                               nb, pk.BF16, None, 0, None) == pk.PA_OK
    # missing or misaligned new rows
    for k_new, v_new in ((None, vn), (kn, None), (kn + 8, vn), (kn, vn + 4)):
        assert pk.pa_decode_append(out, q, k_new, v_new, kc, vc, tb, ln, 8, 0.1, 4, 32, d, 16,
                                   64, nb, pk.BF16, None, 0, None) == pk.PA_ERR_INVALID_ARG
    # a split context without a workspace is refused after the new-row checks pass
    assert pk.pa_decode_append(out, q, kn, vn, kc, vc, tb, ln, 8, 0.1, 4, 32, d, 16, 64, nb,
                               pk.BF16, None, 0, None) == pk.PA_ERR_WORKSPACE
