"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Bit-exact for the scatter write and the block copy (whole pool compared);
attention outputs within max-abs 2e-3 (fp16) / 1e-2 (bf16) of the oracle.
Sizes span several 16-token blocks, several 512-token partitions and ragged
tails; edge cases: one token, empty context, identical keys, permuted
placement, bad indices reported through the device error word.
"""
import numpy as np
import pytest

import oracle
import workloads as wl
from paged_inputs import make_paged, to_f64 as bits_f64

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import gpu_harness as gh  # noqa: E402

pk = pytest.importorskip("paged_kv_cache_425_b200")


def oracle_out(p, seqs=None):
    return oracle.decode(p.q, p.key_cache, p.value_cache, p.tables, p.lens, p.num_kv_heads,
                         p.scale, p.dtype, seqs=seqs)


def gpu_out(p, stream=None):
    return gh.run_decode(pk, p.q, p.key_cache, p.value_cache, p.tables, p.lens, p.num_kv_heads,
                         p.scale, p.dtype, stream=stream)


# ---------------------------------------------------------------- the tiny workload, whole step
def test_tiny_workload_step():
    """4 seqs, 4/4 heads, d 64, fp16, ctx U{1..64}, 64-block pool, one new
    token per sequence written by pa_reshape_and_cache, then pa_decode."""
    w = wl.WORKLOADS["tiny"]
    rng = wl.rng_for(0)
    lens = wl.draw_context_lens(w, rng)
    p = make_paged(rng, w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, lens,
                   w.pool_blocks, w.dtype, scale=w.scale)
    k_new = wl.draw_values(rng, (w.num_seqs, w.num_kv_heads, w.head_dim), w.dtype)
    v_new = wl.draw_values(rng, (w.num_seqs, w.num_kv_heads, w.head_dim), w.dtype)
    pos = lens - 1
    slots = np.array([p.tables[s, pos[s] // 16] * 16 + pos[s] % 16 for s in range(w.num_seqs)],
                     np.int64)
    kc, vc = gh.to_dev(p.key_cache, w.dtype), gh.to_dev(p.value_cache, w.dtype)
    pk.reshape_and_cache(gh.to_dev(k_new, w.dtype), gh.to_dev(v_new, w.dtype), kc, vc,
                         gh.ints(slots, torch.int64))
    out = gh.run_decode(pk, p.q, kc, vc, p.tables, p.lens, w.num_kv_heads, w.scale, w.dtype)
    assert pk.get_error() == (0, 0)
    oracle.reshape_and_cache(k_new, v_new, p.key_cache, p.value_cache, slots)
    assert np.array_equal(gh.to_host_bits(kc), p.key_cache)
    assert np.array_equal(gh.to_host_bits(vc), p.value_cache)
    assert gh.max_err(out, oracle_out(p)) <= gh.TOL[w.dtype]


# ---------------------------------------------------------------- fused append + decode
def append_slots(p):
    """Slot of each sequence's last position (its new token), from its table."""
    return np.array([p.tables[s, (L - 1) // 16] * 16 + (L - 1) % 16 if L > 0 else -1
                     for s, L in enumerate(p.lens)], np.int64)


@pytest.mark.parametrize("hq,hkv,d,dtype", [(4, 4, 64, wl.F16), (32, 32, 128, wl.F16),
                                            (32, 8, 128, wl.BF16), (16, 1, 128, wl.BF16),
                                            (12, 1, 64, wl.F16)])
def test_decode_append_equals_scatter_then_decode(hq, hkv, d, dtype):
    """pa_decode_append against pa_reshape_and_cache + pa_decode on copies of
    one pool: the same pool bytes and the same outputs, bit for bit; and both
    against the oracle's write and attention.  Lengths put the new token
    first in a block, last in a block, alone in a context, and in the last of
    several partitions; one sequence is empty."""
    rng = wl.rng_for(60 + hq + d)
    lens = np.array([1, 16, 17, 32, 100, 511, 513, 1024, 1025, 3000, 0], np.int32)
    p = make_paged(rng, len(lens), hq, hkv, d, lens, wl.blocks_needed(lens, 16) + 5, dtype)
    k_new = wl.draw_values(rng, (len(lens), hkv, d), dtype)
    v_new = wl.draw_values(rng, (len(lens), hkv, d), dtype)
    slots = append_slots(p)
    tbl, ln = gh.ints(p.tables), gh.ints(p.lens)
    dk, dv = gh.to_dev(k_new, dtype), gh.to_dev(v_new, dtype)
    q = gh.to_dev(p.q, dtype)
    ws = gh.workspace_for(pk, len(lens), hq, d, p.tables.shape[1])

    kc1, vc1 = gh.to_dev(p.key_cache, dtype), gh.to_dev(p.value_cache, dtype)
    out1 = torch.full_like(q, float("nan"))
    pk.reshape_and_cache(dk, dv, kc1, vc1, gh.ints(slots, torch.int64))
    pk.decode(out1, q, kc1, vc1, tbl, ln, hkv, p.scale, workspace=ws)
    kc2, vc2 = gh.to_dev(p.key_cache, dtype), gh.to_dev(p.value_cache, dtype)
    out2 = torch.full_like(q, float("nan"))
    pk.decode_append(out2, q, dk, dv, kc2, vc2, tbl, ln, hkv, p.scale, workspace=ws)
    torch.cuda.synchronize()
    assert pk.get_error() == (0, 0)
    assert torch.equal(kc1, kc2) and torch.equal(vc1, vc2)
    assert torch.equal(out1, out2)

    oracle.reshape_and_cache(k_new, v_new, p.key_cache, p.value_cache, slots)
    assert np.array_equal(gh.to_host_bits(kc2), p.key_cache)
    assert np.array_equal(gh.to_host_bits(vc2), p.value_cache)
    assert gh.max_err(out2, oracle_out(p)) <= gh.TOL[dtype]


def test_decode_append_bad_last_block_writes_nothing():
    """An out-of-range id where sequence 1's new token goes: reported as a bad
    block id, nothing written anywhere, the other sequences exact."""
    rng = wl.rng_for(66)
    lens = np.array([40, 70, 300], np.int32)
    p = make_paged(rng, 3, 8, 2, 128, lens, wl.blocks_needed(lens, 16) + 2, wl.BF16)
    k_new = wl.draw_values(rng, (3, 2, 128), wl.BF16)
    v_new = wl.draw_values(rng, (3, 2, 128), wl.BF16)
    slots = append_slots(p)
    p.tables[1, (70 - 1) // 16] = p.key_cache.shape[0] + 3
    kc, vc = gh.to_dev(p.key_cache, wl.BF16), gh.to_dev(p.value_cache, wl.BF16)
    q = gh.to_dev(p.q, wl.BF16)
    out = torch.full_like(q, float("nan"))
    pk.decode_append(out, q, gh.to_dev(k_new, wl.BF16), gh.to_dev(v_new, wl.BF16), kc, vc,
                     gh.ints(p.tables), gh.ints(p.lens), 2, p.scale)
    torch.cuda.synchronize()
    rc, bits = pk.get_error()
    assert rc == pk.PA_ERR_OUT_OF_RANGE and bits & pk.DEVERR_BLOCK_ID
    slots[1] = -1  # the oracle writes the other two
    oracle.reshape_and_cache(k_new, v_new, p.key_cache, p.value_cache, slots)
    assert np.array_equal(gh.to_host_bits(kc), p.key_cache)
    assert np.array_equal(gh.to_host_bits(vc), p.value_cache)
    ref = oracle.decode(p.q, p.key_cache, p.value_cache, p.tables, p.lens, 2, p.scale, wl.BF16,
                        seqs=[0, 2])
    assert gh.max_err(out[[0, 2]], ref) <= gh.TOL[wl.BF16]


def test_decode_append_context_beyond_the_table_writes_nothing():
    """Sequence 1's context length runs past its table: reported as a bad
    context length, its new row is written nowhere (the length is clamped
    for the attention, but position L - 1 has no slot), the other sequence
    is written and exact."""
    rng = wl.rng_for(69)
    lens = np.array([30, 32], np.int32)
    p = make_paged(rng, 2, 4, 2, 64, lens, 6, wl.F16, max_blocks=2)
    k_new = wl.draw_values(rng, (2, 2, 64), wl.F16)
    v_new = wl.draw_values(rng, (2, 2, 64), wl.F16)
    slots = append_slots(p)
    bad = p.lens.copy()
    bad[1] = 32 + 1000
    kc, vc = gh.to_dev(p.key_cache, wl.F16), gh.to_dev(p.value_cache, wl.F16)
    q = gh.to_dev(p.q, wl.F16)
    out = torch.full_like(q, float("nan"))
    pk.decode_append(out, q, gh.to_dev(k_new, wl.F16), gh.to_dev(v_new, wl.F16), kc, vc,
                     gh.ints(p.tables), gh.ints(bad), 2, p.scale)
    torch.cuda.synchronize()
    rc, bits = pk.get_error()
    assert rc == pk.PA_ERR_OUT_OF_RANGE and bits & pk.DEVERR_CONTEXT_LEN
    slots[1] = -1
    oracle.reshape_and_cache(k_new, v_new, p.key_cache, p.value_cache, slots)
    assert np.array_equal(gh.to_host_bits(kc), p.key_cache)
    assert np.array_equal(gh.to_host_bits(vc), p.value_cache)
    ref = oracle.decode(p.q, p.key_cache, p.value_cache, p.tables, p.lens, 2, p.scale, wl.F16,
                        seqs=[0])
    assert gh.max_err(out[:1], ref) <= gh.TOL[wl.F16]


def test_decode_append_checks_its_new_rows():
    rng = wl.rng_for(67)
    lens = np.array([5, 9], np.int32)
    p = make_paged(rng, 2, 4, 4, 64, lens, 4, wl.F16)
    kc, vc = gh.to_dev(p.key_cache, wl.F16), gh.to_dev(p.value_cache, wl.F16)
    q = gh.to_dev(p.q, wl.F16)
    out = torch.empty_like(q)
    kn = torch.zeros((2, 4, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(ValueError):
        pk.decode_append(out, q, kn[:, :2], kn, kc, vc, gh.ints(p.tables), gh.ints(p.lens), 4,
                         p.scale)
    buf = torch.zeros(2 * 4 * 64 + 4, dtype=torch.float16, device="cuda")
    misaligned = buf[4:].view(2, 4, 64)  # 8 bytes past a 16-byte boundary
    with pytest.raises(pk.PagedError) as e:
        pk.decode_append(out, q, misaligned, kn, kc, vc, gh.ints(p.tables), gh.ints(p.lens), 4,
                         p.scale)
    assert e.value.status == pk.PA_ERR_INVALID_ARG


# ---------------------------------------------------------------- shapes x lengths
LENS = [1, 15, 16, 17, 100, 511, 512, 513, 1024, 1500, 2049, 3000]


@pytest.mark.parametrize("dtype", [wl.F16, wl.BF16], ids=["f16", "bf16"])
@pytest.mark.parametrize("hq,hkv,d", [(2, 2, 128), (3, 3, 64), (8, 4, 128), (8, 2, 64),
                                      (16, 4, 128), (8, 1, 128), (12, 1, 64), (16, 1, 128),
                                      (32, 8, 128)])
def test_decode_shapes_and_lengths(dtype, hq, hkv, d):
    rng = wl.rng_for(100 + hq * 7 + hkv + d)
    lens = np.array(LENS, np.int32)
    nb = wl.blocks_needed(lens, 16) + 5
    p = make_paged(rng, len(lens), hq, hkv, d, lens, nb, dtype)
    err = gh.max_err(gpu_out(p), oracle_out(p))
    assert err <= gh.TOL[dtype], err


@pytest.mark.parametrize("hq,hkv,d,dtype", [(2, 2, 64, wl.F16), (8, 2, 128, wl.BF16),
                                            (4, 4, 128, wl.BF16)])
def test_every_context_length_1_to_64(hq, hkv, d, dtype):
    rng = wl.rng_for(7)
    lens = np.arange(1, 65, dtype=np.int32)
    p = make_paged(rng, 64, hq, hkv, d, lens, wl.blocks_needed(lens, 16), dtype)
    assert gh.max_err(gpu_out(p), oracle_out(p)) <= gh.TOL[dtype]


@pytest.mark.parametrize("hq,hkv,dtype", [(8, 8, wl.F16), (16, 4, wl.BF16)])
def test_tables_at_the_wide_partition_threshold(hq, hkv, dtype):
    """Tables of 1023 blocks keep 512-token partitions; 1024 blocks (16384
    tokens) switch to 1024-token ones.  Contexts straddle both boundary sets."""
    lens = np.array([1, 511, 512, 513, 1023, 1024, 1025, 2047, 2049, 15000], np.int32)
    for width in (1023, 1024):
        rng = wl.rng_for(12 + width)
        L = np.minimum(lens, width * 16)
        p = make_paged(rng, len(L), hq, hkv, 128, L, wl.blocks_needed(L, 16) + 2, dtype,
                       max_blocks=width)
        assert gh.max_err(gpu_out(p), oracle_out(p)) <= gh.TOL[dtype], width


@pytest.mark.parametrize("hq,hkv,dtype", [(4, 4, wl.F16), (8, 2, wl.BF16), (16, 1, wl.BF16)])
def test_two_eight_and_nine_partitions(hq, hkv, dtype):
    """Tables of 33, 256 and 257 blocks split a context into up to 2, 8 and 9
    partitions of 512 tokens: the merge kernel loads all of a row's partials
    at once up to 8 partitions and loops over them beyond.  Contexts cover
    one partition, the partition boundaries, and the whole table."""
    for width in (33, 256, 257):
        rng = wl.rng_for(40 + width)
        cap = width * 16
        lens = np.array([1, 16, 511, 512, 513, 1024, 1025, 4095, 4096, cap - 1, cap], np.int32)
        lens = np.minimum(lens, cap)
        p = make_paged(rng, len(lens), hq, hkv, 128, lens, wl.blocks_needed(lens, 16) + 2, dtype,
                       max_blocks=width)
        assert gh.max_err(gpu_out(p), oracle_out(p)) <= gh.TOL[dtype], width
    assert pk.get_error() == (0, 0)


def test_wide_table_many_partitions():
    """Table width 2048 blocks (32 partitions of 1024 tokens) with short and
    long contexts."""
    rng = wl.rng_for(8)
    lens = np.array([5, 8192, 32768, 513, 20000], np.int32)
    nb = wl.blocks_needed(lens, 16) + 3
    p = make_paged(rng, 5, 8, 2, 128, lens, nb, wl.BF16, max_blocks=2048)
    assert gh.max_err(gpu_out(p), oracle_out(p)) <= gh.TOL[wl.BF16]


# ---------------------------------------------------------------- closed forms on the GPU
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2)])
def test_one_token_returns_v0_exactly(hq, hkv):
    rng = wl.rng_for(9)
    p = make_paged(rng, 3, hq, hkv, 128, [1, 1, 1], 3, wl.BF16)
    out = gh.to_host_bits(gpu_out(p))
    G = hq // hkv
    for s in range(3):
        for h in range(hq):
            assert np.array_equal(out[s, h], p.v_dense[s, 0, h // G])


@pytest.mark.parametrize("hq,hkv", [(4, 4), (16, 2)])
def test_empty_context_gives_zeros(hq, hkv):
    rng = wl.rng_for(10)
    p = make_paged(rng, 3, hq, hkv, 64, [0, 700, 0], 50, wl.F16)
    out = gh.to_f64(gpu_out(p))
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    assert np.max(np.abs(out[1] - oracle_out(p)[1])) <= gh.TOL[wl.F16]


def test_identical_keys_give_mean_of_values():
    rng = wl.rng_for(11)
    lens = [37, 600, 5]
    p = make_paged(rng, 3, 8, 2, 128, lens, 60, wl.F16)
    p.key_cache[:] = p.key_cache[0, 0, 0]
    out = gh.to_f64(gpu_out(p))
    for s, L in enumerate(lens):
        mean = bits_f64(p.v_dense[s, :L], wl.F16).mean(axis=0)  # [Hkv, d]
        assert np.max(np.abs(out[s] - np.repeat(mean, 4, axis=0))) <= gh.TOL[wl.F16]


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2)])
def test_physical_placement_is_invisible_bitwise(hq, hkv):
    """Same logical sequences in a differently ordered pool: identical bits."""
    lens = np.array([700, 17, 1, 48, 1100], np.int32)
    nb = wl.blocks_needed(lens, 16)
    a = make_paged(wl.rng_for(12), 5, hq, hkv, 128, lens, nb, wl.BF16)
    order = wl.draw_block_order(nb, wl.rng_for(99))
    from paged_inputs import tables_from_order
    tb = tables_from_order(lens, order, 16, a.tables.shape[1])
    kc = np.zeros_like(a.key_cache)
    vc = np.zeros_like(a.value_cache)
    for s in range(5):
        n = (int(lens[s]) + 15) // 16
        kc[tb[s, :n]] = a.key_cache[a.tables[s, :n]]
        vc[tb[s, :n]] = a.value_cache[a.tables[s, :n]]
    ra = gh.to_host_bits(gpu_out(a))
    rb = gh.to_host_bits(gh.run_decode(pk, a.q, kc, vc, tb, lens, hkv, a.scale, wl.BF16))
    assert np.array_equal(ra, rb)


def test_runs_on_a_side_stream():
    rng = wl.rng_for(13)
    lens = np.array([900, 33, 1025], np.int32)
    p = make_paged(rng, 3, 8, 2, 128, lens, wl.blocks_needed(lens, 16), wl.F16)
    s = torch.cuda.Stream()
    out = gpu_out(p, stream=s)
    assert gh.max_err(out, oracle_out(p)) <= gh.TOL[wl.F16]


# ---------------------------------------------------------------- scatter write / block copy
@pytest.mark.parametrize("d,dtype", [(64, wl.F16), (128, wl.BF16)])
def test_reshape_and_cache_bit_exact(d, dtype):
    rng = wl.rng_for(14)
    nb, hkv, T = 40, 6, 50
    kc = wl.draw_values(rng, (nb, hkv, 16, d), dtype)
    vc = wl.draw_values(rng, (nb, hkv, 16, d), dtype)
    k = wl.draw_values(rng, (T, hkv, d), dtype)
    v = wl.draw_values(rng, (T, hkv, d), dtype)
    slots = rng.choice(nb * 16, size=T, replace=False).astype(np.int64)
    slots[::7] = -1  # padding entries
    dkc, dvc = gh.to_dev(kc, dtype), gh.to_dev(vc, dtype)
    pk.reshape_and_cache(gh.to_dev(k, dtype), gh.to_dev(v, dtype), dkc, dvc,
                         gh.ints(slots, torch.int64))
    assert pk.get_error() == (0, 0)
    assert oracle.reshape_and_cache(k, v, kc, vc, slots) == 0
    assert np.array_equal(gh.to_host_bits(dkc), kc)
    assert np.array_equal(gh.to_host_bits(dvc), vc)


@pytest.mark.parametrize("d,hkv", [(64, 4), (128, 32)])
def test_copy_blocks_bit_exact(d, hkv):
    rng = wl.rng_for(15)
    nb = 300
    kc = wl.draw_values(rng, (nb, hkv, 16, d), wl.BF16)
    vc = wl.draw_values(rng, (nb, hkv, 16, d), wl.BF16)
    perm = rng.permutation(nb)
    pairs = np.stack([perm[:96], perm[96:192]], axis=1).astype(np.int32)
    dkc, dvc = gh.to_dev(kc, wl.BF16), gh.to_dev(vc, wl.BF16)
    pk.copy_blocks(dkc, dvc, gh.ints(pairs))
    assert pk.get_error() == (0, 0)
    oracle.copy_blocks(kc, vc, pairs)
    assert np.array_equal(gh.to_host_bits(dkc), kc)
    assert np.array_equal(gh.to_host_bits(dvc), vc)


def test_copy_blocks_no_pairs_is_a_no_op():
    kc = torch.zeros((4, 2, 16, 64), dtype=torch.float16, device="cuda")
    pk.copy_blocks(kc, kc.clone(), torch.zeros((0, 2), dtype=torch.int32, device="cuda"))


# ---------------------------------------------------------------- copy-on-write workload (scaled)
def test_parallel_sampling_copy_on_write_steps():
    """Prompts forked into branches through the allocator; every step does the
    copy-on-write copies, writes one token per live branch and decodes; the
    pool and outputs match the oracle replaying the same calls."""
    from paged_kv_cache_425_b200 import batch
    w = wl.scaled(wl.WORKLOADS["cow"], prompts=4, prompt_len=100, own_max=20, num_seqs=16)
    rng = wl.rng_for(16)
    own = wl.draw_branch_tokens(w, rng)
    nb = batch.cow_pool_blocks(w)
    fb = batch.ForkedBatch(w, own, wl.draw_block_order(nb, rng), nb)
    H, d, dt = w.num_kv_heads, w.head_dim, w.dtype
    kc = wl.draw_values(rng, (nb, H, 16, d), dt)
    vc = wl.draw_values(rng, (nb, H, 16, d), dt)
    dkc, dvc = gh.to_dev(kc, dt), gh.to_dev(vc, dt)
    total_pairs = 0
    for step in range(fb.num_steps):
        b = fb.step()
        n = len(b.seq_ids)
        q = wl.draw_values(rng, (n, w.num_q_heads, d), dt)
        k_new = wl.draw_values(rng, (n, H, d), dt)
        v_new = wl.draw_values(rng, (n, H, d), dt)
        if len(b.pairs):
            pk.copy_blocks(dkc, dvc, gh.ints(b.pairs))
            oracle.copy_blocks(kc, vc, b.pairs)
            total_pairs += len(b.pairs)
        pk.reshape_and_cache(gh.to_dev(k_new, dt), gh.to_dev(v_new, dt), dkc, dvc,
                             gh.ints(b.slots, torch.int64))
        oracle.reshape_and_cache(k_new, v_new, kc, vc, b.slots)
        out = gh.run_decode(pk, q, dkc, dvc, b.tables, b.context_lens, H, w.scale, dt)
        ref = oracle.decode(q, kc, vc, b.tables, b.context_lens, H, w.scale, dt)
        assert gh.max_err(out, ref) <= gh.TOL[dt], step
        if step in (0, 1, fb.num_steps - 1):
            assert np.array_equal(gh.to_host_bits(dkc), kc)
            assert np.array_equal(gh.to_host_bits(dvc), vc)
    assert total_pairs == w.prompts * (w.branches - 1)
    assert pk.get_error() == (0, 0)


# ---------------------------------------------------------------- errors
def test_bad_block_id_is_reported_and_skipped():
    rng = wl.rng_for(17)
    lens = np.array([40, 40], np.int32)
    p = make_paged(rng, 2, 4, 4, 64, lens, 6, wl.F16)
    ref = oracle_out(p)
    p.tables[1, 1] = 10_000  # out of the pool
    out = gpu_out(p)
    rc, bits = pk.get_error()
    assert rc == pk.PA_ERR_OUT_OF_RANGE and bits & pk.DEVERR_BLOCK_ID
    assert gh.max_err(out[:1], ref[:1]) <= gh.TOL[wl.F16]  # other sequences unaffected
    assert np.all(np.isfinite(gh.to_f64(out)))
    assert pk.get_error() == (0, 0)  # cleared


def test_bad_slot_and_pair_are_reported():
    kc = torch.zeros((4, 2, 16, 64), dtype=torch.float16, device="cuda")
    vc = torch.zeros_like(kc)
    k = torch.ones((2, 2, 64), dtype=torch.float16, device="cuda")
    pk.reshape_and_cache(k, k, kc, vc, torch.tensor([3, 4 * 16], dtype=torch.int64, device="cuda"))
    rc, bits = pk.get_error()
    assert rc == pk.PA_ERR_OUT_OF_RANGE and bits == pk.DEVERR_SLOT
    assert torch.all(kc.view(-1, 64)[3] == 1) and int((kc != 0).sum()) == 2 * 64
    pk.copy_blocks(kc, vc, torch.tensor([[0, 1], [2, 9]], dtype=torch.int32, device="cuda"))
    rc, bits = pk.get_error()
    assert rc == pk.PA_ERR_OUT_OF_RANGE and bits == pk.DEVERR_PAIR


def test_context_len_beyond_table_is_reported_and_clamped():
    rng = wl.rng_for(18)
    lens = np.array([32, 20], np.int32)
    p = make_paged(rng, 2, 2, 2, 64, lens, 4, wl.F16, max_blocks=2)
    ref = oracle_out(p)
    p.lens = np.array([32, 20 + 1000], np.int32)
    out = gpu_out(p)
    rc, bits = pk.get_error()
    assert rc == pk.PA_ERR_OUT_OF_RANGE and bits & pk.DEVERR_CONTEXT_LEN
    assert gh.max_err(out[:1], ref[:1]) <= gh.TOL[wl.F16]


def test_host_side_rejections():
    q = torch.zeros((2, 4, 96), dtype=torch.float16, device="cuda")
    kc = torch.zeros((4, 4, 16, 96), dtype=torch.float16, device="cuda")
    tb = torch.zeros((2, 40), dtype=torch.int32, device="cuda")
    ln = torch.ones(2, dtype=torch.int32, device="cuda")
    with pytest.raises(pk.PagedError) as e:
        pk.decode(q.clone(), q, kc, kc, tb, ln, 4, 0.1)
    assert e.value.status == pk.PA_ERR_UNSUPPORTED
    q = torch.zeros((2, 4, 64), dtype=torch.float16, device="cuda")
    kc = torch.zeros((4, 4, 16, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(pk.PagedError) as e:  # 40 blocks = 3 partitions, no workspace
        pk.decode(q.clone(), q, kc, kc, tb, ln, 4, 0.1)
    assert e.value.status == pk.PA_ERR_WORKSPACE
    with pytest.raises(pk.PagedError) as e:  # 4 q heads over 3 kv heads
        kc3 = torch.zeros((4, 3, 16, 64), dtype=torch.float16, device="cuda")
        pk.decode(q.clone(), q, kc3, kc3, tb[:, :2].contiguous(), ln, 3, 0.1)
    assert e.value.status == pk.PA_ERR_INVALID_ARG


# ---------------------------------------------------------------- automatic prefix caching
def test_prefix_cached_requests_decode_like_unshared_ones():
    """Requests sharing a 96-token system prompt: the allocator reuses its 6
    cached blocks, K/V are written only for the tokens after them, and every
    request's decode equals attention over its own dense rows."""
    import torch.nn.functional as F
    rng = wl.rng_for(19)
    H, Hq, d, dt, nb = 4, 8, 128, wl.BF16, 200
    a = pk.BlockAllocator(nb)
    a.enable_prefix_caching()
    system = rng.integers(0, 32000, 96).astype(np.int32)
    sys_k = wl.draw_values(rng, (96, H, d), dt)
    sys_v = wl.draw_values(rng, (96, H, d), dt)
    kc = wl.draw_values(rng, (nb, H, 16, d), dt)
    vc = wl.draw_values(rng, (nb, H, 16, d), dt)
    dkc, dvc = gh.to_dev(kc, dt), gh.to_dev(vc, dt)
    dense_k, dense_v = [], []
    for r in range(5):
        n_user = int(rng.integers(1, 100))
        toks = np.concatenate([system, rng.integers(0, 32000, n_user).astype(np.int32)])
        k_rows = np.concatenate([sys_k, wl.draw_values(rng, (n_user, H, d), dt)])
        v_rows = np.concatenate([sys_v, wl.draw_values(rng, (n_user, H, d), dt)])
        cached = a.add_seq_tokens(r, toks)
        assert cached == (0 if r == 0 else 96)
        t = a.block_table(r)
        pos = np.arange(cached, len(toks))
        slots = (t[pos // 16].astype(np.int64) * 16 + pos % 16)
        pk.reshape_and_cache(gh.to_dev(k_rows[cached:], dt), gh.to_dev(v_rows[cached:], dt), dkc,
                             dvc, gh.ints(slots, torch.int64))
        oracle.reshape_and_cache(k_rows[cached:], v_rows[cached:], kc, vc, slots)
        dense_k.append(k_rows)
        dense_v.append(v_rows)
    tables, lens = a.build_tables(np.arange(5), 16)
    q = wl.draw_values(rng, (5, Hq, d), dt)
    out = gh.run_decode(pk, q, dkc, dvc, tables, lens, H, 1 / np.sqrt(d), dt)
    assert pk.get_error() == (0, 0)
    assert np.array_equal(gh.to_host_bits(dkc), kc)
    ref = oracle.decode(q, kc, vc, tables, lens, H, 1 / np.sqrt(d), dt)
    assert gh.max_err(out, ref) <= gh.TOL[dt]
    for r in range(5):
        qq = torch.from_numpy(bits_f64(q[r], dt)).reshape(1, Hq, 1, d)
        kk = torch.from_numpy(bits_f64(dense_k[r], dt)).permute(1, 0, 2).unsqueeze(0)
        vv = torch.from_numpy(bits_f64(dense_v[r], dt)).permute(1, 0, 2).unsqueeze(0)
        dense = F.scaled_dot_product_attention(qq, kk, vv, scale=1 / np.sqrt(d), enable_gqa=True)
        assert gh.max_err(out[r], dense.reshape(Hq, d).numpy()) <= gh.TOL[dt]
    assert a.stats()["prefix_hit_blocks"] == 4 * 6


# ---------------------------------------------------------------- swap out / swap in
@pytest.mark.parametrize("pinned", [True, False], ids=["pinned-kernel", "pageable-copies"])
def test_swap_out_and_back_in_is_bit_exact_and_decode_follows(pinned):
    """A sequence's blocks go to a host pool and come back into other device
    blocks; the bytes round-trip exactly and decode through the remapped
    table gives the same bits as before.  A pinned pool takes the kernel
    path, a pageable one the per-run copy path."""
    rng = wl.rng_for(20)
    H, d, dt = 8, 128, wl.BF16
    lens = np.array([300, 77], np.int32)
    nb = 64
    p = make_paged(rng, 2, 16, H, d, lens, nb, dt)
    before = gh.to_host_bits(gpu_out(p))
    dkc, dvc = gh.to_dev(p.key_cache, dt), gh.to_dev(p.value_cache, dt)
    host_k = torch.zeros((40, H, 16, d), dtype=torch.bfloat16)
    host_v = torch.zeros_like(host_k)
    if pinned:
        host_k, host_v = host_k.pin_memory(), host_v.pin_memory()
    n0 = (int(lens[0]) + 15) // 16
    out_pairs = np.stack([p.tables[0, :n0], 5 + np.arange(n0)], axis=1).astype(np.int32)
    pk.swap_blocks(dkc, dvc, host_k, host_v, out_pairs)
    torch.cuda.synchronize()
    hk = host_k.view(torch.int16).numpy().view(np.uint16)
    hv = host_v.view(torch.int16).numpy().view(np.uint16)
    # the whole host pool: the swapped blocks at their destinations, zeros elsewhere
    want_hk = np.zeros_like(hk)
    want_hv = np.zeros_like(hv)
    for src, dst in out_pairs:
        want_hk[dst] = p.key_cache[src]
        want_hv[dst] = p.value_cache[src]
    assert np.array_equal(hk, want_hk) and np.array_equal(hv, want_hv)
    # back into device blocks no table uses (sequence 1 keeps its blocks)
    used = set(p.tables[:, :].ravel().tolist())
    free = np.array([b for b in range(nb) if b not in used][:n0] if nb - len(used) >= n0 else [], np.int32)
    if len(free) < n0:  # reuse sequence 0's own old blocks in reverse order
        free = p.tables[0, :n0][::-1].copy()
    in_pairs = np.stack([5 + np.arange(n0), free], axis=1).astype(np.int32)
    pk.swap_blocks(host_k, host_v, dkc, dvc, in_pairs)
    torch.cuda.synchronize()
    # the whole device pool: the destination blocks hold exactly the host
    # bytes, every other block keeps its own
    want_k, want_v = p.key_cache.copy(), p.value_cache.copy()
    for src, dst in in_pairs:
        want_k[dst] = want_hk[src]
        want_v[dst] = want_hv[src]
    assert np.array_equal(gh.to_host_bits(dkc), want_k)
    assert np.array_equal(gh.to_host_bits(dvc), want_v)
    tables = p.tables.copy()
    tables[0, :n0] = free
    after = gh.to_host_bits(gh.run_decode(pk, p.q, dkc, dvc, tables, lens, H, p.scale, dt))
    assert np.array_equal(before, after)
    with pytest.raises(pk.PagedError) as e:
        pk.swap_blocks(dkc, dvc, host_k, host_v, np.array([[0, 40]], np.int32))
    assert e.value.status == pk.PA_ERR_OUT_OF_RANGE


# ---------------------------------------------------------------- chunked prefill
@pytest.fixture(params=["mma_sync", "tcgen05"])
def prefill_kernel(request):
    """Run the test on each prefill kernel, then restore the default."""
    pk.prefill_select(request.param)
    yield request.param
    pk.prefill_select("auto")


def poisoned(p):
    """Copies of p's pools with every row that holds no token of any
    sequence (unused blocks, tails of last blocks) set to NaN."""
    live = np.zeros(p.key_cache.shape[:1] + p.key_cache.shape[2:3], bool)  # [block, slot]
    for s, L in enumerate(p.lens):
        for t in range(int(L)):
            live[p.tables[s, t // 16], t % 16] = True
    nan = np.uint16(0x7E00 if p.dtype == wl.F16 else 0x7FC0)
    kc, vc = p.key_cache.copy(), p.value_cache.copy()
    dead = ~live
    kc.transpose(0, 2, 1, 3)[dead] = nan
    vc.transpose(0, 2, 1, 3)[dead] = nan
    return kc, vc


def run_prefill(p, qchunk, qlens, max_query_len=None, pools=None):
    qs = np.zeros(len(qlens) + 1, np.int32)
    qs[1:] = np.cumsum(qlens)
    q = gh.to_dev(qchunk, p.dtype)
    out = torch.full_like(q, float("nan"))
    kc, vc = pools if pools is not None else (p.key_cache, p.value_cache)
    pk.prefill(out, q, gh.to_dev(kc, p.dtype), gh.to_dev(vc, p.dtype),
               gh.ints(p.tables), gh.ints(p.lens), gh.ints(qs),
               int(max(qlens)) if max_query_len is None else max_query_len, p.num_kv_heads,
               p.scale)
    torch.cuda.synchronize()
    ref = oracle.prefill(qchunk, p.key_cache, p.value_cache, p.tables, p.lens, qs,
                         p.num_kv_heads, p.scale, p.dtype)
    return out, ref


@pytest.mark.parametrize("hq,hkv,d,dtype", [(4, 4, 64, wl.F16), (8, 2, 128, wl.BF16),
                                            (32, 8, 128, wl.BF16), (8, 1, 64, wl.F16),
                                            (16, 16, 128, wl.F16)])
def test_prefill_matches_oracle(hq, hkv, d, dtype, prefill_kernel):
    rng = wl.rng_for(40 + hq + d)
    lens = np.array([40, 700, 17, 64, 5, 1, 513], np.int32)
    qlens = np.array([40, 300, 1, 16, 5, 1, 77], np.int32)  # whole prompts, chunks, single tokens
    p = make_paged(rng, len(lens), hq, hkv, d, lens, wl.blocks_needed(lens, 16) + 3, dtype)
    qchunk = wl.draw_values(rng, (int(qlens.sum()), hq, d), dtype)
    out, ref = run_prefill(p, qchunk, qlens)
    assert pk.get_error() == (0, 0)
    assert gh.max_excess(out, ref, dtype) <= gh.TOL[dtype]


def test_prefill_one_token_chunks_agree_with_decode(prefill_kernel):
    rng = wl.rng_for(41)
    lens = np.array([33, 1, 1200, 512], np.int32)
    p = make_paged(rng, 4, 8, 2, 128, lens, wl.blocks_needed(lens, 16), wl.BF16)
    out, ref = run_prefill(p, p.q, np.ones(4, np.int32))
    dec = gpu_out(p)
    assert gh.max_excess(out, ref, wl.BF16) <= gh.TOL[wl.BF16]
    assert float((out.float() - dec.float()).abs().max()) <= gh.TOL[wl.BF16]


def test_prefill_long_contexts_and_slack_grid(prefill_kernel):
    """Chunks of 512 over contexts up to 4k, with a grid sized for a larger
    max_query_len than any sequence uses."""
    rng = wl.rng_for(42)
    lens = np.array([4096, 1024, 2600], np.int32)
    qlens = np.array([512, 512, 100], np.int32)
    p = make_paged(rng, 3, 32, 8, 128, lens, wl.blocks_needed(lens, 16) + 1, wl.BF16)
    qchunk = wl.draw_values(rng, (int(qlens.sum()), 32, 128), wl.BF16)
    out, ref = run_prefill(p, qchunk, qlens, max_query_len=900)
    assert gh.max_excess(out, ref, wl.BF16) <= gh.TOL[wl.BF16]


def test_prefill_chunk_longer_than_context_is_reported(prefill_kernel):
    rng = wl.rng_for(43)
    lens = np.array([20, 30], np.int32)
    p = make_paged(rng, 2, 4, 4, 64, lens, 4, wl.F16)
    qlens = np.array([25, 30], np.int32)  # 25 > 20: clamped, flagged
    qchunk = wl.draw_values(rng, (55, 4, 64), wl.F16)
    qs = np.array([0, 25, 55], np.int32)
    q = gh.to_dev(qchunk, wl.F16)
    out = torch.zeros_like(q)
    pk.prefill(out, q, gh.to_dev(p.key_cache, wl.F16), gh.to_dev(p.value_cache, wl.F16),
               gh.ints(p.tables), gh.ints(p.lens), gh.ints(qs), 30, 4, p.scale)
    rc, bits = pk.get_error()
    assert rc == pk.PA_ERR_OUT_OF_RANGE and bits & pk.DEVERR_CONTEXT_LEN
    ref = oracle.prefill(qchunk[25:], p.key_cache, p.value_cache, p.tables[1:], p.lens[1:],
                         np.array([0, 30], np.int32), 4, p.scale, wl.F16)
    assert gh.max_excess(out[25:], ref, wl.F16) <= gh.TOL[wl.F16]


@pytest.mark.parametrize("hq,hkv", [(12, 4), (40, 8), (16, 1), (64, 2)])
def test_prefill_groups_that_do_not_divide_the_tile(hq, hkv, prefill_kernel):
    """Query groups of 3, 5, 16 and 32 heads: the tcgen05 tile holds the
    largest multiple of the group that fits 128 rows (126, 125, 128, 128)."""
    rng = wl.rng_for(44 + hq)
    lens = np.array([300, 77, 1000], np.int32)
    qlens = np.array([300, 50, 129], np.int32)
    p = make_paged(rng, 3, hq, hkv, 128, lens, wl.blocks_needed(lens, 16) + 2, wl.BF16)
    qchunk = wl.draw_values(rng, (int(qlens.sum()), hq, 128), wl.BF16)
    out, ref = run_prefill(p, qchunk, qlens)
    assert pk.get_error() == (0, 0)
    assert gh.max_excess(out, ref, wl.BF16) <= gh.TOL[wl.BF16]


@pytest.mark.parametrize("d,dtype", [(128, wl.BF16), (64, wl.F16)])
def test_prefill_ignores_nan_in_rows_without_tokens(d, dtype, prefill_kernel):
    """Every pool row that holds no token (unused blocks, the tail of each
    last block) is NaN in K and V; the outputs must not see it."""
    rng = wl.rng_for(45 + d)
    lens = np.array([130, 17, 700, 1, 260], np.int32)
    qlens = np.array([130, 3, 200, 1, 60], np.int32)
    p = make_paged(rng, 5, 8, 2, d, lens, wl.blocks_needed(lens, 16) + 4, dtype)
    qchunk = wl.draw_values(rng, (int(qlens.sum()), 8, d), dtype)
    out, ref = run_prefill(p, qchunk, qlens, pools=poisoned(p))
    assert pk.get_error() == (0, 0)
    assert gh.max_excess(out, ref, dtype) <= gh.TOL[dtype]


def test_prefill_bad_block_id_is_reported(prefill_kernel):
    """An out-of-range id inside one sequence's range raises
    PA_DEVERR_BLOCK_ID; the other sequences are still exact."""
    rng = wl.rng_for(46)
    lens = np.array([200, 300], np.int32)
    qlens = np.array([64, 100], np.int32)
    p = make_paged(rng, 2, 8, 2, 128, lens, wl.blocks_needed(lens, 16), wl.BF16)
    p.tables[0, 3] = p.key_cache.shape[0] + 7
    qchunk = wl.draw_values(rng, (int(qlens.sum()), 8, 128), wl.BF16)
    qs = np.array([0, 64, 164], np.int32)
    q = gh.to_dev(qchunk, wl.BF16)
    out = torch.zeros_like(q)
    pk.prefill(out, q, gh.to_dev(p.key_cache, wl.BF16), gh.to_dev(p.value_cache, wl.BF16),
               gh.ints(p.tables), gh.ints(p.lens), gh.ints(qs), 100, 2, p.scale)
    rc, bits = pk.get_error()
    assert rc == pk.PA_ERR_OUT_OF_RANGE and bits & pk.DEVERR_BLOCK_ID
    ref = oracle.prefill(qchunk[64:], p.key_cache, p.value_cache, p.tables[1:], p.lens[1:],
                         np.array([0, 100], np.int32), 2, p.scale, wl.BF16)
    assert gh.max_excess(out[64:], ref, wl.BF16) <= gh.TOL[wl.BF16]


def test_prefill_wide_block_tables(prefill_kernel):
    """Block tables 9000 entries wide (144,000 tokens of room), contexts up to
    3000 tokens: the tcgen05 kernel reads block ids from the table in global
    memory, so the width is not limited by shared memory."""
    rng = wl.rng_for(68)
    lens = np.array([3000, 700, 129], np.int32)
    qlens = np.array([200, 64, 129], np.int32)
    p = make_paged(rng, 3, 16, 4, 128, lens, wl.blocks_needed(lens, 16) + 2, wl.BF16,
                   max_blocks=9000)
    assert p.tables.shape == (3, 9000)
    qchunk = wl.draw_values(rng, (int(qlens.sum()), 16, 128), wl.BF16)
    out, ref = run_prefill(p, qchunk, qlens)
    assert pk.get_error() == (0, 0)
    assert gh.max_excess(out, ref, wl.BF16) <= gh.TOL[wl.BF16]


def test_prefill_output_aligned_to_16_bytes_only(prefill_kernel):
    """q and out start 16 bytes into their buffers: 16-byte aligned, not
    32.  The tcgen05 kernel then stores its rows in 16-byte pieces instead
    of 32-byte ones; results are the same, and nothing around out changes."""
    rng = wl.rng_for(48)
    lens = np.array([300, 77, 1000], np.int32)
    qlens = np.array([300, 50, 129], np.int32)
    hq, hkv, d = 16, 4, 128
    p = make_paged(rng, 3, hq, hkv, d, lens, wl.blocks_needed(lens, 16) + 2, wl.BF16)
    T = int(qlens.sum())
    qchunk = wl.draw_values(rng, (T, hq, d), wl.BF16)
    n = T * hq * d
    qbuf = torch.zeros(n + 16, dtype=torch.bfloat16, device="cuda")
    qbuf[8:8 + n] = gh.to_dev(qchunk, wl.BF16).reshape(-1)
    obuf = torch.full((n + 16,), float("nan"), dtype=torch.bfloat16, device="cuda")
    q, out = qbuf[8:8 + n].view(T, hq, d), obuf[8:8 + n].view(T, hq, d)
    assert out.data_ptr() % 16 == 0 and out.data_ptr() % 32 != 0
    qs = np.zeros(4, np.int32)
    qs[1:] = np.cumsum(qlens)
    pk.prefill(out, q, gh.to_dev(p.key_cache, wl.BF16), gh.to_dev(p.value_cache, wl.BF16),
               gh.ints(p.tables), gh.ints(p.lens), gh.ints(qs), int(qlens.max()), hkv, p.scale)
    torch.cuda.synchronize()
    assert pk.get_error() == (0, 0)
    ref = oracle.prefill(qchunk, p.key_cache, p.value_cache, p.tables, p.lens, qs, hkv,
                         p.scale, wl.BF16)
    assert gh.max_excess(out, ref, wl.BF16) <= gh.TOL[wl.BF16]
    assert torch.isnan(obuf[:8]).all() and torch.isnan(obuf[8 + n:]).all()


@pytest.mark.parametrize("num_seqs", [40, 300])
def test_prefill_many_sequences_with_equal_lengths(num_seqs, prefill_kernel):
    """Many sequences, lengths repeating (ties in the longest-first CTA
    order); 300 sequences is past the size the tcgen05 kernel ranks, which
    then keeps the plain order."""
    rng = wl.rng_for(49 + num_seqs)
    lens = np.array([(17, 200, 64, 1, 130)[i % 5] for i in range(num_seqs)], np.int32)
    qlens = np.minimum(lens, np.array([(5, 64, 64, 1, 40)[i % 5] for i in range(num_seqs)], np.int32))
    p = make_paged(rng, num_seqs, 8, 2, 64, lens, wl.blocks_needed(lens, 16) + 1, wl.F16)
    qchunk = wl.draw_values(rng, (int(qlens.sum()), 8, 64), wl.F16)
    out, ref = run_prefill(p, qchunk, qlens)
    assert pk.get_error() == (0, 0)
    assert gh.max_excess(out, ref, wl.F16) <= gh.TOL[wl.F16]


def test_prefill_kernels_agree():
    """The two prefill kernels on one problem: both within the budget of
    the oracle, and within twice that budget of each other."""
    rng = wl.rng_for(47)
    lens = np.array([2048, 900, 513], np.int32)
    qlens = np.array([512, 512, 513], np.int32)
    p = make_paged(rng, 3, 32, 8, 128, lens, wl.blocks_needed(lens, 16), wl.BF16)
    qchunk = wl.draw_values(rng, (int(qlens.sum()), 32, 128), wl.BF16)
    outs = {}
    try:
        for k in ("mma_sync", "tcgen05"):
            pk.prefill_select(k)
            outs[k], ref = run_prefill(p, qchunk, qlens)
            assert gh.max_excess(outs[k], ref, wl.BF16) <= gh.TOL[wl.BF16], k
    finally:
        pk.prefill_select("auto")
    diff = (outs["mma_sync"].double() - outs["tcgen05"].double()).abs()
    lim = 2 * (gh.TOL[wl.BF16] + gh.REL[wl.BF16] * torch.from_numpy(np.abs(ref)).cuda())
    assert bool((diff <= lim).all())


def test_decode_ignores_nan_in_rows_without_tokens():
    """Decode on a pool whose token-free rows are NaN: every kernel (one
    query head per kv head, grouped, split contexts) must not see it."""
    for hq, hkv, dtype in ((8, 8, wl.F16), (16, 2, wl.BF16)):
        rng = wl.rng_for(48 + hq)
        lens = np.array([1, 17, 513, 1500, 33, 1024], np.int32)
        p = make_paged(rng, 6, hq, hkv, 128, lens, wl.blocks_needed(lens, 16) + 5, dtype)
        kc, vc = poisoned(p)
        out = gh.run_decode(pk, p.q, kc, vc, p.tables, p.lens, hkv, p.scale, dtype)
        assert pk.get_error() == (0, 0)
        assert gh.max_err(out, oracle_out(p)) <= gh.TOL[dtype]


# ---------------------------------------------------------------- CUDA graph capture
def test_decode_step_replays_from_a_cuda_graph():
    """Scatter + decode (split contexts, so the merge runs too) captured once
    in a CUDA graph, with the kernels chained by programmatic dependent
    launch; replays reproduce the eager results bit for bit."""
    rng = wl.rng_for(50)
    lens = np.array([900, 33, 2049, 512], np.int32)
    p = make_paged(rng, 4, 8, 2, 128, lens, wl.blocks_needed(lens, 16) + 2, wl.BF16)
    dkc, dvc = gh.to_dev(p.key_cache, wl.BF16), gh.to_dev(p.value_cache, wl.BF16)
    q = gh.to_dev(p.q, wl.BF16)
    k_new = gh.to_dev(wl.draw_values(rng, (4, 2, 128), wl.BF16), wl.BF16)
    v_new = gh.to_dev(wl.draw_values(rng, (4, 2, 128), wl.BF16), wl.BF16)
    pos = lens - 1
    slots = gh.ints(np.array([p.tables[s, pos[s] // 16] * 16 + pos[s] % 16 for s in range(4)]),
                    torch.int64)
    tables, ln = gh.ints(p.tables), gh.ints(lens)
    ws = gh.workspace_for(pk, 4, 8, 128, p.tables.shape[1])
    out = torch.zeros_like(q)
    stream = torch.cuda.Stream()

    def step():
        pk.reshape_and_cache(k_new, v_new, dkc, dvc, slots, stream=stream)
        pk.decode(out, q, dkc, dvc, tables, ln, 2, p.scale, workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    eager = out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
    assert pk.get_error() == (0, 0)


# ---------------------------------------------------------------- bounded waits
def test_a_wait_that_never_completes_times_out_and_the_context_survives():
    """The bounded mbarrier wait every kernel uses gives up (1 ms here), sets
    the timeout bit, and leaves the context usable for the next call."""
    assert pk.get_error() == (0, 0)
    pk.selftest_wait_timeout(1_000_000)
    rc, bits = pk.get_error()
    assert rc == pk.PA_ERR_TIMEOUT and bits == pk.DEVERR_TIMEOUT
    assert pk.get_error() == (0, 0)
    rng = wl.rng_for(60)
    lens = np.array([600, 20], np.int32)
    p = make_paged(rng, 2, 8, 2, 128, lens, wl.blocks_needed(lens, 16), wl.BF16)
    assert gh.max_err(gpu_out(p), oracle_out(p)) <= gh.TOL[wl.BF16]


# ---------------------------------------------------------------- seeded random configurations
def random_config(seed):
    """A seeded random problem: group size, head dim, dtype, kv heads, batch
    size and context lengths (empty, short, block-aligned, multi-partition)."""
    rng = wl.rng_for(900 + seed)
    G = int(rng.choice([1, 2, 3, 4, 5, 8, 12, 16]))
    hkv = int(rng.choice([1, 2, 4, 8]))
    d = int(rng.choice([64, 128]))
    dtype = wl.F16 if rng.random() < 0.5 else wl.BF16
    S = int(rng.integers(1, 12))
    kinds = rng.integers(0, 4, size=S)
    lens = np.where(kinds == 0, rng.integers(0, 17, size=S),
                    np.where(kinds == 1, 16 * rng.integers(1, 40, size=S),
                             np.where(kinds == 2, rng.integers(17, 600, size=S),
                                      rng.integers(600, 2500, size=S)))).astype(np.int32)
    return rng, G * hkv, hkv, d, dtype, lens


@pytest.mark.parametrize("seed", range(12))
def test_random_configs_decode_append(seed):
    """pa_decode_append and pa_reshape_and_cache + pa_decode on seeded random
    configurations: equal to each other bit for bit, and to the oracle."""
    rng, hq, hkv, d, dtype, lens = random_config(seed)
    S = len(lens)
    p = make_paged(rng, S, hq, hkv, d, lens, wl.blocks_needed(lens, 16) + 3, dtype)
    k_new = wl.draw_values(rng, (S, hkv, d), dtype)
    v_new = wl.draw_values(rng, (S, hkv, d), dtype)
    slots = append_slots(p)
    tbl, ln = gh.ints(p.tables), gh.ints(p.lens)
    dk, dv, q = gh.to_dev(k_new, dtype), gh.to_dev(v_new, dtype), gh.to_dev(p.q, dtype)
    ws = gh.workspace_for(pk, S, hq, d, p.tables.shape[1])
    kc1, vc1 = gh.to_dev(p.key_cache, dtype), gh.to_dev(p.value_cache, dtype)
    out1 = torch.full_like(q, float("nan"))
    pk.reshape_and_cache(dk, dv, kc1, vc1, gh.ints(slots, torch.int64))
    pk.decode(out1, q, kc1, vc1, tbl, ln, hkv, p.scale, workspace=ws)
    kc2, vc2 = gh.to_dev(p.key_cache, dtype), gh.to_dev(p.value_cache, dtype)
    out2 = torch.full_like(q, float("nan"))
    pk.decode_append(out2, q, dk, dv, kc2, vc2, tbl, ln, hkv, p.scale, workspace=ws)
    torch.cuda.synchronize()
    assert pk.get_error() == (0, 0)
    assert torch.equal(kc1, kc2) and torch.equal(vc1, vc2) and torch.equal(out1, out2)
    oracle.reshape_and_cache(k_new, v_new, p.key_cache, p.value_cache, slots)
    assert np.array_equal(gh.to_host_bits(kc2), p.key_cache)
    assert gh.max_err(out2, oracle_out(p)) <= gh.TOL[dtype]


@pytest.mark.parametrize("seed", range(8))
def test_random_configs_prefill(seed, prefill_kernel):
    """Chunked prefill on seeded random configurations (chunks from one token
    to the whole context), on both kernels, against the oracle."""
    rng, hq, hkv, d, dtype, lens = random_config(seed)
    lens = np.maximum(lens, 1)
    qlens = np.array([int(rng.integers(1, L + 1)) if rng.random() < 0.7 else int(L) for L in lens],
                     np.int32)
    qlens = np.minimum(qlens, 300).astype(np.int32)
    p = make_paged(rng, len(lens), hq, hkv, d, lens, wl.blocks_needed(lens, 16) + 3, dtype)
    qchunk = wl.draw_values(rng, (int(qlens.sum()), hq, d), dtype)
    out, ref = run_prefill(p, qchunk, qlens)
    assert pk.get_error() == (0, 0)
    assert gh.max_excess(out, ref, dtype) <= gh.TOL[dtype]
