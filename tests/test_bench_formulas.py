"""The bench's algorithmic-bytes and FLOP formulas against brute-force counts."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_decode_bytes_count_every_token_once():
    lens = np.array([1, 16, 17, 1000], np.int64)
    Hq, Hkv, d = 8, 2, 128
    brute = 0
    for L in lens:
        brute += L * Hkv * d * 2 * 2          # K and V rows of every cached token
        brute += -(-L // 16) * 4              # table entries read
        brute += 4                            # context length
    brute += 2 * len(lens) * Hq * d * 2       # q and out
    assert bench.algorithmic_bytes(lens, Hq, Hkv, d) == brute


def test_append_bytes_add_the_new_rows_of_non_empty_sequences():
    """pa_decode_append also reads each sequence's new K and V rows and writes
    them into the cache; an empty sequence (L = 0) writes nothing."""
    lens = np.array([0, 1, 16, 17, 1000], np.int64)
    Hq, Hkv, d = 8, 2, 128
    rows = 0
    for L in lens:
        if L > 0:
            rows += 2 * Hkv * d * 2 * 2       # K and V rows: read k_new / v_new, write the cache
    assert (bench.algorithmic_bytes(lens, Hq, Hkv, d, append=True)
            == bench.algorithmic_bytes(lens, Hq, Hkv, d) + rows)


def test_prefill_flops_match_a_per_query_count():
    lens = np.array([512, 700, 3000], np.int64)
    chunk, Hq, d = 512, 32, 128
    brute = 0
    for L in lens:
        for i in range(chunk):
            keys = L - chunk + i + 1
            brute += 2 * keys * d * Hq * 2    # q.K and P.V, a multiply-add = 2 FLOPs
    assert bench.prefill_flops(lens, chunk, Hq, d) == brute


def _up(x):
    return (x + 255) // 256 * 256


def test_reported_partitions_follow_the_library_rule():
    """bench.decode_partitions (reported in the config) against the partition
    count the library's workspace size implies, across the wide-table
    threshold (512-token partitions below 16384 tokens, 1024 above)."""
    import pytest
    pk = pytest.importorskip("paged_kv_cache_425_b200")
    for max_blocks in list(range(1, 70)) + [127, 128, 129, 255, 256, 257, 1023, 1024, 1025, 2048]:
        ws = pk.decode_workspace_size(1, 1, 128, max_blocks)
        if ws == 0:
            parts = 1
        else:  # one row: fp32 partials [P][128], then (max, sum) [P], each 256-aligned
            parts = next(p for p in range(2, 9000) if _up(p * 512) + _up(p * 8) == ws)
        assert bench.decode_partitions(max_blocks) == parts, max_blocks


def test_cpu_arm_tables_are_valid_and_its_config_matches_the_gpu_arms():
    """The reference arm builds its tables with numpy.  They must be valid
    tables for the drawn lengths, and both arms must describe the workload
    with the same config (same lengths, pool, partitions, copy pairs)."""
    import pytest
    import workloads as wl
    pytest.importorskip("paged_kv_cache_425_b200")
    from paged_kv_cache_425_b200 import batch
    for name in ("tiny", "llama7b", "llama13b", "gqa_long", "cow"):
        w = wl.WORKLOADS[name]
        lens, nb, tables = bench.host_tables(w, 0)
        need = (lens.astype(np.int64) + 15) // 16
        for s, n in enumerate(need):
            row = tables[s]
            assert np.all((row[:n] >= 0) & (row[:n] < nb)) and np.all(row[n:] == -1), (name, s)
        if name != "cow":  # no sharing: every physical block is used once
            used = tables[tables >= 0]
            assert len(np.unique(used)) == len(used), name
        # the GPU arm's batch, from the allocator and the same draws
        rng = wl.rng_for(0)
        if name == "cow":
            own = wl.draw_branch_tokens(w, rng)
            gnb = batch.cow_pool_blocks(w)
            b = batch.ForkedBatch(w, own, wl.draw_block_order(gnb, rng), gnb).step()
            assert len(b.pairs) == bench.cow_pairs(w)
        else:
            glens = wl.draw_context_lens(w, rng)
            gnb = wl.pool_size(w, glens)
            b = batch.decode_batch(w, glens, wl.draw_block_order(gnb, rng), gnb,
                                   batch.max_blocks_for(w))
        assert np.array_equal(b.context_lens, lens), name
        assert bench.describe(w, b.context_lens, b.num_blocks, b.max_blocks) == \
            bench.describe(w, lens, nb, tables.shape[1]), name
