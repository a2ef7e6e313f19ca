"""Full-size parity: every workload at its real size, built by the host
allocator exactly as bench.py builds it, one layer per call.

The scatter write is checked bit for bit on every written row and on a
sample of untouched blocks; decode outputs are compared with the fp64 oracle
on sampled sequences (all sequences where the oracle finishes in seconds).
"""
import numpy as np
import pytest

import oracle
import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu, pytest.mark.slow]

import gpu_harness as gh  # noqa: E402

pk = pytest.importorskip("paged_kv_cache_425_b200")
from paged_kv_cache_425_b200 import batch  # noqa: E402


def host_pool(rng, nb, w):
    kc = wl.draw_values(rng, (nb, w.num_kv_heads, 16, w.head_dim), w.dtype)
    vc = wl.draw_values(rng, (nb, w.num_kv_heads, 16, w.head_dim), w.dtype)
    return kc, vc


def check_rows(dev_cache, host_cache, slots, rng, nb):
    """Written rows and a random sample of blocks, bit for bit."""
    for s in slots[slots >= 0][:256]:
        b, o = int(s) // 16, int(s) % 16
        assert np.array_equal(gh.to_host_bits(dev_cache[b, :, o]), host_cache[b, :, o])
    for b in rng.choice(nb, size=min(nb, 64), replace=False):
        assert np.array_equal(gh.to_host_bits(dev_cache[int(b)]), host_cache[int(b)])


def run_decode_step(w, b, rng, seqs):
    """Scatter + decode through the C ABI at full size; oracle on `seqs`."""
    nb, dt = b.num_blocks, w.dtype
    S = len(b.seq_ids)
    kc, vc = host_pool(rng, nb, w)
    q = wl.draw_values(rng, (S, w.num_q_heads, w.head_dim), dt)
    k_new = wl.draw_values(rng, (S, w.num_kv_heads, w.head_dim), dt)
    v_new = wl.draw_values(rng, (S, w.num_kv_heads, w.head_dim), dt)
    dkc, dvc = gh.to_dev(kc, dt), gh.to_dev(vc, dt)
    if len(b.pairs):
        pk.copy_blocks(dkc, dvc, gh.ints(b.pairs))
        oracle.copy_blocks(kc, vc, b.pairs)
    pk.reshape_and_cache(gh.to_dev(k_new, dt), gh.to_dev(v_new, dt), dkc, dvc,
                         gh.ints(b.slots, torch.int64))
    out = gh.run_decode(pk, q, dkc, dvc, b.tables, b.context_lens, w.num_kv_heads, w.scale, dt)
    assert pk.get_error() == (0, 0)
    oracle.reshape_and_cache(k_new, v_new, kc, vc, b.slots)
    check_rows(dkc, kc, b.slots, rng, nb)
    check_rows(dvc, vc, b.slots, rng, nb)
    if len(b.pairs):
        for src, dst in b.pairs[:16]:
            assert np.array_equal(gh.to_host_bits(dkc[int(dst)]), kc[int(dst)])
    ref = oracle.decode(q, kc, vc, b.tables, b.context_lens, w.num_kv_heads, w.scale, dt,
                        seqs=seqs)
    err = gh.max_err(out[torch.from_numpy(seqs).long().cuda()], ref)
    assert err <= gh.TOL[dt], err
    return err, dkc, dvc, kc, vc


def decode_batch_for(name):
    w = wl.WORKLOADS[name]
    rng = wl.rng_for(0)
    lens = wl.draw_context_lens(w, rng)
    nb = wl.pool_size(w, lens)
    b = batch.decode_batch(w, lens, wl.draw_block_order(nb, rng), nb, batch.max_blocks_for(w))
    return w, b, rng


def test_llama7b_full_layer_all_sequences():
    w, b, rng = decode_batch_for("llama7b")
    run_decode_step(w, b, rng, np.arange(w.num_seqs, dtype=np.int32))


def test_llama13b_full_layer_sampled_sequences():
    w, b, rng = decode_batch_for("llama13b")
    lens = b.context_lens
    pick = np.unique(np.concatenate([np.argsort(lens)[-3:], np.argsort(lens)[:2],
                                     rng.choice(len(lens), 5, replace=False)])).astype(np.int32)
    run_decode_step(w, b, rng, pick)


def test_gqa_long_full_call_sampled_sequences():
    w, b, rng = decode_batch_for("gqa_long")
    lens = b.context_lens
    pick = np.unique(np.array([np.argmax(lens), np.argmin(lens), 3, 17], np.int32))
    run_decode_step(w, b, rng, pick)


def test_cow_divergence_and_following_steps_full_size():
    w = wl.WORKLOADS["cow"]
    rng = wl.rng_for(0)
    own = wl.draw_branch_tokens(w, rng)
    nb = batch.cow_pool_blocks(w)
    fb = batch.ForkedBatch(w, own, wl.draw_block_order(nb, rng), nb)
    b = fb.step()
    assert len(b.pairs) == 96
    err, dkc, dvc, kc, vc = run_decode_step(w, b, rng, np.arange(128, dtype=np.int32))
    # two more steps on the same pool: no sharing is left, so no copies
    for _ in range(2):
        b = fb.step()
        assert len(b.pairs) == 0
        S = len(b.seq_ids)
        q = wl.draw_values(rng, (S, w.num_q_heads, w.head_dim), w.dtype)
        k_new = wl.draw_values(rng, (S, w.num_kv_heads, w.head_dim), w.dtype)
        v_new = wl.draw_values(rng, (S, w.num_kv_heads, w.head_dim), w.dtype)
        pk.reshape_and_cache(gh.to_dev(k_new, w.dtype), gh.to_dev(v_new, w.dtype), dkc, dvc,
                             gh.ints(b.slots, torch.int64))
        oracle.reshape_and_cache(k_new, v_new, kc, vc, b.slots)
        out = gh.run_decode(pk, q, dkc, dvc, b.tables, b.context_lens, w.num_kv_heads, w.scale,
                            w.dtype)
        sel = np.arange(0, S, 4, dtype=np.int32)
        ref = oracle.decode(q, kc, vc, b.tables, b.context_lens, w.num_kv_heads, w.scale,
                            w.dtype, seqs=sel)
        assert gh.max_err(out[torch.from_numpy(sel).long().cuda()], ref) <= gh.TOL[w.dtype]
    assert np.array_equal(gh.to_host_bits(dkc), kc)
    assert np.array_equal(gh.to_host_bits(dvc), vc)


def test_prefill_workload_full_size_sampled_sequences():
    """16 sequences x 512-token chunks over contexts U{512..4096} (32 q / 8 kv
    heads, bf16), tables from the allocator as in bench.py; the chunk's own
    K/V written by pa_reshape_and_cache, then pa_prefill; the oracle checks
    three whole sequences (every query row of them)."""
    w = wl.WORKLOADS["prefill"]
    rng = wl.rng_for(0)
    lens = wl.draw_context_lens(w, rng)
    nb = wl.pool_size(w, lens)
    a = batch.scattered_allocator(nb, wl.draw_block_order(nb, rng))
    slots = []
    for s, L in enumerate(lens):
        a.add_seq(s, int(L) - w.chunk)
        sl, _ = a.append_slots(np.full(w.chunk, s, np.int64))
        slots.append(sl)
    tables, ctx = a.build_tables(np.arange(len(lens)), batch.max_blocks_for(w))
    slots = np.concatenate(slots)
    T = w.chunk * len(lens)
    H, Hq, d, dt = w.num_kv_heads, w.num_q_heads, w.head_dim, w.dtype
    kc, vc = host_pool(rng, nb, w)
    q = wl.draw_values(rng, (T, Hq, d), dt)
    k_new = wl.draw_values(rng, (T, H, d), dt)
    v_new = wl.draw_values(rng, (T, H, d), dt)
    dkc, dvc = gh.to_dev(kc, dt), gh.to_dev(vc, dt)
    pk.reshape_and_cache(gh.to_dev(k_new, dt), gh.to_dev(v_new, dt), dkc, dvc,
                         gh.ints(slots, torch.int64))
    oracle.reshape_and_cache(k_new, v_new, kc, vc, slots)
    qs = np.arange(0, T + 1, w.chunk, dtype=np.int32)
    out = torch.empty((T, Hq, d), dtype=torch.bfloat16, device="cuda")
    pk.prefill(out, gh.to_dev(q, dt), dkc, dvc, gh.ints(tables), gh.ints(ctx), gh.ints(qs),
               w.chunk, H, w.scale)
    torch.cuda.synchronize()
    assert pk.get_error() == (0, 0)
    for s in (int(np.argmax(ctx)), int(np.argmin(ctx)), 5):
        sl = slice(s * w.chunk, (s + 1) * w.chunk)
        ref = oracle.prefill(q[sl], kc, vc, tables[s:s + 1], ctx[s:s + 1],
                             np.array([0, w.chunk], np.int32), H, w.scale, dt)
        assert gh.max_excess(out[sl], ref, dt) <= gh.TOL[dt], s
