"""Pins of the fp64 oracle against things other than itself (CPU only).

* fp16 / bf16 widening: every one of the 65536 bit patterns against numpy.
* paged decode: torch's fp64 scaled-dot-product attention on K/V rows that
  were drawn densely and never passed through the pool (pins the gather, the
  logical->physical block step and the GQA head grouping).
* closed forms: one token gives V[0]; identical keys give mean(V); constant
  values give that constant; two tokens give logistic weights; a dominant
  logit selects its value row; scale 0 gives mean(V); empty context gives 0.
* invariants: physical block placement does not change the result (bit for
  bit); merging disjoint token ranges by log-sum-exp equals the whole range.
* scatter write / block copy: round trip through the block table, untouched
  rows keep their bytes, negative slots are skipped, bad ids are counted.
"""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads as wl
from paged_inputs import make_paged, tables_from_order, to_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- widening
def test_f16_widening_exhaustive():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.widen(bits, oracle.F16)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_bf16_widening_exhaustive():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.widen(bits, oracle.BF16)
    with np.errstate(invalid="ignore"):  # signalling-NaN patterns are part of the sweep
        ref = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


# ---------------------------------------------------------------- decode vs library attention
def sdpa_dense(p):
    """torch fp64 attention on the dense rows (never through the pool)."""
    S, Hq, d = p.q.shape
    out = np.zeros((S, Hq, d))
    for s in range(S):
        L = int(p.lens[s])
        if L == 0:
            continue
        q = torch.from_numpy(to_f64(p.q[s], p.dtype)).reshape(1, Hq, 1, d)
        k = torch.from_numpy(to_f64(p.k_dense[s, :L], p.dtype)).permute(1, 0, 2).unsqueeze(0)
        v = torch.from_numpy(to_f64(p.v_dense[s, :L], p.dtype)).permute(1, 0, 2).unsqueeze(0)
        o = F.scaled_dot_product_attention(q, k, v, scale=p.scale, enable_gqa=(Hq != k.shape[1]))
        out[s] = o.reshape(Hq, d).numpy()
    return out


def run_oracle(p, seqs=None):
    return oracle.decode(p.q, p.key_cache, p.value_cache, p.tables, p.lens, p.num_kv_heads,
                         p.scale, p.dtype, seqs=seqs)


@pytest.mark.parametrize("dtype", [wl.F16, wl.BF16])
@pytest.mark.parametrize("hq,hkv,d", [(4, 4, 64), (8, 2, 128), (8, 1, 64), (6, 3, 32)])
def test_decode_matches_torch_sdpa(dtype, hq, hkv, d):
    rng = wl.rng_for(1)
    lens = rng.integers(1, 90, size=5)
    nb = wl.blocks_needed(lens, 16) + 7
    p = make_paged(rng, 5, hq, hkv, d, lens, nb, dtype)
    got = run_oracle(p)
    ref = sdpa_dense(p)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_decode_every_context_length_1_to_64():
    rng = wl.rng_for(2)
    lens = np.arange(1, 65)
    nb = wl.blocks_needed(lens, 16)
    p = make_paged(rng, 64, 2, 2, 64, lens, nb, wl.F16)
    np.testing.assert_allclose(run_oracle(p), sdpa_dense(p), rtol=0, atol=1e-12)


def test_decode_tiny_workload_vs_sdpa():
    w = wl.WORKLOADS["tiny"]
    rng = wl.rng_for(0)
    lens = wl.draw_context_lens(w, rng)
    p = make_paged(rng, w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, lens,
                   w.pool_blocks, w.dtype, scale=w.scale)
    np.testing.assert_allclose(run_oracle(p), sdpa_dense(p), rtol=0, atol=1e-12)


def test_seq_selection_matches_full():
    rng = wl.rng_for(3)
    lens = rng.integers(1, 70, size=6)
    p = make_paged(rng, 6, 4, 2, 64, lens, wl.blocks_needed(lens, 16), wl.BF16)
    full = run_oracle(p)
    sel = np.array([4, 1, 5], dtype=np.int32)
    assert np.array_equal(run_oracle(p, seqs=sel), full[sel])


# ---------------------------------------------------------------- closed forms
def test_one_token_returns_v0_exactly():
    rng = wl.rng_for(4)
    p = make_paged(rng, 3, 4, 4, 128, [1, 1, 1], 3, wl.F16)
    got = run_oracle(p)
    for s in range(3):
        assert np.array_equal(got[s], to_f64(p.v_dense[s, 0], wl.F16))


def test_identical_keys_give_mean_of_values():
    rng = wl.rng_for(5)
    lens = [37, 16, 5]
    p = make_paged(rng, 3, 2, 2, 64, lens, 6, wl.F16)
    # overwrite every key row of every used slot with one row
    row = p.key_cache[0, 0, 0].copy()
    p.key_cache[:] = row
    got = run_oracle(p)
    for s, L in enumerate(lens):
        mean = to_f64(p.v_dense[s, :L], wl.F16).mean(axis=0)  # [H, d]
        np.testing.assert_allclose(got[s], mean, rtol=0, atol=1e-13)


def test_constant_values_give_that_constant():
    rng = wl.rng_for(6)
    p = make_paged(rng, 2, 4, 4, 64, [50, 3], 5, wl.BF16)
    c = wl.round_to_bits(np.linspace(-2, 2, 64, dtype=np.float32), wl.BF16)
    p.value_cache[:] = c
    got = run_oracle(p)
    np.testing.assert_allclose(got, np.broadcast_to(to_f64(c, wl.BF16), got.shape), rtol=0,
                               atol=1e-14)


def test_two_tokens_logistic_weights():
    rng = wl.rng_for(7)
    p = make_paged(rng, 4, 2, 2, 64, [2, 2, 2, 2], 4, wl.F16, scale=0.3)
    got = run_oracle(p)
    for s in range(4):
        for h in range(2):
            q = to_f64(p.q[s, h], wl.F16)
            k0, k1 = (to_f64(p.k_dense[s, j, h], wl.F16) for j in (0, 1))
            v0, v1 = (to_f64(p.v_dense[s, j, h], wl.F16) for j in (0, 1))
            z = 0.3 * (q @ k0 - q @ k1)
            w0 = 1.0 / (1.0 + np.exp(-z))
            np.testing.assert_allclose(got[s, h], w0 * v0 + (1.0 - w0) * v1, rtol=0, atol=1e-14)


def test_dominant_logit_selects_its_value():
    rng = wl.rng_for(8)
    L = 40
    p = make_paged(rng, 1, 1, 1, 64, [L], 3, wl.F16)
    q = to_f64(p.q[0, 0], wl.F16)
    # key row 23 := 8 q (rounded to fp16): its logit exceeds the rest by > 50
    j = 23
    b, o = p.tables[0, j // 16], j % 16
    p.key_cache[b, 0, o] = wl.round_to_bits((8 * q).astype(np.float32), wl.F16)
    got = run_oracle(p)
    np.testing.assert_allclose(got[0, 0], to_f64(p.v_dense[0, j, 0], wl.F16), rtol=0, atol=1e-12)


def test_scale_zero_gives_mean_of_values():
    rng = wl.rng_for(9)
    p = make_paged(rng, 2, 2, 1, 64, [33, 16], 4, wl.BF16, scale=0.0)
    got = run_oracle(p)
    for s, L in enumerate([33, 16]):
        mean = to_f64(p.v_dense[s, :L, 0], wl.BF16).mean(axis=0)
        for h in range(2):
            np.testing.assert_allclose(got[s, h], mean, rtol=0, atol=1e-13)


def test_empty_context_gives_zeros():
    rng = wl.rng_for(10)
    p = make_paged(rng, 3, 2, 2, 64, [0, 5, 0], 2, wl.F16)
    got = run_oracle(p)
    assert np.all(got[0] == 0) and np.all(got[2] == 0)
    assert np.any(got[1] != 0)


def test_hand_worked_two_token_example():
    with open(os.path.join(GOLDEN, "hand_two_token.json")) as f:
        g = json.load(f)
    d = 64
    q = np.zeros((1, 1, d), np.float32)
    q[0, 0, :2] = g["q"]
    kc = np.zeros((1, 1, 16, d), np.float32)
    vc = np.zeros((1, 1, 16, d), np.float32)
    kc[0, 0, :2, :2] = g["K"]
    vc[0, 0, :2, :2] = g["V"]
    bits = lambda a: wl.round_to_bits(a, wl.F16)
    out = oracle.decode(bits(q), bits(kc), bits(vc), np.zeros((1, 1), np.int32),
                        np.array([2], np.int32), 1, g["scale"], wl.F16)
    np.testing.assert_allclose(out[0, 0, :2], g["out"], rtol=0, atol=1e-15)
    assert np.all(out[0, 0, 2:] == 0)


# ---------------------------------------------------------------- invariants
def test_physical_placement_does_not_change_result():
    w = wl.WORKLOADS["tiny"]
    lens = np.array([64, 17, 1, 48], np.int32)
    a = make_paged(wl.rng_for(11), 4, 4, 4, 64, lens, 64, wl.F16)
    # same dense rows, same q; a different random order of physical ids
    b = make_paged(wl.rng_for(11), 4, 4, 4, 64, lens, 64, wl.F16)
    order = wl.draw_block_order(64, wl.rng_for(99))
    tb = tables_from_order(lens, order, 16)
    kc = np.zeros_like(b.key_cache)
    vc = np.zeros_like(b.value_cache)
    for s in range(4):
        n = (int(lens[s]) + 15) // 16
        kc[tb[s, :n]] = a.key_cache[a.tables[s, :n]]
        vc[tb[s, :n]] = a.value_cache[a.tables[s, :n]]
    ra = run_oracle(a)
    rb = oracle.decode(a.q, kc, vc, tb, lens, 4, a.scale, wl.F16)
    assert np.array_equal(ra, rb)


@pytest.mark.parametrize("cuts", [(), (16,), (7, 300), (512, 1024), (1, 2, 3, 999)])
def test_lse_merge_of_ranges_equals_whole(cuts):
    rng = wl.rng_for(12)
    lens = np.array([1000, 1023, 600], np.int32)
    p = make_paged(rng, 3, 4, 2, 64, lens, wl.blocks_needed(lens, 16), wl.BF16)
    full, full_lse = oracle.decode_range(p.q, p.key_cache, p.value_cache, p.tables, p.lens, 2,
                                         p.scale, p.dtype)
    bounds = [0, *cuts, 4096]
    parts = [oracle.decode_range(p.q, p.key_cache, p.value_cache, p.tables, p.lens, 2, p.scale,
                                 p.dtype, a, b) for a, b in zip(bounds[:-1], bounds[1:])]
    o = np.stack([x[0] for x in parts], axis=2).reshape(12, len(parts), 64)
    lse = np.stack([x[1] for x in parts], axis=2).reshape(12, len(parts))
    merged = oracle.lse_merge(o, lse).reshape(3, 4, 64)
    np.testing.assert_allclose(merged, full, rtol=0, atol=1e-12)
    # log-sum-exp of the parts is the whole range's
    M = lse.max(axis=1, keepdims=True)
    np.testing.assert_allclose((M[:, 0] + np.log(np.exp(lse - M).sum(axis=1))).reshape(3, 4),
                               full_lse, rtol=0, atol=1e-12)


def test_lse_merge_all_empty_gives_zero():
    o = np.zeros((2, 3, 8))
    lse = np.full((2, 3), -np.inf)
    assert np.all(oracle.lse_merge(o, lse) == 0)


# ---------------------------------------------------------------- scatter write / block copy
def test_reshape_and_cache_round_trip_and_untouched_rows():
    rng = wl.rng_for(13)
    lens = np.array([17, 32, 1, 45], np.int32)
    p = make_paged(rng, 4, 2, 2, 64, lens, 12, wl.F16)
    k_new = wl.draw_values(rng, (4, 2, 64), wl.F16)
    v_new = wl.draw_values(rng, (4, 2, 64), wl.F16)
    pos = lens - 1
    slots = np.array([p.tables[s, pos[s] // 16] * 16 + pos[s] % 16 for s in range(4)], np.int64)
    slots[2] = -1  # padding entry: skipped
    kc0, vc0 = p.key_cache.copy(), p.value_cache.copy()
    bad = oracle.reshape_and_cache(k_new, v_new, p.key_cache, p.value_cache, slots)
    assert bad == 0
    changed = np.zeros(p.key_cache.shape[:1] + p.key_cache.shape[2:3], bool)  # [NB][bs]
    for s in (0, 1, 3):
        b, o = p.tables[s, pos[s] // 16], pos[s] % 16
        assert np.array_equal(p.key_cache[b, :, o], k_new[s])
        assert np.array_equal(p.value_cache[b, :, o], v_new[s])
        changed[b, o] = True
    keep = ~changed
    assert np.array_equal(p.key_cache.transpose(0, 2, 1, 3)[keep], kc0.transpose(0, 2, 1, 3)[keep])
    assert np.array_equal(p.value_cache.transpose(0, 2, 1, 3)[keep], vc0.transpose(0, 2, 1, 3)[keep])
    # out-of-range slots are counted and skipped
    kc1 = p.key_cache.copy()
    assert oracle.reshape_and_cache(k_new[:1], v_new[:1], p.key_cache, p.value_cache,
                                    np.array([12 * 16], np.int64)) == 1
    assert np.array_equal(kc1, p.key_cache)


def test_copy_blocks_copies_whole_blocks_only():
    rng = wl.rng_for(14)
    kc = wl.draw_values(rng, (10, 3, 16, 64), wl.BF16)
    vc = wl.draw_values(rng, (10, 3, 16, 64), wl.BF16)
    k0, v0 = kc.copy(), vc.copy()
    pairs = np.array([[1, 7], [4, 2], [9, 0]], np.int32)
    assert oracle.copy_blocks(kc, vc, pairs) == 0
    for s, d in pairs:
        assert np.array_equal(kc[d], k0[s]) and np.array_equal(vc[d], v0[s])
    rest = [i for i in range(10) if i not in pairs[:, 1]]
    assert np.array_equal(kc[rest], k0[rest]) and np.array_equal(vc[rest], v0[rest])
    assert oracle.copy_blocks(kc, vc, np.array([[3, 10]], np.int32)) == 1


def test_copy_on_write_branch_matches_unshared_sequence():
    """Two branches share a prompt's blocks; a write into the shared last block
    copies it first.  Each branch must then equal the same tokens stored with
    no sharing at all."""
    rng = wl.rng_for(15)
    H, d, bs, prompt = 2, 64, 16, 40          # 3 blocks, the last holds 8 tokens
    dt = wl.F16
    kp = wl.draw_values(rng, (prompt, H, d), dt)
    vp = wl.draw_values(rng, (prompt, H, d), dt)
    q = wl.draw_values(rng, (2, H, d), dt)
    k_new = wl.draw_values(rng, (2, H, d), dt)
    v_new = wl.draw_values(rng, (2, H, d), dt)
    nb = 8
    # shared layout: prompt in blocks 0,1,2; branch 0 copies block 2 -> 3 and
    # writes there; branch 1 (last holder) writes into block 2 in place.
    kc = wl.draw_values(rng, (nb, H, bs, d), dt)
    vc = wl.draw_values(rng, (nb, H, bs, d), dt)
    prompt_slots = np.arange(prompt, dtype=np.int64)
    oracle.reshape_and_cache(kp, vp, kc, vc, prompt_slots)
    oracle.copy_blocks(kc, vc, np.array([[2, 3]], np.int32))
    tables = np.array([[0, 1, 3], [0, 1, 2]], np.int32)
    oracle.reshape_and_cache(k_new, v_new, kc, vc, np.array([3 * 16 + 8, 2 * 16 + 8], np.int64))
    lens = np.array([prompt + 1, prompt + 1], np.int32)
    shared = oracle.decode(q, kc, vc, tables, lens, H, 0.125, dt)
    # unshared: each branch holds its own copy of the prompt
    for b in range(2):
        kc_u = wl.draw_values(rng, (3, H, bs, d), dt)
        vc_u = wl.draw_values(rng, (3, H, bs, d), dt)
        oracle.reshape_and_cache(np.concatenate([kp, k_new[b:b + 1]]),
                                 np.concatenate([vp, v_new[b:b + 1]]), kc_u, vc_u,
                                 np.arange(prompt + 1, dtype=np.int64))
        alone = oracle.decode(q[b:b + 1], kc_u, vc_u, np.array([[0, 1, 2]], np.int32),
                              lens[:1], H, 0.125, dt)
        assert np.array_equal(shared[b], alone[0])


# ---------------------------------------------------------------- chunked prefill
def _chunks(lens, qlens):
    qs = np.zeros(len(lens) + 1, np.int32)
    qs[1:] = np.cumsum(qlens)
    return qs


def sdpa_prefill_dense(p, qchunk, qlens):
    """torch fp64 attention with an explicit causal mask on the dense rows."""
    S = len(p.lens)
    Hq, d = qchunk.shape[1], qchunk.shape[2]
    qs = _chunks(p.lens, qlens)
    out = np.zeros(qchunk.shape)
    for s in range(S):
        L, n = int(p.lens[s]), int(qlens[s])
        if n == 0:
            continue
        q = torch.from_numpy(to_f64(qchunk[qs[s]:qs[s + 1]], p.dtype)).permute(1, 0, 2).unsqueeze(0)
        k = torch.from_numpy(to_f64(p.k_dense[s, :L], p.dtype)).permute(1, 0, 2).unsqueeze(0)
        v = torch.from_numpy(to_f64(p.v_dense[s, :L], p.dtype)).permute(1, 0, 2).unsqueeze(0)
        allowed = np.arange(L)[None, :] <= (L - n + np.arange(n))[:, None]
        o = F.scaled_dot_product_attention(q, k, v, attn_mask=torch.from_numpy(allowed),
                                           scale=p.scale, enable_gqa=(Hq != k.shape[1]))
        out[qs[s]:qs[s + 1]] = o[0].permute(1, 0, 2).numpy()
    return out


@pytest.mark.parametrize("hq,hkv,d,dtype", [(4, 4, 64, wl.F16), (8, 2, 128, wl.BF16)])
def test_prefill_matches_causal_sdpa(hq, hkv, d, dtype):
    rng = wl.rng_for(30)
    lens = np.array([40, 100, 17, 64, 5], np.int32)
    qlens = np.array([40, 33, 1, 16, 5], np.int32)   # whole prompts, chunks, one token
    p = make_paged(rng, 5, hq, hkv, d, lens, wl.blocks_needed(lens, 16) + 3, dtype)
    qchunk = wl.draw_values(rng, (int(qlens.sum()), hq, d), dtype)
    got = oracle.prefill(qchunk, p.key_cache, p.value_cache, p.tables, p.lens,
                         _chunks(lens, qlens), hkv, p.scale, dtype)
    np.testing.assert_allclose(got, sdpa_prefill_dense(p, qchunk, qlens), rtol=0, atol=1e-12)


def test_prefill_of_whole_prompt_is_causal_self_attention():
    rng = wl.rng_for(31)
    L = 70
    p = make_paged(rng, 1, 2, 2, 64, [L], 5, wl.F16)
    qchunk = wl.draw_values(rng, (L, 2, 64), wl.F16)
    got = oracle.prefill(qchunk, p.key_cache, p.value_cache, p.tables, p.lens,
                         np.array([0, L], np.int32), 2, p.scale, wl.F16)
    q = torch.from_numpy(to_f64(qchunk, wl.F16)).permute(1, 0, 2).unsqueeze(0)
    k = torch.from_numpy(to_f64(p.k_dense[0, :L], wl.F16)).permute(1, 0, 2).unsqueeze(0)
    v = torch.from_numpy(to_f64(p.v_dense[0, :L], wl.F16)).permute(1, 0, 2).unsqueeze(0)
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=p.scale)
    np.testing.assert_allclose(got, ref[0].permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
    # the first query row sees only token 0: its output is V[0]
    assert np.array_equal(got[0], to_f64(p.v_dense[0, 0], wl.F16))


def test_prefill_with_one_token_chunks_equals_decode():
    rng = wl.rng_for(32)
    lens = np.array([33, 1, 200], np.int32)
    p = make_paged(rng, 3, 8, 2, 128, lens, wl.blocks_needed(lens, 16), wl.BF16)
    got = oracle.prefill(p.q, p.key_cache, p.value_cache, p.tables, p.lens,
                         np.arange(4, dtype=np.int32), 2, p.scale, wl.BF16)
    assert np.array_equal(got, run_oracle(p))
