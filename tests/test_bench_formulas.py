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


def test_prefill_flops_match_a_per_query_count():
    lens = np.array([512, 700, 3000], np.int64)
    chunk, Hq, d = 512, 32, 128
    brute = 0
    for L in lens:
        for i in range(chunk):
            keys = L - chunk + i + 1
            brute += 2 * keys * d * Hq * 2    # q.K and P.V, a multiply-add = 2 FLOPs
    assert bench.prefill_flops(lens, chunk, Hq, d) == brute
