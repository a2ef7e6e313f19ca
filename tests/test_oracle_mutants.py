"""The oracle's pins must reject plausible mistakes (CPU only).

Each case copies pa_oracle.c, plants one mistake (a wrong index, a dropped
term, a flipped sign, a swapped operand), compiles the copy with gcc into a
temporary library and runs the pin tests against it in a child process (a
mistake that reads out of bounds may crash that process, which also counts
as caught).  At least one pin must fail for every planted mistake.
"""
import os
import subprocess
import sys
import tempfile

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "pa_oracle.c")

# (name, text to replace, replacement)
MUTANTS = [
    ("block index uses offset", "int64_t b = table_row[j / block_size];",
     "int64_t b = table_row[j % block_size];"),
    ("row index uses block", "int64_t o = j % block_size;\n        int64_t base",
     "int64_t o = (j / block_size) % block_size;\n        int64_t base"),
    ("scale dropped", "x[j] = scale * dot;", "x[j] = dot;"),
    ("softmax sign flipped", "double w = exp(x[j] - m);", "double w = exp(m - x[j]);"),
    ("value operand swapped for key", "o[i] += w * V[(int64_t)j * head_dim + i];",
     "o[i] += w * K[(int64_t)j * head_dim + i];"),
    ("normalisation dropped", "        o[i] /= den;\n    free(x);", "    free(x);"),
    ("kv head grouping interleaved", "int32_t kvh = h / group;", "int32_t kvh = h % num_kv_heads;"),
    ("fp16 exponent bias off by one", "mag = ldexp((double)(f | 0x400), e - 25);",
     "mag = ldexp((double)(f | 0x400), e - 24);"),
    ("fp16 subnormal scale", "mag = ldexp((double)f, -24);", "mag = ldexp((double)f, -25);"),
    ("bf16 exponent bias off by one", "mag = ldexp((double)(f | 0x80), e - 134);",
     "mag = ldexp((double)(f | 0x80), e - 133);"),
    ("merge weight sign flipped", "double w = exp(lse_parts[r * num_parts + p] - M);",
     "double w = exp(M - lse_parts[r * num_parts + p]);"),
    ("lse drops the max", "return m + log(den);", "return log(den);"),
    ("scatter writes v into the key cache", "key_cache[dst + i] = k[src + i];",
     "key_cache[dst + i] = v[src + i];"),
    ("scatter row from block", "int64_t o = slot % block_size;", "int64_t o = slot / block_size % block_size;"),
    ("copy direction swapped",
     "key_cache[dst * per_block + e] = key_cache[src * per_block + e];",
     "key_cache[src * per_block + e] = key_cache[dst * per_block + e];"),
    ("negative slot not skipped", "if (slot < 0)\n            continue;", "if (slot < -1)\n            continue;"),
    ("last token dropped", "int32_t n = b > a ? b - a : 0;", "int32_t n = b - 1 > a ? b - 1 - a : 0;"),
    ("prefill causal bound excludes the query's own token", "int32_t n = pos + 1 > 0 ? pos + 1 : 0;",
     "int32_t n = pos > 0 ? pos : 0;"),
    ("prefill chunk placed at the start of the context",
     "int32_t pos = context_lens[s] - n_s + (t - query_start[s]);",
     "int32_t pos = (t - query_start[s]);"),
]

PIN_TESTS = [
    pins.test_f16_widening_exhaustive,
    pins.test_bf16_widening_exhaustive,
    lambda: pins.test_decode_matches_torch_sdpa(pins.wl.F16, 8, 2, 128),
    lambda: pins.test_decode_matches_torch_sdpa(pins.wl.BF16, 6, 3, 32),
    pins.test_decode_every_context_length_1_to_64,
    pins.test_one_token_returns_v0_exactly,
    pins.test_identical_keys_give_mean_of_values,
    pins.test_constant_values_give_that_constant,
    pins.test_two_tokens_logistic_weights,
    pins.test_hand_worked_two_token_example,
    lambda: pins.test_lse_merge_of_ranges_equals_whole((7, 300)),
    pins.test_reshape_and_cache_round_trip_and_untouched_rows,
    pins.test_copy_blocks_copies_whole_blocks_only,
    pins.test_copy_on_write_branch_matches_unshared_sequence,
    lambda: pins.test_prefill_matches_causal_sdpa(4, 4, 64, pins.wl.F16),
    pins.test_prefill_of_whole_prompt_is_causal_self_attention,
]


def _build_mutant(tmp, text, old, new):
    assert text.count(old) == 1, f"mutation anchor not unique: {old!r}"
    src = os.path.join(tmp, "mutant.c")
    lib = os.path.join(tmp, "libmutant.so")
    with open(src, "w") as f:
        f.write(text.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", lib,
                           src, "-lm"])
    return lib


def _pins_all_pass():
    for t in PIN_TESTS:
        try:
            t()
        except AssertionError:
            return False
    return True


def _pins_pass_in_child(lib) -> bool:
    """Run every pin against library `lib` in a fresh interpreter."""
    here = os.path.dirname(os.path.abspath(__file__))
    code = ("import sys; sys.path[:0] = [%r, %r]\n"
            "import oracle, test_oracle_mutants as m\n"
            "oracle._swap_library(%r)\n"
            "sys.exit(0 if m._pins_all_pass() else 1)\n") % (here, os.path.dirname(here), lib)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, timeout=600)
    return r.returncode == 0


def test_unmutated_copy_passes_every_pin():
    text = open(SRC).read()
    with tempfile.TemporaryDirectory() as tmp:
        lib = _build_mutant(tmp, text, "double oracle_f16_to_f64", "double oracle_f16_to_f64")
        assert _pins_pass_in_child(lib)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(name, old, new):
    text = open(SRC).read()
    with tempfile.TemporaryDirectory() as tmp:
        lib = _build_mutant(tmp, text, old, new)
        assert not _pins_pass_in_child(lib), f"no pin rejects the planted mistake: {name}"
