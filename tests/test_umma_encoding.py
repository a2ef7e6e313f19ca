"""CPU check of the tcgen05 descriptor encodings used by the prefill kernel.

The shared-memory and instruction descriptors are packed by hand in
pa_umma.cuh; a wrong bit position there would make tcgen05.mma read the
wrong operands (or raise an illegal-instruction error).  This compiles a
host-only program that packs the same fields through CUTLASS's own
definitions (cute::UMMA::make_instr_desc and the SmemDescriptor bitfields)
and compares.  Skipped when nvcc or the CUTLASS headers are absent.
"""
import importlib.util
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def cutlass_include():
    for mod, sub in (("flashinfer", ("data", "cutlass", "include")),
                     ("tilelang", ("3rdparty", "cutlass", "include"))):
        spec = importlib.util.find_spec(mod)
        if spec is None or not spec.submodule_search_locations:
            continue
        path = os.path.join(list(spec.submodule_search_locations)[0], *sub)
        if os.path.exists(os.path.join(path, "cute", "arch", "mma_sm100_desc.hpp")):
            return path
    return None


def test_descriptor_encodings_match_cutlass(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    inc = cutlass_include()
    if not os.path.exists(nvcc) or inc is None:
        pytest.skip("nvcc or CUTLASS headers not available")
    exe = str(tmp_path / "umma_encoding_check")
    subprocess.check_call([nvcc, "-std=c++17", "-O0", "-I", inc,
                           "-I", os.path.join(ROOT, "paged_kv_cache_425_b200", "csrc"),
                           "-I", os.path.join(ROOT, "include"),
                           "-o", exe, os.path.join(ROOT, "tests", "umma_encoding_check.cu")])
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr


def test_fma_pipe_exp2_accuracy(tmp_path):
    """The polynomial 2^a the tcgen05 softmax runs beside the special-function
    unit: relative error below 1e-4 on [-125, 8] against double precision,
    and tiny positive values below -125 (masked scores)."""
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    exe = str(tmp_path / "exp2_fma_check")
    subprocess.check_call([nvcc, "-std=c++17", "-O2",
                           "-I", os.path.join(ROOT, "paged_kv_cache_425_b200", "csrc"),
                           "-o", exe, os.path.join(ROOT, "tests", "exp2_fma_check.cu")])
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.startswith("ok"), r.stdout + r.stderr
