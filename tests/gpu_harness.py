"""Test-side glue: move host problems onto the GPU, run the library's calls,
bring results back.  The oracle is never called from here."""
from __future__ import annotations

import numpy as np
import torch

import workloads as wl

TOL = {wl.F16: 2e-3, wl.BF16: 1e-2}
# Chunked prefill has no stated budget; it takes the decode budget plus the
# rounding of the output itself (half an ulp of the 16-bit type), because an
# early query row attends to few keys and |out| can exceed 4, where half an
# ulp of bf16 (0.0156) alone is above 1e-2.
REL = {wl.F16: 2.0 ** -11, wl.BF16: 2.0 ** -8}


def tdtype(dtype):
    return torch.float16 if dtype == wl.F16 else torch.bfloat16


def to_dev(bits: np.ndarray, dtype) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(tdtype(dtype)).cuda()


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def ints(a, dtype=torch.int32) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype).cuda()


def workspace_for(pk, S, hq, d, max_blocks):
    n = pk.decode_workspace_size(S, hq, d, max_blocks)
    return torch.empty(max(n, 256), dtype=torch.uint8, device="cuda") if n else None


def run_decode(pk, q_bits, kc, vc, tables, lens, num_kv_heads, scale, dtype, stream=None):
    """kc / vc may be host bits or device tensors; returns the output tensor."""
    if isinstance(kc, np.ndarray):
        kc, vc = to_dev(kc, dtype), to_dev(vc, dtype)
    q = to_dev(q_bits, dtype)
    S, hq, d = q.shape
    out = torch.full_like(q, float("nan"))
    tbl = ints(tables)
    ln = ints(lens)
    ws = workspace_for(pk, S, hq, d, tbl.shape[1])
    pk.decode(out, q, kc, vc, tbl, ln, num_kv_heads, scale, workspace=ws, stream=stream)
    torch.cuda.synchronize()
    return out


def max_excess(gpu: torch.Tensor, ref: np.ndarray, dtype) -> float:
    """max |gpu - ref| - REL[dtype] |ref|: compare with TOL[dtype]."""
    g = to_f64(gpu)
    assert np.all(np.isfinite(g)), "non-finite output"
    return float(np.max(np.abs(g - ref) - REL[dtype] * np.abs(ref))) if g.size else 0.0


def max_err(gpu: torch.Tensor, ref: np.ndarray) -> float:
    g = to_f64(gpu)
    assert np.all(np.isfinite(g)), "non-finite output"
    return float(np.max(np.abs(g - ref))) if g.size else 0.0
