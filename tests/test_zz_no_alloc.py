"""pa_decode_static_workspace: decode for callers that cannot allocate.

Some callers cannot hand pa_decode a workspace: a serving process whose
device memory is reserved up front by its own pools, a hot loop that must
not call cudaMalloc (it can synchronise the device), or a foreign-language
caller with no device allocator.  This entry point uses a fixed array in the
library instead.  It launches the same kernels with the same partitioning on
the same inputs as pa_decode, so its output must be bit-identical to
pa_decode's, on two calls in a row (the array keeps the first call's
contents), and within the attention tolerance of the fp64 oracle.  Sizes
beyond its array must be refused without anything being launched.

The file is named to be collected last, so a run that stops at the first
failure has already run every other test; it also passes on its own.
"""
import numpy as np
import pytest

import oracle
import workloads as wl
from paged_inputs import make_paged

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import gpu_harness as gh  # noqa: E402

pk = pytest.importorskip("paged_kv_cache_425_b200")


def both_ways(p):
    """(pa_decode with a caller workspace, pa_decode_static_workspace)."""
    ref = gh.run_decode(pk, p.q, p.key_cache, p.value_cache, p.tables, p.lens, p.num_kv_heads,
                        p.scale, p.dtype)
    q = gh.to_dev(p.q, p.dtype)
    kc, vc = gh.to_dev(p.key_cache, p.dtype), gh.to_dev(p.value_cache, p.dtype)
    out = torch.full_like(q, float("nan"))
    pk.decode_static_workspace(out, q, kc, vc, gh.ints(p.tables), gh.ints(p.lens),
                               p.num_kv_heads, p.scale)
    torch.cuda.synchronize()
    return ref, out


@pytest.mark.parametrize("hq,hkv,dtype", [(8, 2, wl.BF16), (4, 4, wl.F16)])
def test_matches_pa_decode_on_two_calls_in_a_row(hq, hkv, dtype):
    for call in range(2):
        rng = wl.rng_for(500 + call)
        # contexts over several 512-token partitions, so the scratch is used
        lens = np.array([3000, 17, 1200, 2049, 513, 1], np.int32) if call == 0 else \
            np.array([700, 4000, 33, 1025], np.int32)
        p = make_paged(rng, len(lens), hq, hkv, 128, lens, wl.blocks_needed(lens, 16) + 3, dtype)
        assert pk.decode_workspace_size(len(lens), hq, 128, p.tables.shape[1]) > 0
        ref, out = both_ways(p)
        assert torch.equal(ref, out), (call, float((ref.float() - out.float()).abs().max()))
        want = oracle.decode(p.q, p.key_cache, p.value_cache, p.tables, p.lens, p.num_kv_heads,
                             p.scale, p.dtype)
        assert gh.max_err(out, want) <= gh.TOL[dtype], call
    assert pk.get_error() == (0, 0)


def test_refuses_sizes_beyond_its_array():
    # 4096 sequences x 64 heads x 16 partitions of fp32 partials: far beyond the array
    S, Hq, Hkv, d, maxb = 4096, 64, 8, 128, 512
    need = pk.decode_workspace_size(S, Hq, d, maxb)
    assert need > pk.STATIC_WORKSPACE_BYTES
    q = torch.zeros((S, Hq, d), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((4, Hkv, 16, d), dtype=torch.bfloat16, device="cuda")
    tables = torch.zeros((S, maxb), dtype=torch.int32, device="cuda")
    lens = torch.ones(S, dtype=torch.int32, device="cuda")
    out = torch.full_like(q, float("nan"))
    torch.cuda.synchronize()
    with pytest.raises(pk.PagedError) as e:
        pk.decode_static_workspace(out, q, kc, kc, tables, lens, Hkv, 0.1)
    assert e.value.status == pk.PA_ERR_WORKSPACE
    torch.cuda.synchronize()
    # nothing ran: the output is untouched and no kernel reported anything
    assert bool(torch.isnan(out).all())
    assert pk.get_error() == (0, 0)
