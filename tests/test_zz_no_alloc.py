"""GPU test of gla_fwd_f32_noalloc, the fp32 GLA forward for callers that cannot
allocate device memory (a framework that owns the memory pool, a real-time
program that allocates only at start-up, work captured into a graph without
memory nodes).  It must give the same result as gla_fwd_f32 -- within the fp32
path's 1e-4 max-abs tolerance -- on two calls in a row, whose scratch array is
shared and keeps the previous call's contents.

The file name sorts last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import ctypes

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

F32_MAX_ABS = 1e-4


@pytest.fixture(scope="module")
def lib():
    import gated_linear_attention_chunkwise_b200 as pkg
    L = pkg.lib()
    vp, i = ctypes.c_void_p, ctypes.c_int
    L.gla_fwd_f32_noalloc.argtypes = [vp, vp, vp, vp] + [i] * 7 + [vp, vp]
    L.gla_fwd_f32_noalloc.restype = ctypes.c_int
    return pkg, L


def _inputs(B, H, Hg, Wg, d, seed):
    w = workloads.custom(B, H, Hg, Wg, d, d, "f32")
    return w, [t.cuda() for t in workloads.gla_inputs(w, seed=seed)]


def _noalloc(L, w, q, k, v, la, direction):
    out = torch.full((w.B, w.T, w.H, w.dv), float("nan"), device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = L.gla_fwd_f32_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), la.data_ptr(), w.B, w.H, w.Hgrid,
                               w.Wgrid, w.dk, w.dv, direction, out.data_ptr(), stream)
    assert rc == 0, rc
    return out


def test_noalloc_matches_gla_fwd_f32_on_two_calls(lib):
    pkg, L = lib
    # Call 1: the fp32 workload (B=2, H=6, 16x16, d=64, left-to-right).
    w1, (q, k, v, la) = _inputs(2, 6, 16, 16, 64, seed=0)
    got = _noalloc(L, w1, q, k, v, la, 0)
    want = pkg.gla_fwd_f32(q, k, v, la, w1.Hgrid, w1.Wgrid, 0)
    torch.cuda.synchronize()
    assert torch.isfinite(got).all()
    assert (got - want).abs().max().item() <= F32_MAX_ABS
    # Call 2, right after, on different shapes and a column-major scan: the
    # shared scratch still holds call 1's values.
    w2, (q, k, v, la) = _inputs(1, 3, 10, 13, 72, seed=1)
    got = _noalloc(L, w2, q, k, v, la, 3)
    want = pkg.gla_fwd_f32(q, k, v, la, w2.Hgrid, w2.Wgrid, 3)
    torch.cuda.synchronize()
    assert torch.isfinite(got).all()
    assert (got - want).abs().max().item() <= F32_MAX_ABS
    assert pkg.device_status() == 0


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    pkg, L = lib
    w, (q, k, v, la) = _inputs(8, 8, 32, 32, 128, seed=2)   # needs ~134 MB of scratch
    out = torch.empty((w.B, w.T, w.H, w.dv), device="cuda")
    rc = L.gla_fwd_f32_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), la.data_ptr(), w.B, w.H, w.Hgrid,
                               w.Wgrid, w.dk, w.dv, 0, out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == -2   # GLA_ERR_UNSUPPORTED, nothing launched
