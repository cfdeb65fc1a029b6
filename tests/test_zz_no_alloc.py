"""GPU test of gla_fwd_f32_noalloc, the fp32 GLA forward for callers that cannot
allocate device memory (a framework that owns the memory pool, a real-time
program that allocates only at start-up, work captured into a graph without
memory nodes).  On two calls in a row, whose scratch array is shared and keeps
the previous call's contents, it must give the same result as gla_fwd_f32 and
as the fp64 oracle, within the fp32 path's 1e-4 max-abs tolerance.

The first call's gates contain full resets and very strong decays, so some of
its chunks take the exact token-serial path (which leaves a flag and the
incoming state in the scratch); the second call, of the same shape with plain
gates, must not see any of that.

The file name sorts last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

F32_MAX_ABS = 1e-4
SCRATCH = 8 << 20


@pytest.fixture(scope="module")
def lib():
    import gated_linear_attention_chunkwise_b200 as pkg
    L = pkg.lib()
    vp, i = ctypes.c_void_p, ctypes.c_int
    L.gla_fwd_f32_noalloc.argtypes = [vp, vp, vp, vp] + [i] * 7 + [vp, vp]
    L.gla_fwd_f32_noalloc.restype = ctypes.c_int
    return pkg, L


def _noalloc(L, w, q, k, v, la, direction):
    out = torch.full((w.B, w.T, w.H, w.dv), float("nan"), device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = L.gla_fwd_f32_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), la.data_ptr(), w.B, w.H, w.Hgrid,
                               w.Wgrid, w.dk, w.dv, direction, out.data_ptr(), stream)
    assert rc == 0, rc
    return out


def _check(pkg, L, w, q, k, v, la, direction):
    dq, dk_, dv_, dla = (t.cuda() for t in (q, k, v, la))
    got = _noalloc(L, w, dq, dk_, dv_, dla, direction)
    sibling = pkg.gla_fwd_f32(dq, dk_, dv_, dla, w.Hgrid, w.Wgrid, direction)
    torch.cuda.synchronize()
    got = got.cpu().numpy().astype(np.float64)
    ref = oracle.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, direction)
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - ref)) <= F32_MAX_ABS
    assert np.max(np.abs(got - sibling.cpu().numpy())) <= F32_MAX_ABS


def _scratch_bytes(B, H, T, dk, dv):
    """The capacity formula stated for gla_fwd_f32_noalloc in include/dig_gla.h."""
    rup = lambda x: -(-x // 256) * 256  # noqa: E731
    n = B * H * -(-T // 64)
    return 2 * rup(n * dk * dv * 4) + rup(n * dk * 4) + rup(n * 4)


def test_noalloc_matches_oracle_on_two_calls(lib):
    pkg, L = lib
    w = workloads.custom(2, 3, 20, 13, 72, 72, "f32")
    q, k, v, la = workloads.gla_inputs(w, seed=0)
    # Call 1: full resets and decays of e^-30 per token in a few places, so some
    # chunks are evaluated token by token.
    gen = torch.Generator().manual_seed(5)
    m = torch.rand(la.shape, generator=gen)
    la1 = torch.where(m < 0.01, torch.full_like(la, -math.inf), la)
    la1 = torch.where((m >= 0.01) & (m < 0.03), torch.full_like(la, -30.0), la1)
    _check(pkg, L, w, q, k, v, la1, 3)
    # Call 2, right after, same shape, plain gates: nothing of call 1 may leak in.
    _check(pkg, L, w, q, k, v, la, 3)
    # Call 3: the fp32 workload (B=2, H=6, 16x16, d=64, left-to-right).
    w1 = workloads.WORKLOADS["c1"]
    _check(pkg, L, w1, *workloads.gla_inputs(w1, seed=0), 0)
    assert pkg.device_status() == 0


def test_noalloc_capacity_boundary(lib):
    """B=H=1, dk=dv=128: 63 chunks of 64 tokens fit in the 8 MiB array, 64 do not."""
    pkg, L = lib
    assert _scratch_bytes(1, 1, 63 * 64, 128, 128) <= SCRATCH < _scratch_bytes(1, 1, 64 * 64, 128, 128)
    w = workloads.custom(1, 1, 63, 64, 128, 128, "f32")
    _check(pkg, L, w, *workloads.gla_inputs(w, seed=3), 1)
    w = workloads.custom(1, 1, 64, 64, 128, 128, "f32")
    q, k, v, la = (t.cuda() for t in workloads.gla_inputs(w, seed=3))
    out = torch.empty((w.B, w.T, w.H, w.dv), device="cuda")
    rc = L.gla_fwd_f32_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), la.data_ptr(), w.B, w.H, w.Hgrid,
                               w.Wgrid, w.dk, w.dv, 0, out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == -2   # GLA_ERR_UNSUPPORTED, nothing launched


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    pkg, L = lib
    w = workloads.custom(8, 8, 32, 32, 128, 128, "f32")   # needs ~134 MB of scratch
    q, k, v, la = (t.cuda() for t in workloads.gla_inputs(w, seed=2))
    out = torch.empty((w.B, w.T, w.H, w.dv), device="cuda")
    rc = L.gla_fwd_f32_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), la.data_ptr(), w.B, w.H, w.Hgrid,
                               w.Wgrid, w.dk, w.dv, 0, out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == -2   # GLA_ERR_UNSUPPORTED, nothing launched
