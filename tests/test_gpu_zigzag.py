"""GPU parity along the zigzag scan orders (codes 4..11) against the fp64 oracle:
the reorientation bit-exact, the GLA forward (bf16 and fp32) and backward with the
same gates as the four SREM orders (tests/test_gpu_parity.py, tests/test_gpu_bwd.py).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

from test_gpu_bwd import run_case as run_bwd_case
from test_gpu_parity import F32_MAX_ABS, check_bf16, gpu_gla

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dig():
    import gated_linear_attention_chunkwise_b200 as pkg
    return pkg


@pytest.mark.parametrize("j", range(8))
def test_reorient_zigzag_bit_exact(dig, j):
    for (B, Hg, Wg, C, dt) in [(2, 7, 13, 24, torch.bfloat16), (1, 16, 16, 8, torch.float32)]:
        x = workloads.grid_tensor(B, Hg, Wg, C, dtype=dt, seed=j)
        xd = x.reshape(B, Hg * Wg, C).cuda()
        y = dig.srem_reorient(xd, 4 + j, 0, Hg, Wg)
        back = dig.srem_reorient(y, 4 + j, 1, Hg, Wg)
        torch.cuda.synchronize()
        want = oracle.reorient(x.reshape(B, Hg * Wg, C).view(torch.int16 if dt == torch.bfloat16 else torch.int32)
                               .numpy(), 4 + j, 0, Hg, Wg)
        got = y.cpu().view(torch.int16 if dt == torch.bfloat16 else torch.int32).numpy()
        assert np.array_equal(got, want)
        assert torch.equal(back.cpu(), x.reshape(B, Hg * Wg, C))


@pytest.mark.parametrize("j", range(8))
def test_gla_bf16_zigzag(dig, j):
    """A 9x23 grid (ragged chunks, rows and columns of odd length) and d=72."""
    w = workloads.custom(2, 2, 9, 23, 72, 72, "bf16")
    q, k, v, la = workloads.gla_inputs(w, seed=20 + j)
    got = gpu_gla(dig, q, k, v, la, w.Hgrid, w.Wgrid, 4 + j)
    ref = oracle.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, 4 + j)
    check_bf16(got, ref, f"zigzag {j}", scan=(w.Hgrid, w.Wgrid, 4 + j))


@pytest.mark.parametrize("j", [0, 3, 5, 6])
def test_gla_bf16_zigzag_c2(dig, j):
    """DiG-S/2 at 512 (B=8, H=6, 32x32, d=64) along four of the schemes."""
    w = workloads.WORKLOADS["c2"]
    q, k, v, la = workloads.gla_inputs(w, seed=j)
    got = gpu_gla(dig, q, k, v, la, w.Hgrid, w.Wgrid, 4 + j)
    ref = oracle.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, 4 + j)
    check_bf16(got, ref, f"c2 zigzag {j}", scan=(w.Hgrid, w.Wgrid, 4 + j))


@pytest.mark.parametrize("j", range(8))
def test_gla_f32_zigzag(dig, j):
    w = workloads.custom(2, 3, 11, 6, 64, 64, "f32")
    q, k, v, la = workloads.gla_inputs(w, seed=40 + j)
    got = gpu_gla(dig, q, k, v, la, w.Hgrid, w.Wgrid, 4 + j)
    ref = oracle.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, 4 + j)
    assert np.max(np.abs(got - ref)) <= F32_MAX_ABS


@pytest.mark.parametrize("j", [1, 4, 7])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_gla_bwd_zigzag(dig, j, dtype):
    run_bwd_case(dig, workloads.custom(2, 2, 10, 7, 64, 64, dtype), 4 + j, seed=60 + j)


def test_zigzag_rejected_where_unsupported(dig):
    w = workloads.custom(1, 1, 4, 4, 64, 64, "f32")
    q, k, v, la = (t.cuda() for t in workloads.gla_inputs(w))
    out = torch.empty_like(v)
    L = dig.lib()
    import ctypes
    vp, i = ctypes.c_void_p, ctypes.c_int
    L.gla_fwd_f32_noalloc.argtypes = [vp, vp, vp, vp] + [i] * 7 + [vp, vp]
    L.gla_fwd_f32_noalloc.restype = ctypes.c_int
    st = torch.cuda.current_stream().cuda_stream
    args = [q.data_ptr(), k.data_ptr(), v.data_ptr(), la.data_ptr(), 1, 1, 4, 4, 64, 64]
    assert L.gla_fwd_f32_noalloc(*args, 4, out.data_ptr(), st) == -2     # fixed scratch: codes 0..3 only
    assert L.gla_fwd_f32(*args, 12, out.data_ptr(), st) == -1           # no code 12
    assert dig.device_status() == 0
