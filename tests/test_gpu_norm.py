"""GPU parity of the normalised variant (gla_norm_fwd, gla_norm_fwd_f32) against the
fp64 oracle (oracle.gla_norm_fwd).  The kernels compute in fp32 throughout, so:
fp32 outputs max-abs <= 1e-4 (the GLA path's fp32 bar); bf16 outputs every element
within 2^-8 |oracle| + 1e-3 RMS(head) (the store's rounding plus fp32 arithmetic)
and a relative RMS error <= 2e-2 per head.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads

from test_gpu_bwd import check

pytestmark = pytest.mark.gpu
EPS = 1e-6


@pytest.fixture(scope="module")
def dig():
    import gated_linear_attention_chunkwise_b200 as pkg
    return pkg


def run(dig, w, direction, seed=0, scale=None, eps=EPS, q_shift=0.0):
    q, k, v, _ = workloads.gla_inputs(w, seed=seed, qkv_scale=scale)
    if q_shift:
        q = (q.float() + q_shift).to(q.dtype)
    fn = dig.gla_norm_fwd if w.dtype == "bf16" else dig.gla_norm_fwd_f32
    got = fn(q.cuda(), k.cuda(), v.cuda(), w.Hgrid, w.Wgrid, direction, eps=eps)
    torch.cuda.synchronize()
    assert dig.device_status() == 0
    got = got.float().cpu().numpy().astype(np.float64)
    ref = oracle.gla_norm_fwd(q, k, v, w.Hgrid, w.Wgrid, direction, eps=eps)
    check(got, ref, f"norm dir {direction}", w.dtype == "bf16", elt_rms=1e-3)
    return got, ref


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_norm_f32_c1_shape(dig, direction):
    run(dig, workloads.WORKLOADS["c1"], direction)


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_norm_bf16_c2(dig, direction):
    run(dig, workloads.WORKLOADS["c2"], direction, seed=3)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_norm_ragged_d72_and_zigzag(dig, dtype):
    w = workloads.custom(2, 2, 9, 23, 72, 72, dtype)
    for direction in (0, 3, 4 + 5):
        run(dig, w, direction, seed=5)


def test_norm_strong_gates_take_the_exact_path(dig):
    """q, k at scale 2: q * k of order 4, sigmoid gates down to e^-4 per token, so
    64-token chunks decay far beyond e^80 and run token by token."""
    run(dig, workloads.custom(1, 2, 12, 12, 64, 64, "f32"), 2, seed=6, scale=2.0)


def test_norm_single_token_is_v(dig):
    w = workloads.custom(2, 3, 1, 1, 64, 64, "f32")
    got, _ = run(dig, w, 0, seed=7)
    v = workloads.gla_inputs(w, seed=7)[2].numpy()
    assert np.max(np.abs(got - v)) <= 1e-5


def test_norm_clamp(dig):
    """q shifted by -40: phi(q) = e^q ~ 1e-18, the denominator falls below eps = 1e-3
    and the output is the numerator over eps (tiny)."""
    got, ref = run(dig, workloads.custom(1, 2, 6, 6, 64, 64, "f32"), 0, seed=8, eps=1e-3, q_shift=-40.0)
    assert np.max(np.abs(ref)) < 1e-12


def test_norm_rejects(dig):
    L = dig.lib()
    w = workloads.custom(1, 1, 4, 4, 64, 128, "f32")
    q, k, v, _ = (t.cuda() for t in workloads.gla_inputs(w))
    out = torch.empty_like(v)
    st = torch.cuda.current_stream().cuda_stream
    args = [q.data_ptr(), k.data_ptr(), v.data_ptr(), 1, 1, 4, 4, 64, 128, 0]
    assert L.gla_norm_fwd_f32(*args, 1e-6, out.data_ptr(), st) == -2     # dv > 120: no room for the ones column
    args[8] = 64
    assert L.gla_norm_fwd_f32(*args, 0.0, out.data_ptr(), st) == -1      # eps must be positive
    assert L.gla_norm_fwd_f32(*args, 1e-6, v.data_ptr(), st) == -1       # out over an input
    assert dig.device_status() == 0
