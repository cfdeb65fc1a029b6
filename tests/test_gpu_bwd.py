"""GPU parity of the GLA backward (gla_bwd, gla_bwd_f32) against the fp64 oracle's
reverse sweep (oracle.gla_bwd), through the C ABI.

The pages state no tolerance for the backward; the gates follow its arithmetic:
  * gla_bwd_f32 (fp32 inputs, every product and sum in fp32 on CUDA cores): the GLA
    path's fp32 bar, max-abs error <= 1e-4, and a relative RMS error <= 1e-4 per
    (batch, head) (fp32 rounding over a few hundred terms, with margin);
  * gla_bwd (bf16 inputs; for dk, dv <= 80 the chunk products run on tensor cores
    from bf16 operands Q~, K^, A, P, G, D with fp32 accumulation): the forward's bf16
    gates on all four outputs -- relative RMS error <= 2e-2 per (batch, head), every
    element within 2^-8 |oracle| + 0.1 RMS(head).
Inputs: workloads.gla_inputs and workloads.gla_dout (seeded, synthetic).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

F32_MAX_ABS = 1e-4
F32_REL_RMS = 1e-4
BF16_REL_RMS = 2e-2
BF16_ELT_REL = 2.0 ** -8
BF16_ELT_RMS = 0.1
NAMES = ("dq", "dk", "dv", "dlog_alpha")


@pytest.fixture(scope="module")
def dig():
    import gated_linear_attention_chunkwise_b200 as pkg
    return pkg


def per_head(a):
    B, T, H, d = a.shape
    return a.transpose(0, 2, 1, 3).reshape(B * H, T, d)


def check(got, ref, name, bf16_store, elt_rms=BF16_ELT_RMS):
    assert np.all(np.isfinite(got)), name
    g, r = per_head(got), per_head(ref)
    for h in range(g.shape[0]):
        err = g[h] - r[h]
        rms = math.sqrt(float(np.mean(r[h] ** 2))) if r[h].size else 0.0
        rel = float(np.linalg.norm(err) / max(np.linalg.norm(r[h]), 1e-300))
        if bf16_store:
            assert rel <= BF16_REL_RMS, f"{name} head {h}: relative RMS {rel:.3e}"
            bound = BF16_ELT_REL * np.abs(r[h]) + elt_rms * rms
            worst = float(np.max(np.abs(err) - bound)) if err.size else -1.0
            assert worst <= 0.0, f"{name} head {h}: element bound exceeded by {worst:.3e} (RMS {rms:.3e})"
        else:
            assert float(np.max(np.abs(err))) <= F32_MAX_ABS, f"{name} head {h}: max-abs {np.max(np.abs(err)):.3e}"
            if rms > 1e-12:
                assert rel <= F32_REL_RMS, f"{name} head {h}: relative RMS {rel:.3e}"


def run_case(dig, w, direction, seed=0, la=None, heads=None):
    q, k, v, la0 = workloads.gla_inputs(w, seed=seed)
    la = la0 if la is None else la
    do = workloads.gla_dout(w, seed=seed)
    dev = [t.to("cuda") for t in (q, k, v, la, do)]
    fn = dig.gla_bwd if w.dtype == "bf16" else dig.gla_bwd_f32
    got = fn(*dev, w.Hgrid, w.Wgrid, direction)
    torch.cuda.synchronize()
    assert dig.device_status() == 0
    got = [t.float().cpu().numpy().astype(np.float64) for t in got]
    if heads is None:
        ref = oracle.gla_bwd(q, k, v, la, do, w.Hgrid, w.Wgrid, direction)
        for g, r, n in zip(got, ref, NAMES):
            check(g, r, n, w.dtype == "bf16")
        return got, ref
    for lo, hi in heads:
        ref = oracle.gla_bwd(q, k, v, la, do, w.Hgrid, w.Wgrid, direction, nthreads=1, heads=(lo, hi))
        for g, r, n in zip(got, ref, NAMES):
            check(per_head(g)[lo:hi][None].transpose(0, 2, 1, 3), per_head(r)[lo:hi][None].transpose(0, 2, 1, 3),
                  f"{n} heads {lo}:{hi}", w.dtype == "bf16")
    return got, None


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_bwd_f32_c1(dig, direction):
    """The fp32 workload (B=2, H=6, 16x16, d=64), every direction."""
    run_case(dig, workloads.WORKLOADS["c1"], direction)


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_bwd_bf16_c2(dig, direction):
    """DiG-S/2 at 512 (B=8, H=6, 32x32, d=64): the whole workload."""
    run_case(dig, workloads.WORKLOADS["c2"], direction)


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_bwd_ragged_d72(dig, direction, dtype):
    """d = 72 (the DiG-XL/2 head width), a 9x23 grid: 207 tokens, six full chunks of
    32 and a ragged one; columns of 9 split across chunks."""
    run_case(dig, workloads.custom(2, 3, 9, 23, 72, 72, dtype), direction, seed=4)


@pytest.mark.parametrize("dims", [(128, 128), (32, 96), (88, 40)])
def test_bwd_wide_heads(dig, dims):
    """Heads wider than 80 channels (the largest shared-memory footprint) and dk != dv."""
    dk, dv = dims
    for direction in (0, 3):
        run_case(dig, workloads.custom(1, 2, 7, 11, dk, dv, "bf16"), direction, seed=5)


@pytest.mark.parametrize("dims", [(8, 8), (16, 80), (80, 16), (48, 72), (80, 80)])
def test_bwd_tensor_core_head_shapes(dig, dims):
    """bf16 heads of at most 80 channels take the tensor-core kernels: the smallest
    head, dk != dv both ways, and the widest (80 x 80, where only S_in and D are staged
    with the tiles and the end-of-chunk carry reads S_out from global memory); a 9x23
    grid gives one full 128-row chunk and a ragged one."""
    dk, dv = dims
    for direction in (0, 3):
        run_case(dig, workloads.custom(1, 2, 9, 23, dk, dv, "bf16"), direction, seed=21)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bwd_tiny_and_single_token(dig, dtype):
    """One token, one row of five, a 3x2 grid: a single, mostly empty chunk (on the
    tensor-core path for bf16: 127 of 128 rows padding for the single token)."""
    for Hg, Wg in [(1, 1), (1, 5), (3, 2)]:
        for direction in range(4):
            run_case(dig, workloads.custom(1, 2, Hg, Wg, 16, 8, dtype), direction, seed=6)


@pytest.mark.parametrize("direction", [0, 2, 3])
def test_bwd_resets_and_strong_decays(dig, direction):
    """Full resets (-inf) and decays of e^-30 per token in a few places: those chunks
    take the exact token-by-token sweep, the rest the factorised form."""
    for dtype in ("f32", "bf16"):
        w = workloads.custom(2, 2, 12, 17, 64, 64, dtype)
        _, _, _, la = workloads.gla_inputs(w, seed=7)
        gen = torch.Generator().manual_seed(8)
        m = torch.rand(la.shape, generator=gen)
        la = torch.where(m < 0.004, torch.full_like(la, -math.inf), la)
        la = torch.where((m >= 0.004) & (m < 0.01), torch.full_like(la, -30.0), la)
        run_case(dig, w, direction, seed=7, la=la)


def test_bwd_ungated_and_mild_growth(dig):
    """log_alpha = 0 (masked causal linear attention) and small growth gates."""
    w = workloads.custom(1, 2, 10, 13, 64, 64, "f32")
    _, _, _, la = workloads.gla_inputs(w, seed=9)
    run_case(dig, w, 1, seed=9, la=torch.zeros_like(la))
    run_case(dig, w, 2, seed=9, la=la.abs() * 0.05)


def test_bwd_c4_sampled_heads(dig):
    """DiG-XL/2 at 1792 (B=2, H=16, 112x112, d=72) in bf16, the launch the benchmark
    times: flattened heads 0, 15 and 31 against the oracle, two directions."""
    w = workloads.WORKLOADS["c4"]
    for direction in (0, 3):
        run_case(dig, w, direction, seed=1, heads=[(0, 1), (15, 16), (31, 32)])


def test_bwd_deterministic(dig):
    w = workloads.custom(2, 2, 16, 16, 64, 64, "bf16")
    q, k, v, la = (t.cuda() for t in workloads.gla_inputs(w, seed=2))
    do = workloads.gla_dout(w, seed=2).cuda()
    a = dig.gla_bwd(q, k, v, la, do, 16, 16, 2)
    b = dig.gla_bwd(q, k, v, la, do, 16, 16, 2)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int16) if x.dtype == torch.bfloat16 else x.view(torch.int32),
                           y.view(torch.int16) if y.dtype == torch.bfloat16 else y.view(torch.int32))


def test_bwd_rejects_bad_arguments(dig):
    w = workloads.custom(1, 2, 4, 4, 64, 64, "bf16")
    q, k, v, la = (t.cuda() for t in workloads.gla_inputs(w))
    do = workloads.gla_dout(w).cuda()
    L = dig.lib()
    st = torch.cuda.current_stream().cuda_stream
    dq, dk_, dv_, dla = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(la)
    args = [q.data_ptr(), k.data_ptr(), v.data_ptr(), la.data_ptr(), do.data_ptr(), 1, 2, 4, 4, 64, 64, 0,
            dq.data_ptr(), dk_.data_ptr(), dv_.data_ptr(), dla.data_ptr(), st]
    bad = list(args)
    bad[15] = la.data_ptr()            # dlog_alpha over an input
    assert L.gla_bwd(*bad) == -1
    bad = list(args)
    bad[13] = dq.data_ptr()            # two outputs on one buffer
    assert L.gla_bwd(*bad) == -1
    bad = list(args)
    bad[9] = 12                        # dk not a multiple of 8
    assert L.gla_bwd(*bad) == -2
    bad = list(args)
    bad[4] = None
    assert L.gla_bwd(*bad) == -1
    assert L.gla_bwd(*args) == 0
    assert dig.device_status() == 0
