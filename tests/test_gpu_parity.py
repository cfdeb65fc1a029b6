"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Tolerances (the GLA path's stated bars: max-abs 1e-4 for fp32 inputs, 2e-2
relative to RMS for bf16 inputs with fp32 state):
  * bf16 q/k/v, fp32 state.  Three gates, each per (batch, head):
      - relative RMS error  ||gpu - oracle||_2 / ||oracle||_2 <= 2e-2;
      - every block of 128 consecutive tokens: RMS of the error <= 2e-2 * RMS of
        the head's oracle output (localised damage, such as one wrong chunk,
        fails here even when the head's norm hides it);
      - every element: |gpu - oracle| <= 2^-8 |oracle| + 0.1 * RMS(head).  2^-8
        |oracle| is the worst case of rounding the exact value to bf16 (half an
        ulp with an 8-bit significand); 0.1 RMS is about the largest of 10^5-10^7
        Gaussian deviations whose RMS sits at the 2e-2 bar (5 sigma).
    A max-abs reading of "2e-2 relative to RMS" cannot be met by a bf16 output:
    rounding the exact result to bf16 alone moves the largest outputs (about 7 RMS)
    by up to 7 * 2^-8 RMS = 0.027 RMS.
  * fp32 q/k/v/out: max-abs error <= 1e-4.
  * reorientation: bit-exact.
  * bf16 conv: every element within 2^-8 |oracle| + 1e-5 RMS (bf16 rounding of
    an fp32 accumulation), identity kernel bit-exact; fp32 conv: max-abs
    <= 1e-5 * (1 + |y|).
Inputs come from workloads.py (seeded, synthetic) for both sides.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

BF16_REL_RMS = 2e-2
F32_MAX_ABS = 1e-4


@pytest.fixture(scope="module")
def dig():
    import gated_linear_attention_chunkwise_b200 as pkg
    return pkg


def rel_rms(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def to_dev(*ts):
    return [t.to("cuda") for t in ts]


def gpu_gla(dig, q, k, v, la, Hg, Wg, d):
    qd, kd, vd, ld = to_dev(q, k, v, la)
    fn = dig.gla_fwd if q.dtype == torch.bfloat16 else dig.gla_fwd_f32
    out = fn(qd, kd, vd, ld, Hg, Wg, d)
    assert dig.device_status() == 0
    return out.float().cpu().numpy().astype(np.float64)


def heads_view(a: np.ndarray, lo: int, hi: int, H: int) -> np.ndarray:
    """Rows of flattened heads bh in [lo, hi) from a [B, T, H, d] array."""
    B, T, _, d = a.shape
    flat = a.transpose(0, 2, 1, 3).reshape(B * H, T, d)
    return flat[lo:hi]


BF16_ELT_REL = 2.0 ** -8      # bf16 rounding of the exact value (half ulp, 8-bit significand)
BF16_ELT_RMS = 0.1            # 5 sigma of an error field at the 2e-2 RMS bar
BLOCK = 128                   # tokens per block of the local RMS gate


def check_bf16(got, ref, what, scan=None):
    """The three bf16 gates (see the module docstring).  got/ref: [B, T, H, d] or
    [n, T, d] arrays of float64.  scan = (Hgrid, Wgrid, dir): the blocks of the
    local gate are then cut in that scan order (the kernel's chunk order)."""
    assert np.all(np.isfinite(got)), what
    if got.ndim == 4:
        B, T, H, d = got.shape
        got = got.transpose(0, 2, 1, 3).reshape(B * H, T, d)
        ref = ref.transpose(0, 2, 1, 3).reshape(B * H, T, d)
    if scan is not None:
        order = oracle.scan_order(scan[2], scan[0], scan[1])
        got, ref = got[:, order], ref[:, order]
    n, T, d = got.shape
    err = got - ref
    rms = np.sqrt(np.mean(ref ** 2, axis=(1, 2)))                      # per head
    rel = np.sqrt(np.mean(err ** 2, axis=(1, 2))) / np.maximum(rms, 1e-300)
    nb = -(-T // BLOCK)
    pad = nb * BLOCK - T
    e2 = np.pad(err ** 2, ((0, 0), (0, pad), (0, 0)))
    cnt = np.pad(np.ones((T,)), (0, pad)).reshape(nb, BLOCK).sum(1)
    blk = np.sqrt(e2.reshape(n, nb, BLOCK, d).sum(axis=(2, 3)) / (cnt[None, :] * d)) / np.maximum(rms[:, None], 1e-300)
    bound = BF16_ELT_REL * np.abs(ref) + BF16_ELT_RMS * rms[:, None, None]
    ratio = np.abs(err) / np.maximum(bound, 1e-300)
    mx = float(np.max(np.abs(err) / np.maximum(rms[:, None, None], 1e-300)))
    print(f"{what}: rel_rms max/head={rel.max():.3e} block_rms max={blk.max():.3e} "
          f"max_abs/rms={mx:.3e} element bound use={ratio.max():.3f}")
    assert rel.max() <= BF16_REL_RMS, f"{what}: relative RMS error {rel.max():.3e} > {BF16_REL_RMS} (head {rel.argmax()})"
    hb = np.unravel_index(np.argmax(blk), blk.shape)
    assert blk.max() <= BF16_REL_RMS, f"{what}: block RMS error {blk.max():.3e} > {BF16_REL_RMS} at head/block {hb}"
    bad = np.unravel_index(np.argmax(ratio), ratio.shape)
    assert ratio.max() <= 1.0, (f"{what}: element {bad} off by {abs(err[bad]):.3e} "
                                f"(oracle {ref[bad]:.3e}, head RMS {rms[bad[0]]:.3e})")


def check_conv_bf16(got, ref, what):
    """bf16 conv: each element within the bf16 rounding of an fp32 accumulation."""
    assert np.all(np.isfinite(got)), what
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = np.abs(got - ref)
    ratio = err / (BF16_ELT_REL * np.abs(ref) + 1e-5 * rms)
    print(f"{what}: rel_rms={rel_rms(got, ref):.3e} max_abs/rms={err.max() / max(rms, 1e-300):.3e} "
          f"element bound use={ratio.max():.3f}")
    assert ratio.max() <= 1.0, f"{what}: element off by {err.max():.3e}"


# --------------------------------------------------------------------------- reorientation
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("Hg,Wg,C", [(32, 32, 384), (10, 13, 64), (7, 5, 8), (1, 1, 8), (112, 112, 1152)])
@pytest.mark.parametrize("d", [0, 1, 2, 3])
def test_reorient_bit_exact(dig, dtype, Hg, Wg, C, d):
    if C * (2 if dtype == torch.bfloat16 else 4) % 16:
        pytest.skip("row pitch must be a multiple of 16 bytes")
    B = 2
    x = workloads.grid_tensor(B, Hg, Wg, C, dtype=dtype, seed=d)
    xd = x.to("cuda").view(B, Hg * Wg, C)
    for inverse in (0, 1):
        y = dig.srem_reorient(xd, d, inverse, Hg, Wg)
        raw = x.view(B, Hg * Wg, C).view(torch.int16 if dtype == torch.bfloat16 else torch.int32).numpy()
        want = oracle.reorient(raw, d, inverse, Hg, Wg)
        got = y.cpu().view(torch.int16 if dtype == torch.bfloat16 else torch.int32).numpy()
        np.testing.assert_array_equal(got, want)
        back = dig.srem_reorient(y, d, 1 - inverse, Hg, Wg)
        assert torch.equal(back.view(torch.int16 if dtype == torch.bfloat16 else torch.int32),
                           xd.view(torch.int16 if dtype == torch.bfloat16 else torch.int32))


# --------------------------------------------------------------------------- conv
@pytest.mark.parametrize("B,Hg,Wg,C", [(8, 32, 32, 384), (1, 10, 13, 64), (2, 3, 5, 8), (1, 1, 1, 8),
                                       (2, 112, 112, 1152), (1, 17, 3, 24)])
def test_dwconv_bf16(dig, B, Hg, Wg, C):
    x = workloads.grid_tensor(B, Hg, Wg, C, dtype=torch.bfloat16, seed=C)
    w = workloads.conv_weight(C, seed=Hg)
    y = dig.dwconv3x3(x.to("cuda"), w.to("cuda")).float().cpu().numpy()
    check_conv_bf16(y, oracle.dwconv3x3(x, w), f"dwconv bf16 {B}x{Hg}x{Wg}x{C}")


@pytest.mark.parametrize("B,Hg,Wg,C", [(2, 16, 16, 64), (1, 10, 13, 4), (1, 9, 1, 12)])
def test_dwconv_f32(dig, B, Hg, Wg, C):
    x = workloads.grid_tensor(B, Hg, Wg, C, dtype=torch.float32, seed=1)
    w = workloads.conv_weight(C, seed=2, noise=0.3)
    y = dig.dwconv3x3(x.to("cuda"), w.to("cuda")).cpu().numpy()
    ref = oracle.dwconv3x3(x, w)
    assert np.all(np.abs(y - ref) <= 1e-5 * (1 + np.abs(ref)))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_dwconv_identity_kernel_is_exact(dig, dtype):
    """SREM's identity initialisation: centre 1, rest 0 -> output == input bit for bit."""
    x = workloads.grid_tensor(2, 13, 11, 64, dtype=dtype, seed=5)
    w = torch.zeros(64, 3, 3)
    w[:, 1, 1] = 1
    y = dig.dwconv3x3(x.to("cuda"), w.to("cuda")).cpu()
    assert torch.equal(y, x)


# --------------------------------------------------------------------------- GLA bf16
SMALL_CASES = [
    # (B, H, Hg, Wg, dk, dv)
    (2, 2, 16, 16, 64, 64),     # two full chunks
    (1, 3, 10, 13, 64, 64),     # ragged tail (T = 130), column runs of 10
    (1, 2, 12, 12, 64, 72),     # dk != dv
    (1, 2, 12, 12, 72, 64),
    (2, 1, 9, 15, 72, 72),      # T = 135
    (1, 1, 3, 5, 64, 64),       # a single partial chunk
    (1, 2, 8, 40, 8, 8),        # smallest dims
    (1, 1, 20, 13, 128, 128),   # largest dims
    (1, 2, 16, 24, 16, 48),
    (1, 1, 1, 1, 64, 64),       # T = 1
    (1, 2, 130, 3, 64, 64),     # columns longer than a chunk: two pieces per column
]


@pytest.mark.parametrize("case", SMALL_CASES, ids=lambda c: "x".join(map(str, c)))
@pytest.mark.parametrize("d", [0, 1, 2, 3])
def test_gla_bf16_small(dig, case, d):
    B, H, Hg, Wg, dk, dv = case
    w = workloads.custom(B, H, Hg, Wg, dk, dv, "bf16")
    q, k, v, la = workloads.gla_inputs(w, seed=11 * d + dk)
    got = gpu_gla(dig, q, k, v, la, Hg, Wg, d)
    check_bf16(got, oracle.gla_fwd(q, k, v, la, Hg, Wg, d), f"gla bf16 {case} dir{d}", (Hg, Wg, d))


@pytest.mark.parametrize("name", ["c2", "c3"])
@pytest.mark.parametrize("d", [0, 1, 2, 3])
def test_gla_bf16_full_config(dig, name, d):
    w = workloads.WORKLOADS[name]
    q, k, v, la = workloads.gla_inputs(w, seed=d)
    got = gpu_gla(dig, q, k, v, la, w.Hgrid, w.Wgrid, d)
    check_bf16(got, oracle.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, d), f"gla {name} dir{d}", (w.Hgrid, w.Wgrid, d))


@pytest.mark.parametrize("name,heads", [("c4", (0, 3)), ("c4", (15, 17)), ("c4", (29, 32)), ("c5", (0, 2)), ("c5", (7, 9)),
                                        ("c5", (14, 16))])
@pytest.mark.parametrize("d", [0, 1, 2, 3])
def test_gla_bf16_large_config_sampled_heads(dig, name, heads, d):
    """Full-size launch; the oracle recomputes a sample of whole heads."""
    w = workloads.WORKLOADS[name]
    q, k, v, la = workloads.gla_inputs(w, seed=d)
    got = gpu_gla(dig, q, k, v, la, w.Hgrid, w.Wgrid, d)
    ref = oracle.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, d, heads=heads)
    check_bf16(heads_view(got, *heads, w.H), heads_view(ref, *heads, w.H), f"gla {name} heads{heads} dir{d}",
               (w.Hgrid, w.Wgrid, d))


def test_gla_bf16_ungated(dig):
    """log_alpha = 0: masked causal linear attention."""
    w = workloads.custom(1, 2, 16, 20, 64, 64, "bf16")
    q, k, v, _ = workloads.gla_inputs(w, seed=3)
    la = torch.zeros(q.shape, dtype=torch.float32)
    for d in range(4):
        check_bf16(gpu_gla(dig, q, k, v, la, 16, 20, d), oracle.gla_fwd(q, k, v, la, 16, 20, d), f"ungated dir{d}",
                   (16, 20, d))


@pytest.mark.parametrize("fill", [-1e4, -math.inf])
def test_gla_bf16_full_forget(dig, fill):
    """alpha -> 0: every output is (q_t . k_t) v_t; the chunks take the exact serial path."""
    w = workloads.custom(1, 2, 12, 17, 72, 72, "bf16")
    q, k, v, _ = workloads.gla_inputs(w, seed=4)
    la = torch.full(q.shape, fill, dtype=torch.float32)
    for d in range(4):
        got = gpu_gla(dig, q, k, v, la, 12, 17, d)
        want = (q.double() * k.double()).sum(-1, keepdim=True) * v.double()
        check_bf16(got, want.numpy(), f"full forget {fill} dir{d}", (12, 17, d))


def test_gla_bf16_mixed_resets(dig):
    """Random full resets (-inf) and strong decays mixed into ordinary gates."""
    w = workloads.custom(2, 2, 24, 24, 64, 64, "bf16")
    q, k, v, la = workloads.gla_inputs(w, seed=8)
    gen = torch.Generator().manual_seed(8)
    m = torch.rand(la.shape, generator=gen)
    la = torch.where(m < 0.01, torch.full_like(la, -math.inf), la)
    la = torch.where((m >= 0.01) & (m < 0.03), torch.full_like(la, -30.0), la)
    for d in range(4):
        check_bf16(gpu_gla(dig, q, k, v, la, 24, 24, d), oracle.gla_fwd(q, k, v, la, 24, 24, d), f"mixed dir{d}",
                   (24, 24, d))


def test_gla_growth_overflow_is_reported(dig):
    """log_alpha = +2 everywhere grows the state by e^256 per chunk: the library
    records GLA_ERR_RANGE in the device status instead of failing silently."""
    w = workloads.custom(1, 1, 16, 16, 64, 64, "bf16")
    q, k, v, _ = workloads.gla_inputs(w, seed=1)
    la = torch.full(q.shape, 2.0, dtype=torch.float32)
    qd, kd, vd, ld = to_dev(q, k, v, la)
    dig.gla_fwd(qd, kd, vd, ld, 16, 16, 0)
    assert dig.device_status() == -7
    assert dig.device_status() == 0       # read-and-clear


def test_gla_deterministic_and_guarded(dig):
    """Two calls agree bit for bit, and nothing is written outside `out`."""
    w = workloads.custom(2, 3, 10, 13, 72, 72, "bf16")
    q, k, v, la = to_dev(*workloads.gla_inputs(w, seed=6))
    n = q.shape[0] * q.shape[1] * q.shape[2] * 72
    guard = 4096
    buf = torch.full((n + 2 * guard,), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = buf[guard:guard + n].view(q.shape[0], q.shape[1], q.shape[2], 72)
    for d in range(4):
        a = dig.gla_fwd(q, k, v, la, 10, 13, d, out=out).clone()
        b = dig.gla_fwd(q, k, v, la, 10, 13, d)
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
        assert torch.isnan(buf[:guard].float()).all() and torch.isnan(buf[guard + n:].float()).all()


def test_gla_on_side_stream(dig):
    w = workloads.custom(1, 2, 16, 16, 64, 64, "bf16")
    q, k, v, la = workloads.gla_inputs(w, seed=2)
    qd, kd, vd, ld = to_dev(q, k, v, la)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = dig.gla_fwd(qd, kd, vd, ld, 16, 16, 2)
    s.synchronize()
    check_bf16(out.float().cpu().numpy(), oracle.gla_fwd(q, k, v, la, 16, 16, 2), "side stream", (16, 16, 2))


def test_gla_lookback_wait_runs_out_and_reports_timeout(dig):
    """A look-back flag that nothing sets: the wait gives up, the status word says so,
    and the context stays usable.  32x32 grid = 8 chunks = 3 segments, one head; the
    test hook leaves out segment 0, whose flags the other two segments wait for."""
    import time
    w = workloads.custom(1, 1, 32, 32, 64, 64, "bf16")
    q, k, v, la = workloads.gla_inputs(w, seed=4)
    qd, kd, vd, ld = to_dev(q, k, v, la)
    assert dig.device_status() == 0
    dig.skip_items_for_test(1)
    t0 = time.monotonic()
    dig.gla_fwd(qd, kd, vd, ld, 32, 32, 0)
    status = dig.device_status()
    waited = time.monotonic() - t0
    print(f"bounded look-back wait: status {dig.status_string(status)} after {waited:.2f} s")
    assert status == -5  # GLA_ERR_TIMEOUT
    assert waited < 60.0
    # The hook applies to one call only, and the next call is exact again.
    got = gpu_gla(dig, q, k, v, la, 32, 32, 0)
    check_bf16(got, oracle.gla_fwd(q, k, v, la, 32, 32, 0), "after a timed-out call", (32, 32, 0))


# --------------------------------------------------------------------------- GLA fp32
def test_gla_f32_config_c1(dig):
    w = workloads.WORKLOADS["c1"]
    q, k, v, la = workloads.gla_inputs(w, seed=0)
    got = gpu_gla(dig, q, k, v, la, w.Hgrid, w.Wgrid, 0)
    err = float(np.max(np.abs(got - oracle.gla_fwd(q, k, v, la, w.Hgrid, w.Wgrid, 0))))
    print(f"c1 fp32 max-abs error {err:.3e}")
    assert err <= F32_MAX_ABS


@pytest.mark.parametrize("case", [(1, 2, 10, 13, 64, 64), (1, 1, 12, 12, 72, 40), (2, 1, 3, 5, 8, 8),
                                  (1, 1, 9, 20, 128, 128)], ids=lambda c: "x".join(map(str, c)))
@pytest.mark.parametrize("d", [0, 1, 2, 3])
def test_gla_f32_small(dig, case, d):
    B, H, Hg, Wg, dk, dv = case
    w = workloads.custom(B, H, Hg, Wg, dk, dv, "f32")
    q, k, v, la = workloads.gla_inputs(w, seed=d + 100)
    got = gpu_gla(dig, q, k, v, la, Hg, Wg, d)
    assert np.max(np.abs(got - oracle.gla_fwd(q, k, v, la, Hg, Wg, d))) <= F32_MAX_ABS


def test_gla_f32_full_forget_and_resets(dig):
    w = workloads.custom(1, 2, 11, 9, 64, 64, "f32")
    q, k, v, la = workloads.gla_inputs(w, seed=9)
    gen = torch.Generator().manual_seed(9)
    la = torch.where(torch.rand(la.shape, generator=gen) < 0.05, torch.full_like(la, -math.inf), la)
    for d in range(4):
        got = gpu_gla(dig, q, k, v, la, 11, 9, d)
        assert np.max(np.abs(got - oracle.gla_fwd(q, k, v, la, 11, 9, d))) <= F32_MAX_ABS
    la = torch.full(q.shape, -1e4)
    got = gpu_gla(dig, q, k, v, la, 11, 9, 1)
    want = ((q.double() * k.double()).sum(-1, keepdim=True) * v.double()).numpy()
    assert np.max(np.abs(got - want)) <= F32_MAX_ABS


# --------------------------------------------------------------------------- guards and repeats
def _guarded(shape, dtype, guard=4096):
    """A NaN-filled buffer with `guard` elements on each side of a view of `shape`."""
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * guard,), float("nan"), dtype=dtype, device="cuda")
    return buf, buf[guard:guard + n].view(*shape), guard, n


def _guards_intact(buf, guard, n):
    return bool(torch.isnan(buf[:guard].float()).all() and torch.isnan(buf[guard + n:].float()).all())


def _bits(t):
    return t.view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_dwconv_deterministic_and_guarded(dig, dtype):
    x = workloads.grid_tensor(2, 13, 11, 64, dtype=dtype, seed=7).cuda()
    w = workloads.conv_weight(64, seed=3, noise=0.2).cuda()
    buf, out, guard, n = _guarded(tuple(x.shape), dtype)
    a = dig.dwconv3x3(x, w, out=out).clone()
    b = dig.dwconv3x3(x, w)
    assert torch.equal(_bits(a), _bits(b))
    assert _guards_intact(buf, guard, n)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_reorient_guarded(dig, dtype):
    B, Hg, Wg, C = 2, 10, 13, 64
    x = workloads.grid_tensor(B, Hg, Wg, C, dtype=dtype, seed=8).cuda().view(B, Hg * Wg, C)
    for d in range(4):
        for inverse in (0, 1):
            buf, out, guard, n = _guarded((B, Hg * Wg, C), dtype)
            a = dig.srem_reorient(x, d, inverse, Hg, Wg, out=out).clone()
            b = dig.srem_reorient(x, d, inverse, Hg, Wg)
            assert torch.equal(_bits(a), _bits(b))
            assert _guards_intact(buf, guard, n)


def test_gla_f32_deterministic_and_guarded(dig):
    w = workloads.custom(2, 3, 10, 13, 72, 40, "f32")
    q, k, v, la = to_dev(*workloads.gla_inputs(w, seed=12))
    for d in range(4):
        buf, out, guard, n = _guarded((w.B, w.T, w.H, w.dv), torch.float32)
        a = dig.gla_fwd_f32(q, k, v, la, w.Hgrid, w.Wgrid, d, out=out).clone()
        b = dig.gla_fwd_f32(q, k, v, la, w.Hgrid, w.Wgrid, d)
        assert torch.equal(_bits(a), _bits(b))
        assert _guards_intact(buf, guard, n)
