"""Pins for the fp64 CPU oracle -- checked against mathematics, not against itself.

Every check below derives its expected value independently of the oracle's code:
  * scan orders from closed-form index formulas (and group identities) instead of
    the oracle's transpose-and-flip table;
  * the GLA recurrence from the O(T^2) unrolled sum
        o_t = sum_{s<=t} (q_t * prod_{r=s+1..t} alpha_r) . k_s  v_s
    (the recurrence S_t = Diag(alpha_t) S_{t-1} + k_t^T v_t, o_t = q_t S_t
    written out), and from textbook special cases: log_alpha = 0 is masked causal
    linear attention (Q K^T * M) V; a constant per-channel gate gives the decay
    matrix gamma^(t-s); log_alpha -> -inf leaves only (q_t . k_t) v_t;
  * the conv from the identity / shifted-delta kernels (the SREM identity
    initialisation, DiG notes "SREM") and from torch's grouped conv2d;
  * planted mistakes in the oracle must each fail at least one of these pins.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------- helpers
def zigzag_closed_form(j, Hg, Wg):
    """Zigzag scheme j (scan order code 4 + j) from index formulas: line k of the walk
    and position i along it, the line's grid index, the walking direction by parity."""
    T = Hg * Wg
    p = np.arange(T)
    cols = j >= 4
    nl, ln = (Wg, Hg) if cols else (Hg, Wg)
    k, i = p // ln, p % ln
    line = nl - 1 - k if (j >> 1) & 1 else k
    backwards = (k % 2 == 1) ^ bool(j & 1)
    at = np.where(backwards, ln - 1 - i, i)
    y, x = (at, line) if cols else (line, at)
    return y * Wg + x


def closed_form_order(direction, Hg, Wg):
    """Scan position -> raster token id, from closed-form index formulas."""
    T = Hg * Wg
    p = np.arange(T)
    if direction >= 4:
        return zigzag_closed_form(direction - 4, Hg, Wg)
    if direction == 0:
        return p
    if direction == 1:
        return T - 1 - p
    col_major = (p % Hg) * Wg + p // Hg
    if direction == 2:
        return col_major
    return col_major[T - 1 - p]


def rand_inputs(rng, B, H, Hg, Wg, dk, dv, gate_scale=1.0):
    T = Hg * Wg
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    la = -np.abs(rng.standard_normal((B, T, H, dk))) * gate_scale
    return q, k, v, la


def bruteforce(q, k, v, la, Hg, Wg, direction):
    """O(T^2) unrolled sum over scan positions (numpy, fp64)."""
    B, T, H, dk = q.shape
    order = closed_form_order(direction, Hg, Wg)
    out = np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            Q = q[b, order, h]      # [T, dk] in scan order
            K = k[b, order, h]
            V = v[b, order, h]
            L = la[b, order, h]
            csum = np.concatenate([np.zeros((1, dk)), np.cumsum(L, axis=0)])  # csum[p] = sum_{r<p}
            for p in range(T):
                acc = np.zeros(V.shape[1])
                for s in range(p + 1):
                    decay = np.exp(csum[p + 1] - csum[s + 1])   # prod_{r=s+1..p} alpha_r
                    acc += np.dot(Q[p] * decay, K[s]) * V[s]
                out[b, order[p], h] = acc
    return out


def oracle_gla(q, k, v, la, Hg, Wg, d, planted=0):
    return oracle.gla_fwd(q, k, v, la, Hg, Wg, d, nthreads=1, planted=planted)


GRIDS = [(3, 5), (4, 4), (1, 7), (5, 2), (2, 3)]


# --------------------------------------------------------------------------- pins as functions
# Each pin takes a GLA callable and returns True when it holds; the planted-mistake
# test reuses them.
def pin_bruteforce(gla, rng):
    for (Hg, Wg) in [(3, 5), (4, 3)]:
        q, k, v, la = rand_inputs(rng, 1, 2, Hg, Wg, 4, 3 if Hg == 3 else 4, gate_scale=0.7)
        for d in range(4):
            got = gla(q, k, v, la, Hg, Wg, d)
            if not np.allclose(got, bruteforce(q, k, v, la, Hg, Wg, d), rtol=1e-12, atol=1e-12):
                return False
    return True


def pin_ungated_is_masked_linear_attention(gla, rng):
    Hg, Wg, dk, dv = 4, 5, 6, 6
    q, k, v, _ = rand_inputs(rng, 2, 2, Hg, Wg, dk, dv)
    la = np.zeros(q.shape)
    for d in range(4):
        got = gla(q, k, v, la, Hg, Wg, d)
        order = closed_form_order(d, Hg, Wg)
        for b in range(2):
            for h in range(2):
                Q, K, V = q[b, order, h], k[b, order, h], v[b, order, h]
                ref = np.tril(Q @ K.T) @ V
                if not np.allclose(got[b, order, h], ref, rtol=1e-12, atol=1e-12):
                    return False
    return True


def pin_constant_gate_closed_form(gla, rng):
    Hg, Wg, dk, dv = 3, 6, 5, 5
    q, k, v, _ = rand_inputs(rng, 1, 1, Hg, Wg, dk, dv)
    gam = np.exp(-rng.uniform(0.05, 1.5, size=dk))           # one constant gate per key channel
    la = np.broadcast_to(np.log(gam), q.shape).copy()
    T = Hg * Wg
    for d in range(4):
        got = gla(q, k, v, la, Hg, Wg, d)
        order = closed_form_order(d, Hg, Wg)
        Q, K, V = q[0, order, 0], k[0, order, 0], v[0, order, 0]
        tt = np.arange(T)
        lag = tt[:, None] - tt[None, :]                       # t - s
        Dm = np.where(lag[:, :, None] >= 0, gam[None, None, :] ** np.maximum(lag, 0)[:, :, None], 0.0)
        A = np.einsum("ti,si,tsi->ts", Q, K, Dm)              # (Q K^T * gamma^(t-s)) per channel
        if not np.allclose(got[0, order, 0], A @ V, rtol=1e-12, atol=1e-12):
            return False
    return True


def pin_full_forget(gla, rng):
    Hg, Wg, dk, dv = 3, 4, 4, 6
    q, k, v, _ = rand_inputs(rng, 1, 3, Hg, Wg, dk, dv)
    la = np.full(q.shape, -1e4)                               # alpha = exp(-1e4) = 0 in fp64
    want = np.einsum("bthi,bthi->bth", q, k)[..., None] * v
    for d in range(4):
        if not np.allclose(gla(q, k, v, la, Hg, Wg, d), want, rtol=1e-13, atol=1e-13):
            return False
    return True


def pin_direction_conjugation(gla, rng):
    """dir d on x equals dir 0 on the scan-permuted tokens, mapped back."""
    Hg, Wg, dk, dv = 4, 3, 3, 5
    q, k, v, la = rand_inputs(rng, 1, 2, Hg, Wg, dk, dv, gate_scale=0.5)
    base = lambda a, order: a[:, order]
    for d in (1, 2, 3):
        order = closed_form_order(d, Hg, Wg)
        T = Hg * Wg
        # dir 0 over a 1 x T grid of the permuted tokens is a plain causal scan of them
        o0 = gla(base(q, order), base(k, order), base(v, order), base(la, order), 1, T, 0)
        back = np.empty_like(o0)
        back[:, order] = o0
        if not np.allclose(gla(q, k, v, la, Hg, Wg, d), back, rtol=1e-12, atol=1e-12):
            return False
    return True


ALL_PINS = [pin_bruteforce, pin_ungated_is_masked_linear_attention, pin_constant_gate_closed_form,
            pin_full_forget, pin_direction_conjugation]


# --------------------------------------------------------------------------- scan order
@pytest.mark.parametrize("Hg,Wg", GRIDS + [(16, 16), (7, 13), (1, 1)])
@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_scan_order_closed_form_and_bijection(Hg, Wg, direction):
    got = oracle.scan_order(direction, Hg, Wg)
    np.testing.assert_array_equal(got, closed_form_order(direction, Hg, Wg))
    assert np.array_equal(np.sort(got), np.arange(Hg * Wg))       # a bijection on [0, T)


@pytest.mark.parametrize("n", [1, 2, 5, 8])
def test_scan_orders_form_klein_group_on_square_grids(n):
    """On a square grid flip and transpose are commuting involutions, so the four
    orders {id, flip, transpose, transpose.flip} form the Klein four-group."""
    P = [oracle.scan_order(d, n, n) for d in range(4)]
    ident = np.arange(n * n)
    for d in range(4):
        np.testing.assert_array_equal(P[d][P[d]], ident)          # each is an involution
    np.testing.assert_array_equal(P[1][P[2]], P[3])
    np.testing.assert_array_equal(P[2][P[1]], P[3])


def test_scan_order_transpose_inverse_nonsquare():
    """The inverse of the T->B order on Hg x Wg is the T->B order on the Wg x Hg grid."""
    Hg, Wg = 3, 7
    P = oracle.scan_order(2, Hg, Wg)
    inv = np.empty_like(P)
    inv[P] = np.arange(Hg * Wg)
    np.testing.assert_array_equal(inv, oracle.scan_order(2, Wg, Hg))
    # flip is an involution on any grid
    F = oracle.scan_order(1, Hg, Wg)
    np.testing.assert_array_equal(F[F], np.arange(Hg * Wg))


def test_scan_order_rejects_bad_args():
    with pytest.raises(RuntimeError):
        oracle.scan_order(12, 2, 2)      # codes 0..3 SREM, 4..11 zigzag
    with pytest.raises(RuntimeError):
        oracle.scan_order(-1, 2, 2)
    with pytest.raises(RuntimeError):
        oracle.scan_order(0, 0, 2)


# --------------------------------------------------------------------------- GLA pins
@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_gla_pin(pin):
    assert pin(oracle_gla, np.random.default_rng(1234))


@pytest.mark.parametrize("Hg,Wg", GRIDS)
@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_gla_matches_bruteforce_grids(Hg, Wg, direction):
    rng = np.random.default_rng(Hg * 100 + Wg * 10 + direction)
    q, k, v, la = rand_inputs(rng, 2, 2, Hg, Wg, 3, 5, gate_scale=0.8)
    np.testing.assert_allclose(oracle_gla(q, k, v, la, Hg, Wg, direction),
                               bruteforce(q, k, v, la, Hg, Wg, direction), rtol=1e-12, atol=1e-12)


def test_gla_single_token_and_first_step():
    """T = 1, and the first scanned token of any sequence: o = (q.k) v whatever the gate."""
    rng = np.random.default_rng(7)
    q, k, v, la = rand_inputs(rng, 1, 1, 1, 1, 4, 3, gate_scale=3.0)
    want = np.dot(q[0, 0, 0], k[0, 0, 0]) * v[0, 0, 0]
    np.testing.assert_allclose(oracle_gla(q, k, v, la, 1, 1, 0)[0, 0, 0], want, rtol=1e-14)
    q, k, v, la = rand_inputs(rng, 1, 1, 3, 4, 4, 3, gate_scale=3.0)
    for d in range(4):
        first = closed_form_order(d, 3, 4)[0]
        got = oracle_gla(q, k, v, la, 3, 4, d)[0, first, 0]
        np.testing.assert_allclose(got, np.dot(q[0, first, 0], k[0, first, 0]) * v[0, first, 0], rtol=1e-14)


def test_gla_scalar_two_steps_by_hand():
    """d = 1, T = 2 written out: o_0 = q0 k0 v0, o_1 = q1 (a1 k0 v0 + k1 v1)."""
    q = np.array([2.0, 3.0]).reshape(1, 2, 1, 1)
    k = np.array([5.0, 7.0]).reshape(1, 2, 1, 1)
    v = np.array([11.0, 13.0]).reshape(1, 2, 1, 1)
    a1 = 0.25
    la = np.log(np.array([0.5, a1])).reshape(1, 2, 1, 1)
    got = oracle_gla(q, k, v, la, 1, 2, 0).ravel()
    assert got[0] == pytest.approx(2 * 5 * 11, rel=1e-15)
    assert got[1] == pytest.approx(3 * (a1 * 5 * 11 + 7 * 13), rel=1e-15)
    # right-to-left: token 1 is scanned first
    got = oracle_gla(q, k, v, la, 1, 2, 1).ravel()
    assert got[1] == pytest.approx(3 * 7 * 13, rel=1e-15)
    assert got[0] == pytest.approx(2 * (0.5 * 7 * 13 + 5 * 11), rel=1e-15)


def test_gla_linearity():
    rng = np.random.default_rng(11)
    Hg, Wg = 4, 4
    q, k, v, la = rand_inputs(rng, 1, 2, Hg, Wg, 5, 4, gate_scale=0.4)
    v2 = rng.standard_normal(v.shape)
    q2 = rng.standard_normal(q.shape)
    for d in range(4):
        f = lambda qq, vv: oracle_gla(qq, k, vv, la, Hg, Wg, d)
        np.testing.assert_allclose(f(q, 2.5 * v + v2), 2.5 * f(q, v) + f(q, v2), rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(f(-1.5 * q + q2, v), -1.5 * f(q, v) + f(q2, v), rtol=1e-11, atol=1e-11)


def test_gla_heads_subset_matches_full():
    rng = np.random.default_rng(3)
    q, k, v, la = rand_inputs(rng, 2, 3, 3, 4, 4, 4, gate_scale=0.5)
    full = oracle.gla_fwd(q, k, v, la, 3, 4, 2, nthreads=4)
    part = oracle.gla_fwd(q, k, v, la, 3, 4, 2, nthreads=2, heads=(1, 4))
    flat_full = full.transpose(0, 2, 1, 3).reshape(6, 12, 4)
    flat_part = part.transpose(0, 2, 1, 3).reshape(6, 12, 4)
    np.testing.assert_array_equal(flat_part[1:4], flat_full[1:4])
    assert not flat_part[0].any() and not flat_part[4:].any()


def test_gla_threads_do_not_change_results():
    rng = np.random.default_rng(5)
    q, k, v, la = rand_inputs(rng, 2, 4, 4, 4, 8, 8)
    a = oracle.gla_fwd(q, k, v, la, 4, 4, 3, nthreads=1)
    b = oracle.gla_fwd(q, k, v, la, 4, 4, 3, nthreads=8)
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("planted", range(1, 8))
def test_planted_mistake_fails_a_pin(planted):
    """Each planted mistake (read before update, gate on the value axis, decay after
    the write, gate dropped, grid sides swapped, sign of the log-gate, k read in
    place of q) must be caught by at least one pin."""
    bad = lambda q, k, v, la, Hg, Wg, d: oracle_gla(q, k, v, la, Hg, Wg, d, planted=planted)
    results = [pin(bad, np.random.default_rng(1234)) for pin in ALL_PINS]
    assert not all(results), f"planted mistake {planted} passed every pin"


# --------------------------------------------------------------------------- conv pins
def _conv_inputs(rng, B=2, Hg=5, Wg=7, C=6):
    return rng.standard_normal((B, Hg, Wg, C))


def test_conv_identity_kernel_is_exact_copy():
    """SREM's identity initialisation (centre 1, rest 0) makes the conv the identity."""
    rng = np.random.default_rng(0)
    x = _conv_inputs(rng)
    w = np.zeros((x.shape[3], 3, 3))
    w[:, 1, 1] = 1.0
    np.testing.assert_array_equal(oracle.dwconv3x3(x, w), x)


@pytest.mark.parametrize("di,dj", [(-1, -1), (-1, 0), (0, 1), (1, 1), (1, -1)])
def test_conv_delta_kernel_shifts_with_zero_fill(di, dj):
    rng = np.random.default_rng(1)
    x = _conv_inputs(rng)
    B, Hg, Wg, C = x.shape
    w = np.zeros((C, 3, 3))
    w[:, di + 1, dj + 1] = 1.0
    want = np.zeros_like(x)
    for y in range(Hg):
        for xx in range(Wg):
            ys, xs = y + di, xx + dj
            if 0 <= ys < Hg and 0 <= xs < Wg:
                want[:, y, xx] = x[:, ys, xs]
    np.testing.assert_array_equal(oracle.dwconv3x3(x, w), want)


def test_conv_matches_torch_grouped_conv2d():
    rng = np.random.default_rng(2)
    x = _conv_inputs(rng, B=2, Hg=6, Wg=9, C=5)
    w = rng.standard_normal((5, 3, 3))
    xt = torch.from_numpy(x).permute(0, 3, 1, 2)          # NCHW
    ref = torch.nn.functional.conv2d(xt, torch.from_numpy(w)[:, None], padding=1, groups=5)
    np.testing.assert_allclose(oracle.dwconv3x3(x, w), ref.permute(0, 2, 3, 1).numpy(), rtol=1e-12, atol=1e-12)


def test_conv_is_not_flipped_cross_correlation():
    """A single tap at (row -1, col -1) reads the up-left neighbour (no kernel flip)."""
    x = np.zeros((1, 3, 3, 1))
    x[0, 0, 0, 0] = 1.0
    w = np.zeros((1, 3, 3))
    w[0, 0, 0] = 1.0
    y = oracle.dwconv3x3(x, w)
    assert y[0, 1, 1, 0] == 1.0 and y.sum() == 1.0


# --------------------------------------------------------------------------- reorient pins
@pytest.mark.parametrize("direction", [0, 1, 2, 3])
@pytest.mark.parametrize("Hg,Wg", [(3, 5), (4, 4), (6, 2)])
def test_reorient_gather_and_inverse(direction, Hg, Wg):
    rng = np.random.default_rng(direction)
    x = torch.randn(2, Hg * Wg, 10).to(torch.bfloat16).view(torch.int16).numpy()
    y = oracle.reorient(x, direction, 0, Hg, Wg)
    order = closed_form_order(direction, Hg, Wg)
    np.testing.assert_array_equal(y, x[:, order])
    np.testing.assert_array_equal(oracle.reorient(y, direction, 1, Hg, Wg), x)
    del rng


def test_reorient_byte_exact_for_nan_payloads():
    x = np.arange(2 * 12 * 4, dtype=np.uint32).reshape(2, 12, 4) | np.uint32(0x7FC00000)  # NaN bit patterns
    y = oracle.reorient(x.view(np.float32), 3, 0, 3, 4)
    np.testing.assert_array_equal(y.view(np.uint32), x[:, closed_form_order(3, 3, 4)])


# --------------------------------------------------------------------------- golden regression
def test_golden_fixture_regression():
    """Stored outputs written by tests/golden/make_golden.py (which calls only the
    oracle) must not drift."""
    path = os.path.join(GOLDEN, "oracle_small.json")
    with open(path) as f:
        g = json.load(f)
    for case in g["gla"]:
        inp = {n: np.array(case[n]) for n in ("q", "k", "v", "log_alpha")}
        out = oracle.gla_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], case["Hgrid"], case["Wgrid"],
                             case["dir"], nthreads=1)
        np.testing.assert_allclose(out, np.array(case["out"]), rtol=1e-13, atol=1e-15)
    for case in g["conv"]:
        out = oracle.dwconv3x3(np.array(case["x"]), np.array(case["w"]))
        np.testing.assert_allclose(out, np.array(case["y"]), rtol=1e-13, atol=1e-15)
