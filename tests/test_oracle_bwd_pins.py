"""Pins for the fp64 oracle's GLA backward (oracle.gla_bwd) -- checked against
mathematics, not against itself.

The backward is the exact gradient of the forward recurrence (pinned in
test_oracle_pins.py), so every expected value below comes from somewhere else:
  * central finite differences of the forward oracle, loss = sum(dout * out);
  * torch autograd through the O(T^2) unrolled sum
        o_t = sum_{s<=t} (q_t * prod_{r=s+1..t} alpha_r) . k_s  v_s
    written with plain tensor ops on tiny grids, all four scan orders;
  * with log_alpha = 0 the forward is masked causal linear attention
    O = (Q K^T * M) V, whose gradients are the textbook products
    dQ = (dO V^T * M) K, dK = (dO V^T * M)^T Q, dV = (Q K^T * M)^T dO;
  * log_alpha enters only through the prefix sums b_t = sum_{r<=t} log_alpha_r,
    and o_t depends on b through q_t e^{b_t} and k_s e^{-b_s}; hence
        dlog_alpha_r = sum_{t >= r} (q_t * dq_t - k_t * dk_t)   (scan order),
    an identity the recurrence's reverse sweep never uses;
  * a full reset (log_alpha = -inf on every channel) splits the sequence into two
    independent ones, whose backward passes can be run separately;
  * planted mistakes in the backward sweep must each fail at least one pin.
"""
import numpy as np
import pytest
import torch

import oracle

from test_oracle_pins import closed_form_order, rand_inputs


def bwd(q, k, v, la, do, Hg, Wg, d, planted=0):
    return oracle.gla_bwd(q, k, v, la, do, Hg, Wg, d, nthreads=1, planted=planted)


def _inputs(rng, B, H, Hg, Wg, dk, dv, gate_scale=0.5):
    q, k, v, la = rand_inputs(rng, B, H, Hg, Wg, dk, dv, gate_scale)
    do = rng.standard_normal(v.shape)
    return q, k, v, la, do


# --------------------------------------------------------------------------- pins as functions
def pin_finite_differences(g, rng):
    """Central differences of loss = sum(dout * gla_fwd(...)) on every input element."""
    B, H, Hg, Wg, dk, dv = 1, 2, 2, 3, 3, 2
    h = 1e-5
    for d in range(4):
        q, k, v, la, do = _inputs(rng, B, H, Hg, Wg, dk, dv)
        grads = g(q, k, v, la, do, Hg, Wg, d)

        def loss(q_, k_, v_, la_):
            return float(np.sum(do * oracle.gla_fwd(q_, k_, v_, la_, Hg, Wg, d, nthreads=1)))

        base = [q, k, v, la]
        for which in range(4):
            fd = np.zeros_like(base[which])
            for idx in np.ndindex(base[which].shape):
                plus = [a.copy() for a in base]
                minus = [a.copy() for a in base]
                plus[which][idx] += h
                minus[which][idx] -= h
                fd[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
            np.testing.assert_allclose(grads[which], fd, rtol=1e-6, atol=1e-7,
                                       err_msg=f"input {which}, direction {d}")


def _bruteforce_torch(q, k, v, la, Hg, Wg, direction):
    """The unrolled O(T^2) sum with torch ops (differentiable), scan order from the
    closed-form index formulas."""
    B, T, H, dk = q.shape
    order = closed_form_order(direction, Hg, Wg)
    out = torch.zeros(v.shape, dtype=torch.float64)
    for b in range(B):
        for hh in range(H):
            Q, K, V, L = (x[b, order, hh] for x in (q, k, v, la))
            csum = torch.cat([torch.zeros(1, dk, dtype=torch.float64), torch.cumsum(L, 0)])
            rows = []
            for p in range(T):
                acc = torch.zeros(V.shape[1], dtype=torch.float64)
                for s in range(p + 1):
                    decay = torch.exp(csum[p + 1] - csum[s + 1])
                    acc = acc + torch.dot(Q[p] * decay, K[s]) * V[s]
                rows.append(acc)
            res = torch.stack(rows)                     # scan order
            canon = torch.zeros_like(res)
            canon[torch.as_tensor(order)] = res
            out[b, :, hh] = canon
    return out


def pin_autograd_bruteforce(g, rng):
    for Hg, Wg in [(3, 4), (2, 5)]:
        for d in range(4):
            q, k, v, la, do = _inputs(rng, 1, 2, Hg, Wg, 3, 4)
            ts = [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v, la)]
            out = _bruteforce_torch(*ts, Hg, Wg, d)
            (out * torch.tensor(do)).sum().backward()
            grads = g(q, k, v, la, do, Hg, Wg, d)
            for which in range(4):
                np.testing.assert_allclose(grads[which], ts[which].grad.numpy(), rtol=1e-10, atol=1e-11,
                                           err_msg=f"input {which}, grid {Hg}x{Wg}, direction {d}")


def pin_ungated_textbook(g, rng):
    Hg, Wg = 3, 5
    for d in range(4):
        q, k, v, la, do = _inputs(rng, 2, 2, Hg, Wg, 4, 3)
        la = np.zeros_like(la)
        dq, dk, dv, _ = g(q, k, v, la, do, Hg, Wg, d)
        order = closed_form_order(d, Hg, Wg)
        T = Hg * Wg
        M = np.tril(np.ones((T, T)))                      # s <= t in scan order
        for b in range(2):
            for h in range(2):
                Q, K, V, dO = (x[b, order, h] for x in (q, k, v, do))
                A = (dO @ V.T) * M
                np.testing.assert_allclose(dq[b, order, h], A @ K, rtol=1e-12, atol=1e-12)
                np.testing.assert_allclose(dk[b, order, h], A.T @ Q, rtol=1e-12, atol=1e-12)
                np.testing.assert_allclose(dv[b, order, h], ((Q @ K.T) * M).T @ dO, rtol=1e-12, atol=1e-12)


def pin_prefix_identity(g, rng):
    """dlog_alpha_r = sum_{t >= r} (q_t * dq_t - k_t * dk_t) along the scan order."""
    Hg, Wg = 5, 6
    for d in range(4):
        q, k, v, la, do = _inputs(rng, 1, 2, Hg, Wg, 4, 5, gate_scale=0.3)
        dq, dk, _, dla = g(q, k, v, la, do, Hg, Wg, d)
        order = closed_form_order(d, Hg, Wg)
        for h in range(2):
            db = (q * dq - k * dk)[0, order, h]           # [T, dk] in scan order
            suffix = np.cumsum(db[::-1], axis=0)[::-1]
            np.testing.assert_allclose(dla[0, order, h], suffix, rtol=1e-9, atol=1e-10)


def pin_reset_splits_sequence(g, rng):
    """Left-to-right scan of a 4x3 grid with every channel reset at the first token of
    row 2: the backward equals the backward of rows 0-1 and rows 2-3 run alone."""
    Hg, Wg = 4, 3
    q, k, v, la, do = _inputs(rng, 1, 2, Hg, Wg, 3, 2)
    la[:, 2 * Wg] = -np.inf
    whole = g(q, k, v, la, do, Hg, Wg, 0)
    top = g(*(x[:, : 2 * Wg] for x in (q, k, v, la, do)), 2, Wg, 0)
    bottom = g(*(x[:, 2 * Wg:] for x in (q, k, v, la, do)), 2, Wg, 0)
    for which in range(4):
        np.testing.assert_allclose(whole[which][:, : 2 * Wg], top[which], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(whole[which][:, 2 * Wg:], bottom[which], rtol=1e-12, atol=1e-13)
    assert np.all(whole[3][:, 2 * Wg] == 0.0)              # alpha = 0: no gradient to its log


ALL_PINS = [pin_finite_differences, pin_autograd_bruteforce, pin_ungated_textbook, pin_prefix_identity,
            pin_reset_splits_sequence]


# --------------------------------------------------------------------------- tests
@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_gla_bwd_pin(pin):
    pin(bwd, np.random.default_rng(11))


@pytest.mark.parametrize("planted", range(1, 7))
def test_planted_backward_mistake_fails_a_pin(planted):
    def wrong(q, k, v, la, do, Hg, Wg, d):
        return bwd(q, k, v, la, do, Hg, Wg, d, planted=planted)

    failed = []
    for pin in ALL_PINS:
        try:
            pin(wrong, np.random.default_rng(11))
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"planted backward mistake {planted} passed every pin"


def test_gla_bwd_heads_subset_and_threads():
    rng = np.random.default_rng(3)
    q, k, v, la, do = _inputs(rng, 2, 3, 4, 5, 4, 3)
    full = oracle.gla_bwd(q, k, v, la, do, 4, 5, 2, nthreads=1)
    many = oracle.gla_bwd(q, k, v, la, do, 4, 5, 2, nthreads=4)
    part = oracle.gla_bwd(q, k, v, la, do, 4, 5, 2, nthreads=2, heads=(2, 5))
    for a, b_, c in zip(full, many, part):
        assert np.array_equal(a, b_)
        flat_a, flat_c = a.reshape(2, 20, 3, -1), c.reshape(2, 20, 3, -1)
        # flattened heads 2, 3, 4 = (b0, h2), (b1, h0), (b1, h1)
        assert np.array_equal(flat_a[0, :, 2], flat_c[0, :, 2])
        assert np.array_equal(flat_a[1, :, :2], flat_c[1, :, :2])
        assert not np.any(flat_c[0, :, :2]) and not np.any(flat_c[1, :, 2])


def test_gla_bwd_single_token_by_hand():
    """T = 1: out = (q.k) v, so dq = (dO.v) k, dk = (dO.v) q, dv = (q.k) dO, and the
    gate multiplies the zero initial state: dlog_alpha = 0."""
    q = np.array([[[[1.0, 2.0]]]])
    k = np.array([[[[3.0, -1.0]]]])
    v = np.array([[[[0.5, 2.0, -1.0]]]])
    la = np.array([[[[-0.3, -2.0]]]])
    do = np.array([[[[1.0, -1.0, 2.0]]]])
    dq, dk, dv, dla = oracle.gla_bwd(q, k, v, la, do, 1, 1, 0)
    dov = 0.5 - 2.0 - 2.0
    np.testing.assert_array_equal(dq, dov * k)
    np.testing.assert_array_equal(dk, dov * q)
    np.testing.assert_array_equal(dv, (3.0 - 2.0) * do)
    np.testing.assert_array_equal(dla, np.zeros_like(la))
