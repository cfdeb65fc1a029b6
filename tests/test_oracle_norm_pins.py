"""Pins for the oracle's normalised variant (oracle.gla_norm_fwd): the diffusers
draft's gated linear attention (page 4, `gated_linear_attention`) with elu+1
features, the forget gate sigmoid(q * k), a gated denominator and an eps clamp.

Expected values come from elsewhere than the oracle's loop:
  * T = 1: the output is v itself (numerator (phi(q).phi(k)) v over denominator
    phi(q).phi(k));
  * the O(T^2) unrolled sums of numerator and denominator, with the features, the
    gate and the products of gates written out in numpy;
  * the un-normalised GLA oracle (pinned in test_oracle_pins.py) run twice, on v and
    on a column of ones, with q, k replaced by their features and log_alpha by
    log sigmoid(q * k);
  * every output is a convex combination of the values seen so far, so a constant v
    comes back unchanged and every output lies within the running range of v;
  * the clamp: features of very negative q are tiny, the denominator falls below
    eps and the output is the numerator divided by eps;
  * five planted mistakes each fail at least one pin.
"""
import numpy as np
import pytest

import oracle

from test_oracle_pins import closed_form_order

EPS = 1e-6


def feat(x):
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def sig(x):
    return 1.0 / (1.0 + np.exp(-x))


def norm(q, k, v, Hg, Wg, d, eps=EPS, planted=0):
    return oracle.gla_norm_fwd(q, k, v, Hg, Wg, d, eps=eps, nthreads=1, planted=planted)


def bruteforce_norm(q, k, v, Hg, Wg, d, eps=EPS):
    B, T, H, dk = q.shape
    order = closed_form_order(d, Hg, Wg)
    out = np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            Q, K, V = q[b, order, h], k[b, order, h], v[b, order, h]
            fQ, fK, G = feat(Q), feat(K), sig(Q * K)
            for t in range(T):
                num = np.zeros(V.shape[1])
                den = 0.0
                for s in range(t + 1):
                    decay = np.prod(G[s + 1:t + 1], axis=0) if t > s else np.ones(dk)
                    w = np.sum(fQ[t] * fK[s] * decay)
                    num += w * V[s]
                    den += w
                out[b, order[t], h] = num / max(den, eps)
    return out


def _inputs(rng, B, H, Hg, Wg, dk, dv, scale=1.0):
    T = Hg * Wg
    return (rng.standard_normal((B, T, H, dk)) * scale, rng.standard_normal((B, T, H, dk)) * scale,
            rng.standard_normal((B, T, H, dv)))


# --------------------------------------------------------------------------- pins as functions
def pin_single_token_returns_v(g, rng):
    q, k, v = _inputs(rng, 2, 3, 1, 1, 5, 4)
    np.testing.assert_allclose(g(q, k, v, 1, 1, 0), v, rtol=1e-13, atol=1e-14)


def pin_bruteforce(g, rng):
    for Hg, Wg in [(3, 4), (2, 5)]:
        for d in (0, 1, 2, 3, 5):
            q, k, v = _inputs(rng, 1, 2, Hg, Wg, 3, 4)
            np.testing.assert_allclose(g(q, k, v, Hg, Wg, d), bruteforce_norm(q, k, v, Hg, Wg, d), rtol=1e-11,
                                       atol=1e-12)


def pin_reduces_to_unnormalised_gla(g, rng):
    Hg, Wg = 4, 5
    q, k, v = _inputs(rng, 2, 2, Hg, Wg, 6, 4)
    la = np.log(sig(q * k))
    for d in (0, 3, 9):
        num = oracle.gla_fwd(feat(q), feat(k), v, la, Hg, Wg, d, nthreads=1)
        den = oracle.gla_fwd(feat(q), feat(k), np.ones(v.shape[:3] + (1,)), la, Hg, Wg, d, nthreads=1)
        np.testing.assert_allclose(g(q, k, v, Hg, Wg, d), num / np.maximum(den, EPS), rtol=1e-11, atol=1e-12)


def pin_convex_combination(g, rng):
    Hg, Wg = 3, 6
    q, k, v = _inputs(rng, 1, 2, Hg, Wg, 4, 3)
    const = np.broadcast_to(rng.standard_normal((1, 1, 2, 3)), v.shape).copy()
    np.testing.assert_allclose(g(q, k, const, Hg, Wg, 2), const, rtol=1e-12, atol=1e-13)
    out = g(q, k, v, Hg, Wg, 1)
    order = closed_form_order(1, Hg, Wg)
    for h in range(2):
        V, O = v[0, order, h], out[0, order, h]
        lo, hi = np.minimum.accumulate(V, axis=0), np.maximum.accumulate(V, axis=0)
        assert np.all(O >= lo - 1e-12) and np.all(O <= hi + 1e-12)


def pin_eps_clamp(g, rng):
    Hg, Wg = 2, 3
    q, k, v = _inputs(rng, 1, 1, Hg, Wg, 3, 2)
    q = -40.0 - np.abs(q)                      # phi(q) = e^q ~ 1e-18: the denominator < eps
    got = g(q, k, v, Hg, Wg, 0, eps=1e-3)
    np.testing.assert_allclose(got, bruteforce_norm(q, k, v, Hg, Wg, 0, eps=1e-3), rtol=1e-11, atol=1e-30)
    assert np.max(np.abs(got)) < 1e-12        # numerator / eps, not numerator / denominator


ALL_PINS = [pin_single_token_returns_v, pin_bruteforce, pin_reduces_to_unnormalised_gla, pin_convex_combination,
            pin_eps_clamp]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_norm_pin(pin):
    pin(norm, np.random.default_rng(21))


@pytest.mark.parametrize("planted", range(1, 6))
def test_planted_norm_mistake_fails_a_pin(planted):
    def wrong(q, k, v, Hg, Wg, d, eps=EPS):
        return norm(q, k, v, Hg, Wg, d, eps=eps, planted=planted)

    failed = []
    for pin in ALL_PINS:
        try:
            pin(wrong, np.random.default_rng(21))
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"planted mistake {planted} passed every pin"


def test_norm_threads_do_not_change_results():
    rng = np.random.default_rng(4)
    q, k, v = _inputs(rng, 2, 3, 4, 4, 5, 5)
    assert np.array_equal(oracle.gla_norm_fwd(q, k, v, 4, 4, 2, nthreads=1),
                          oracle.gla_norm_fwd(q, k, v, 4, 4, 2, nthreads=4))
