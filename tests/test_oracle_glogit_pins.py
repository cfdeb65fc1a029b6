"""Pins for oracle.gla_fwd_glogit, the forward with the gate given as logits g:
log_alpha = logsigmoid(g) / gate_norm (the GLA configurations' gate, gate_norm 16).

  * it equals the pinned forward oracle run on log_alpha from torch's logsigmoid
    (a library routine) in fp64;
  * g -> +inf opens the gate (alpha = 1): masked causal linear attention tril(QK^T)V;
  * g -> -inf closes it (alpha = 0): out_t = (q_t . k_t) v_t;
  * large negative logits, where e^{-g} overflows, stay finite and exact.
"""
import numpy as np
import torch

import oracle

from test_oracle_pins import closed_form_order, rand_inputs


def test_glogit_equals_forward_on_library_logsigmoid():
    rng = np.random.default_rng(31)
    q, k, v, _ = rand_inputs(rng, 2, 2, 4, 5, 6, 3)
    g = rng.standard_normal(q.shape) * 3.0
    la = torch.nn.functional.logsigmoid(torch.from_numpy(g)).numpy() / 16.0
    for d in (0, 1, 2, 3, 6):
        np.testing.assert_allclose(oracle.gla_fwd_glogit(q, k, v, g, 4, 5, d, 16.0, nthreads=1),
                                   oracle.gla_fwd(q, k, v, la, 4, 5, d, nthreads=1), rtol=1e-13, atol=1e-14)
    la4 = torch.nn.functional.logsigmoid(torch.from_numpy(g)).numpy() / 4.0
    np.testing.assert_allclose(oracle.gla_fwd_glogit(q, k, v, g, 4, 5, 2, 4.0, nthreads=1),
                               oracle.gla_fwd(q, k, v, la4, 4, 5, 2, nthreads=1), rtol=1e-13, atol=1e-14)


def test_glogit_open_and_closed_gates():
    rng = np.random.default_rng(32)
    Hg, Wg = 3, 4
    q, k, v, _ = rand_inputs(rng, 1, 2, Hg, Wg, 4, 3)
    out = oracle.gla_fwd_glogit(q, k, v, np.full(q.shape, np.inf), Hg, Wg, 1, nthreads=1)
    order = closed_form_order(1, Hg, Wg)
    for h in range(2):
        Q, K, V = q[0, order, h], k[0, order, h], v[0, order, h]
        np.testing.assert_allclose(out[0, order, h], np.tril(Q @ K.T) @ V, rtol=1e-12, atol=1e-12)
    out = oracle.gla_fwd_glogit(q, k, v, np.full(q.shape, -np.inf), Hg, Wg, 3, nthreads=1)
    np.testing.assert_allclose(out, np.einsum("bthi,bthi->bth", q, k)[..., None] * v, rtol=1e-13, atol=1e-14)


def test_glogit_stable_for_large_negative_logits():
    rng = np.random.default_rng(33)
    q, k, v, _ = rand_inputs(rng, 1, 1, 2, 3, 3, 2)
    g = np.full(q.shape, -800.0)                       # e^{800} overflows fp64
    got = oracle.gla_fwd_glogit(q, k, v, g, 2, 3, 0, 16.0, nthreads=1)
    assert np.all(np.isfinite(got))
    np.testing.assert_allclose(got, oracle.gla_fwd(q, k, v, np.full(q.shape, -50.0), 2, 3, 0, nthreads=1),
                               rtol=1e-12, atol=1e-300)
