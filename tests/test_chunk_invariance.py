"""Chunk-size invariance of the chunk-wise decomposition, checked against the oracle.

The GLA kernels cut each scan into chunks of M positions (128 for the bf16 forward,
64 for the fp32 forward and the backward, 32 for wide heads) and rely on the chunk-wise
form reaching the recurrence's result exactly, whatever M is (the pages give no M; the
result must not depend on it).  This file writes that decomposition out in numpy,
fp64, for chunk sizes from 1 to 128 and ragged tails, and compares it with the
step-by-step oracle (oracle.gla_fwd, oracle.gla_bwd):

forward, per chunk (b = inclusive prefix of the log-gates in scan order, g = total):
    O = tril(Q e^{b} (K e^{-b})^T) V + (Q e^{b}) S_in,
    S_out = Diag(e^{g}) S_in + (K e^{g-b})^T V;
backward, per chunk (u = g - b the gates after each row, Q~ = Q e^{-u},
K^ = K e^{u}, G = Diag(e^{g}) S_in, A = tril(dO V^T), P = tril(Q~ K^T), D the
gradient of the state leaving the chunk):
    dQ = e^{-u} (dO G^T + A K^),  dK = e^{u} (A^T Q~ + V D^T),  dV = P^T dO + K^ D,
    D entering = Diag(e^{g}) D + (Q e^{b})^T dO,
    dlog_alpha_r = sum over the chunk's positions at or after r of (q dq - k dk)
                   + sum_j D[i][j] S_out[i][j]  (the gradient of a gate at the chunk's end).
"""
import numpy as np
import pytest

import oracle

from test_oracle_pins import closed_form_order, rand_inputs


def chunked_forward(Q, K, V, L, M):
    """One head in scan order: Q, K, L [T, dk]; V [T, dv] -> O [T, dv]."""
    T, dk = Q.shape
    S = np.zeros((dk, V.shape[1]))
    out = np.zeros((T, V.shape[1]))
    for c0 in range(0, T, M):
        q, k, v, la = Q[c0:c0 + M], K[c0:c0 + M], V[c0:c0 + M], L[c0:c0 + M]
        b = np.cumsum(la, axis=0)
        g = b[-1]
        Qt, Kt = q * np.exp(b), k * np.exp(-b)
        out[c0:c0 + M] = np.tril(Qt @ Kt.T) @ v + Qt @ S
        S = np.exp(g)[:, None] * S + (k * np.exp(g - b)).T @ v
    return out


def chunked_backward(Q, K, V, L, dO, M):
    """One head in scan order: returns dQ, dK, dV, dL by the chunk-wise formulas."""
    T, dk = Q.shape
    dv = V.shape[1]
    starts = list(range(0, T, M))
    # forward scan: S_in of every chunk
    S_in = []
    S = np.zeros((dk, dv))
    for c0 in starts:
        k, v, la = K[c0:c0 + M], V[c0:c0 + M], L[c0:c0 + M]
        b = np.cumsum(la, axis=0)
        g = b[-1]
        S_in.append(S)
        S = np.exp(g)[:, None] * S + (k * np.exp(g - b)).T @ v
    S_out = S_in[1:] + [S]
    # reverse scan: D leaving every chunk
    D_out = [None] * len(starts)
    D = np.zeros((dk, dv))
    for ci in range(len(starts) - 1, -1, -1):
        c0 = starts[ci]
        q, la, do = Q[c0:c0 + M], L[c0:c0 + M], dO[c0:c0 + M]
        b = np.cumsum(la, axis=0)
        g = b[-1]
        D_out[ci] = D
        D = np.exp(g)[:, None] * D + (q * np.exp(b)).T @ do
    dQ, dK, dV, dL = (np.zeros_like(x) for x in (Q, K, V, L))
    for ci, c0 in enumerate(starts):
        q, k, v, la, do = Q[c0:c0 + M], K[c0:c0 + M], V[c0:c0 + M], L[c0:c0 + M], dO[c0:c0 + M]
        b = np.cumsum(la, axis=0)
        g = b[-1]
        u = g - b                                   # sum of the gates after each row
        Qt, Kh = q * np.exp(-u), k * np.exp(u)
        G = np.exp(g)[:, None] * S_in[ci]
        A = np.tril(do @ v.T)
        P = np.tril(Qt @ Kh.T)
        Dc = D_out[ci]
        dQt = do @ G.T + A @ Kh
        dKh = A.T @ Qt + v @ Dc.T
        dQ[c0:c0 + M] = np.exp(-u) * dQt
        dK[c0:c0 + M] = np.exp(u) * dKh
        dV[c0:c0 + M] = P.T @ do + Kh @ Dc
        db = Qt * dQt - Kh * dKh
        carry = np.sum(Dc * S_out[ci], axis=1)
        dL[c0:c0 + M] = np.cumsum(db[::-1], axis=0)[::-1] + carry
    return dQ, dK, dV, dL


@pytest.mark.parametrize("M", [1, 2, 7, 16, 32, 64, 128])
def test_forward_chunk_size_invariance(M):
    rng = np.random.default_rng(50 + M)
    Hg, Wg = 9, 23                                  # T = 207: ragged tails for every M > 1
    q, k, v, la = rand_inputs(rng, 1, 2, Hg, Wg, 5, 4, gate_scale=0.05)
    for d in (0, 3, 7):
        ref = oracle.gla_fwd(q, k, v, la, Hg, Wg, d, nthreads=1)
        order = closed_form_order(d, Hg, Wg)
        for h in range(2):
            got = chunked_forward(q[0, order, h], k[0, order, h], v[0, order, h], la[0, order, h], M)
            np.testing.assert_allclose(got, ref[0, order, h], rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("M", [1, 8, 32, 64])
def test_backward_chunk_size_invariance(M):
    rng = np.random.default_rng(70 + M)
    Hg, Wg = 7, 11                                  # T = 77
    q, k, v, la = rand_inputs(rng, 1, 2, Hg, Wg, 4, 3, gate_scale=0.05)
    do = rng.standard_normal(v.shape)
    for d in (1, 2):
        refs = oracle.gla_bwd(q, k, v, la, do, Hg, Wg, d, nthreads=1)
        order = closed_form_order(d, Hg, Wg)
        for h in range(2):
            got = chunked_backward(q[0, order, h], k[0, order, h], v[0, order, h], la[0, order, h],
                                   do[0, order, h], M)
            for g, r in zip(got, refs):
                np.testing.assert_allclose(g, r[0, order, h], rtol=1e-9, atol=1e-10)
