"""The dataflow of the chunked backward's kernels (csrc/bwd_chunk.cu), restated in fp64
matrix form, against the oracle's chunk adjoint (no GPU).

The kernels do not compute the adjoint in the oracle's order: the reverse scan applies the
transposed affine chunk map dS = Gamma_C dS_next + P^T dS_next + Qh^T dO, and the chunk
kernel forms every gradient from transposed feature-by-token products (W^T, U'^T, dU'^T,
dW^T, dV^T, dQ^T, dK^T), with the decays relative to each chunk (D_ri = exp(G_r - G_i),
f = Gamma_C / Gamma), the two dT terms as one product of the stacked [dU'; dW] with the
stacked [V; K], and post-scalings by f, Gamma and beta. This restatement of that sequence
must give the oracle's gradients to rounding, so a change to the kernels' algebra has a
written specification to be checked against.
"""
import importlib

import numpy as np
import pytest

oc = importlib.import_module("oracle.chunked")   # the module (the package exports a function of that name)


def kernel_dataflow(K, Q, V, g, b, S, dO, dSn):
    """One chunk, scalar gate: the products in the chunk kernel's order and orientation."""
    n = K.shape[0]
    G = np.cumsum(g)
    Gam = np.exp(G)
    GC = Gam[-1]
    f = GC / Gam
    Dm = np.exp(G[:, None] - G[None, :]) * (np.arange(n)[:, None] >= np.arange(n)[None, :])
    # T as the forward stores it
    A = np.tril(b[:, None] * (K @ K.T) * Dm, -1)
    T = np.linalg.inv(np.eye(n) + A)
    # the reverse scan's step (affine map of the forward, transposed)
    W = (T * (b * Gam)[None, :]) @ K
    Kt = f[:, None] * K
    M = np.tril((Q @ K.T) * Dm, 0)
    P = -Kt.T @ W
    Qh = Gam[:, None] * Q - M @ W
    dS0 = GC * dSn + P.T @ dSn + Qh.T @ dO
    # the chunk kernel: batch 1 ([K; Q] K^T, W^T, U^T, S dO^T, dS_next^T K^T)
    ST, dSnT = S.T, dSn.T
    KK = K @ K.T
    WT = K.T @ (T * (b * Gam)[None, :]).T
    UT = V.T @ (T * b[None, :]).T
    QAT = ST.T @ dO.T
    DUBT = dSnT @ K.T
    # batch 2: U'^T = U^T - S^T W^T, dO^T M
    UtT = UT - ST @ WT
    dUtT = dO.T @ M + DUBT * f[None, :]
    # batch 3: dM (token by token), dK3^T, dW^T, dV^T
    dMD = np.tril(dO @ UtT, 0) * Dm
    K3T = dSnT.T @ UtT
    dWT = -(ST.T @ dUtT)
    DVT = dUtT @ T
    dV = (DVT * b[None, :]).T
    dbeta = np.sum(V.T * DVT, axis=0)
    # batch 4: K^T (dM*D)^T, Q^T (dM*D), dW^T T and the stacked dT product
    QBT = K.T @ dMD.T
    K2T = Q.T @ dMD
    K1AT = dWT @ T
    stack = np.concatenate([dUtT.T, dWT.T], 0) @ np.concatenate([V, K], 0).T
    dT = b[None, :] * (stack[:n, :n] + Gam[None, :] * stack[n:, n:])
    # batches 5 and 6: X = T^T dT, Y = X T^T; dA and dB * D
    Y = (T.T @ dT) @ T.T
    dA = np.tril(-Y, -1)
    dbeta = dbeta + np.sum(dA * np.tril(KK * Dm, -1), axis=1)
    dBD = b[:, None] * dA * Dm
    # batch 7 and the epilogues
    K1BT = K.T @ dBD.T
    K2T = K2T + K.T @ dBD
    dQ = (Gam[None, :] * QAT + QBT).T
    k3 = f[None, :] * K3T
    k1 = (Gam * b)[None, :] * K1AT
    dK = (k3 + k1 + K1BT + K2T).T
    dbeta = dbeta + Gam * np.sum(K.T * K1AT, axis=0)
    dG = np.sum(K.T * (k1 + K1BT - K2T - k3), axis=0) + np.sum(dQ * Q, axis=1)
    dG[-1] += np.sum(k3 * K.T) + GC * np.sum(dSnT * ST)
    dg = np.cumsum(dG[::-1])[::-1]
    return dQ, dK, dV, dg, dbeta, dS0


@pytest.mark.parametrize("n", [64, 40, 1])
@pytest.mark.parametrize("seed", [0, 1])
def test_kernel_dataflow_equals_the_oracle_chunk_adjoint(n, seed):
    rng = np.random.default_rng(seed)
    Dk = Dv = 32
    K = rng.standard_normal((n, Dk))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    Q = rng.standard_normal((n, Dk))
    Q /= np.linalg.norm(Q, axis=1, keepdims=True)
    V = rng.standard_normal((n, Dv))
    g = -rng.uniform(0.01, 0.3, n)
    b = rng.uniform(0.1, 0.9, n)
    S = 0.3 * rng.standard_normal((Dk, Dv))
    dO = rng.standard_normal((n, Dv))
    dSn = 0.3 * rng.standard_normal((Dk, Dv))
    got = kernel_dataflow(K, Q, V, g, b, S, dO, dSn)
    ref = oc._chunk_bwd(K, Q, V, g, b, S, dO, dSn)
    for name, x, y in zip(("dq", "dk", "dv", "dg", "dbeta", "dS"), got, ref):
        assert np.max(np.abs(x - y)) <= 1e-12 * max(1.0, np.max(np.abs(y))), name
