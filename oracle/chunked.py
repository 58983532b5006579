"""Exact chunkwise (UT/WY) form of the gated delta rule in fp64 numpy.

TEST INFRASTRUCTURE ONLY (see the package docstring).

This is the algebra the CUDA kernels implement, written plainly so it can be
read against its derivation; it is pinned against the token recurrence
(``oracle.recurrent``) as the SinkProbe (Attention-Sink) README describes for
its delta-rule layer: the exact chunkwise form must agree with the 64-bit
token-by-token recurrence at chunk sizes 1, 8, 16 and 64 within 1e-10, for the
outputs and for the memory (the state).

Derivation (state S is Dk x Dv, decay before the delta update, readout after it;
NextTransformer "Source notes", section "Linear attention", rows gdn and kda).
Inside one chunk of n tokens r = 0..n-1 entered with state S0, let
G_r = sum_{j<=r} g_j (per key channel; a scalar gate is broadcast) and
Gamma_r = exp(G_r). Writing u_r = beta_r (v_r - (D_r S_{r-1})^T k_r), the
recurrence is S_r = D_r S_{r-1} + k_r u_r^T, which unrolls to

    S_r = diag(Gamma_r) S0 + sum_{i<=r} diag(Gamma_r / Gamma_i) k_i u_i^T .

Substituting into u_r gives (I + A) U_true = diag(beta) V - diag(beta) (K*Gamma) S0
with the strictly lower-triangular

    A = tril(diag(beta) (K*Gamma) (K/Gamma)^T, -1),

so with T = (I + A)^-1, W = T diag(beta) (K*Gamma), U = T diag(beta) V:

    U_true = U - W S0
    O      = (Q*Gamma) S0 + tril((Q*Gamma) (K/Gamma)^T, 0) U_true
    S_n    = diag(Gamma_n) S0 + (K * (Gamma_n / Gamma))^T U_true .

A library triangular solve serves as the step "T = (I + A)^-1".
"""
import numpy as np
from scipy.linalg import solve_triangular


def _chunk(Kc, Qc, Vc, gc, bc, S):
    n, Dk = Kc.shape
    if gc.ndim == 1:
        gc = np.repeat(gc[:, None], Dk, axis=1)
    G = np.cumsum(gc, axis=0)                       # n x Dk
    Gam = np.exp(G)
    KG, KiG, QG = Kc * Gam, Kc / Gam, Qc * Gam
    A = np.tril(bc[:, None] * (KG @ KiG.T), -1)
    IA = np.eye(n) + A
    W = solve_triangular(IA, bc[:, None] * KG, lower=True, unit_diagonal=True)
    U = solve_triangular(IA, bc[:, None] * Vc, lower=True, unit_diagonal=True)
    Ut = U - W @ S
    O = QG @ S + np.tril(QG @ KiG.T, 0) @ Ut
    S_next = Gam[-1][:, None] * S + (Kc * (Gam[-1][None, :] / Gam)).T @ Ut
    return O, S_next


def chunked(q, k, v, g, beta, h0=None, chunk=64):
    """fp64 chunkwise forward. Same argument layouts as ``oracle.recurrent``.

    The last chunk of a sequence may be partial (T not a multiple of ``chunk``).
    Returns (o [B,T,Hv,Dv], hT [B,Hv,Dk,Dv]).
    """
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    B, T, Hk, Dk = q.shape
    Hv, Dv = v.shape[2], v.shape[3]
    grp = Hv // Hk
    o = np.zeros((B, T, Hv, Dv))
    hT = np.zeros((B, Hv, Dk, Dv))
    for b in range(B):
        for h in range(Hv):
            hk = h // grp
            S = np.zeros((Dk, Dv)) if h0 is None else np.array(h0[b, h], dtype=np.float64)
            for s in range(0, T, chunk):
                e = min(T, s + chunk)
                O, S = _chunk(k[b, s:e, hk], q[b, s:e, hk], v[b, s:e, h], g[b, s:e, h],
                              beta[b, s:e, h], S)
                o[b, s:e, h] = O
            hT[b, h] = S
    return o, hT


# ----------------------------------------------------------------------------- backward
#
# Adjoint of the chunk map above, the blueprint of a chunked backward. For upstream
# gradients dO (of the chunk's outputs) and dS_n (of the state leaving it), with
# B = (K*Gamma) (K/Gamma)^T and M = tril((Q*Gamma) (K/Gamma)^T, 0), reverse-mode
# differentiation of each line gives, in order:
#
#   dU_true = M^T dO + Kt dS_n                       Kt = K * (Gamma_n / Gamma)
#   dM      = tril(dO U_true^T, 0)
#   d(Q*Gamma) = dO S0^T + dM (K/Gamma),   d(K/Gamma) = dM^T (Q*Gamma)
#   dS0     = (Q*Gamma)^T dO + diag(Gamma_n) dS_n - W^T dU_true
#   dKt     = U_true dS_n^T,   dGamma_n = rowsum(dS_n * S0)
#   dW      = -dU_true S0^T,   dU = dU_true
#   with U = T Y_U, W = T Y_W (Y_U = diag(beta) V, Y_W = diag(beta) (K*Gamma)):
#   dY_U = T^T dU,  dY_W = T^T dW,  dT = dU Y_U^T + dW Y_W^T
#   dV = diag(beta) dY_U,  dbeta = rowsum(V * dY_U) + rowsum((K*Gamma) * dY_W)
#   d(K*Gamma) = diag(beta) dY_W
#   T = (I + A)^-1:  dA = tril(-T^T dT T^T, -1)
#   A = tril(diag(beta) B, -1):  dbeta += rowsum(dA * B),  dB = diag(beta) dA
#   d(K*Gamma) += dB (K/Gamma),  d(K/Gamma) += dB^T (K*Gamma)
#
# and, through Gamma = exp(G) (so that d/dG of X*Gamma is X*Gamma and of X/Gamma is
# -X/Gamma), the gradients of K, Q and the cumulative gate G:
#
#   dK = d(K*Gamma) Gamma + d(K/Gamma) / Gamma + dKt Gamma_n / Gamma,   dQ = d(Q*Gamma) Gamma
#   dG = d(K*Gamma) (K*Gamma) - d(K/Gamma) (K/Gamma) + d(Q*Gamma) (Q*Gamma) - dKt Kt
#   dG_{n-1} += colsum(dKt Kt) + dGamma_n Gamma_n
#   dg_j = sum_{r >= j} dG_r   (a scalar gate sums over the key channels).
#
# dS0 is the upstream state gradient of the previous chunk; after the first chunk it is dh0.


def _chunk_bwd(Kc, Qc, Vc, gc, bc, S, dO, dSn):
    n, Dk = Kc.shape
    scalar = gc.ndim == 1
    if scalar:
        gc = np.repeat(gc[:, None], Dk, axis=1)
    G = np.cumsum(gc, axis=0)
    Gam = np.exp(G)
    GamN = Gam[-1]
    KG, KiG, QG = Kc * Gam, Kc / Gam, Qc * Gam
    Kt = Kc * (GamN[None, :] / Gam)
    Bm = KG @ KiG.T
    IA = np.eye(n) + np.tril(bc[:, None] * Bm, -1)
    T = solve_triangular(IA, np.eye(n), lower=True, unit_diagonal=True)
    YU, YW = bc[:, None] * Vc, bc[:, None] * KG
    U, W = T @ YU, T @ YW
    Ut = U - W @ S
    M = np.tril(QG @ KiG.T, 0)

    dUt = M.T @ dO + Kt @ dSn
    dM = np.tril(dO @ Ut.T, 0)
    dQG = dO @ S.T + dM @ KiG
    dKiG = dM.T @ QG
    dS0 = QG.T @ dO + GamN[:, None] * dSn - W.T @ dUt
    dKt = Ut @ dSn.T
    dGamN = np.sum(dSn * S, axis=1)
    dU, dW = dUt, -dUt @ S.T
    dYU, dYW = T.T @ dU, T.T @ dW
    dT = dU @ YU.T + dW @ YW.T
    dV = bc[:, None] * dYU
    dbeta = np.sum(Vc * dYU, axis=1) + np.sum(KG * dYW, axis=1)
    dKG = bc[:, None] * dYW
    dA = np.tril(-T.T @ dT @ T.T, -1)
    dbeta += np.sum(dA * Bm, axis=1)
    dB = bc[:, None] * dA
    dKG += dB @ KiG
    dKiG += dB.T @ KG

    dK = dKG * Gam + dKiG / Gam + dKt * (GamN[None, :] / Gam)
    dQ = dQG * Gam
    dG = dKG * KG - dKiG * KiG + dQG * QG - dKt * Kt
    dG[-1] += np.sum(dKt * Kt, axis=0) + dGamN * GamN
    dg = np.cumsum(dG[::-1], axis=0)[::-1]
    if scalar:
        dg = dg.sum(axis=1)
    return dQ, dK, dV, dg, dbeta, dS0


def chunked_backward(q, k, v, g, beta, h0, do, dhT=None, chunk=64):
    """fp64 chunkwise backward: the gradients of L = sum(do * o) + sum(dhT * hT), by a
    forward pass that keeps each chunk's entering state, then the adjoint above chunk by
    chunk in reverse. Same layouts and result as ``oracle.backward``."""
    q, k, v, g, beta, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta, do))
    B, T, Hk, Dk = q.shape
    Hv, Dv = v.shape[2], v.shape[3]
    grp = Hv // Hk
    out = {"dq": np.zeros(q.shape), "dk": np.zeros(k.shape), "dv": np.zeros(v.shape),
           "dg": np.zeros(g.shape), "dbeta": np.zeros(beta.shape), "dh0": np.zeros((B, Hv, Dk, Dv))}
    for b in range(B):
        for h in range(Hv):
            hk = h // grp
            S = np.zeros((Dk, Dv)) if h0 is None else np.array(h0[b, h], dtype=np.float64)
            bounds = [(s, min(T, s + chunk)) for s in range(0, T, chunk)]
            entering = []
            for s, e in bounds:
                entering.append(S)
                _, S = _chunk(k[b, s:e, hk], q[b, s:e, hk], v[b, s:e, h], g[b, s:e, h], beta[b, s:e, h], S)
            dS = np.zeros((Dk, Dv)) if dhT is None else np.array(dhT[b, h], dtype=np.float64)
            for (s, e), S0 in zip(reversed(bounds), reversed(entering)):
                dQ, dK, dV, dg, db, dS = _chunk_bwd(k[b, s:e, hk], q[b, s:e, hk], v[b, s:e, h], g[b, s:e, h],
                                                   beta[b, s:e, h], S0, do[b, s:e, h], dS)
                out["dq"][b, s:e, hk] += dQ
                out["dk"][b, s:e, hk] += dK
                out["dv"][b, s:e, h] = dV
                out["dg"][b, s:e, h] = dg
                out["dbeta"][b, s:e, h] = db
            out["dh0"][b, h] = dS
    return out
