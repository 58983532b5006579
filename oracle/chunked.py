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
