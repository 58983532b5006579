"""The dataflow of the tcgen05 chunked forward (csrc/chunk_tc.cu), restated in fp64 matrix
form, against the oracle's token recurrence (no GPU).

The kernel does not run the pages' chunk scan (U' = U - W S, then the output and the state
update) but its affine form: per chunk, S_next = Gamma_C S + P S + R and O = Qh S + Uh, with
P, R, Qh and Uh formed from the chunk's inputs alone, one chunk ahead. It inverts I + A by
blocks of 16: each diagonal block in the product form (I + N)^-1 = (I - N)(I + N^2)(I + N^4)
(I + N^8), each off-diagonal block as the sums of chains D A D A ... D that its warps
evaluate. The scalar gate's decays exp(G_r - G_i) are factored through the first row of r's
16-row block; the per-channel gate's ride on operands relative to the chunk's row 31. This
restatement must reproduce the token recurrence, over several chunks with a ragged last
one, so a change to the kernel's algebra has a written specification to be checked against.
"""
import numpy as np
import pytest

import oracle

C = 64


def inverse_as_kernel(A):
    """(I + A)^-1 for A strictly lower 64 x 64, by the kernel's 16 x 16 blocks."""
    I16 = np.eye(16)
    blk = lambda i, j: A[16 * i:16 * i + 16, 16 * j:16 * j + 16]
    D = []
    for b in range(4):
        N = blk(b, b)
        N2 = N @ N
        N4 = N2 @ N2
        N8 = N4 @ N4
        D.append((I16 - N) @ (I16 + N2) @ (I16 + N4) @ (I16 + N8))
    T = np.zeros((C, C))
    put = lambda i, j, x: T.__setitem__((slice(16 * i, 16 * i + 16), slice(16 * j, 16 * j + 16)), x)
    for b in range(4):
        put(b, b, D[b])
    put(1, 0, -D[1] @ blk(1, 0) @ D[0])
    put(2, 1, -D[2] @ blk(2, 1) @ D[1])
    put(3, 2, -D[3] @ blk(3, 2) @ D[2])
    put(2, 0, (D[2] @ blk(2, 1) @ D[1] @ blk(1, 0) - D[2] @ blk(2, 0)) @ D[0])
    put(3, 1, (D[3] @ blk(3, 2) @ D[2] @ blk(2, 1) - D[3] @ blk(3, 1)) @ D[1])
    Qc = D[3] @ blk(3, 2) @ D[2]
    put(3, 0, ((D[3] @ blk(3, 1) - Qc @ blk(2, 1)) @ D[1] @ blk(1, 0) + Qc @ blk(2, 0) - D[3] @ blk(3, 0)) @ D[0])
    return T


def chunk_maps_scalar(K, Q, V, g, b):
    """P, R, Qh, Uh and Gamma_C of one zero-padded chunk, scalar gate."""
    G = np.cumsum(g)
    Gam = np.exp(G)
    r = np.arange(C)
    base = 16 * (r // 16)
    erow = np.exp(G - G[base])                                   # exp(G_r - G_16R)
    ecol = np.exp(G[base][:, None] - G[None, :])                 # exp(G_16R - G_i)
    E = erow[:, None] * ecol                                      # = exp(G_r - G_i) for i <= r
    A = np.tril(b[:, None] * E * (K @ K.T), -1)
    M = np.tril(E * (Q @ K.T), 0)
    T = inverse_as_kernel(A)
    WT = K.T @ (T * (b * Gam)[None, :]).T                         # W^T = K^T T'^T
    UT = V.T @ (T * b[None, :]).T                                 # U^T = V^T T''^T
    Kt = (Gam[-1] / Gam)[:, None] * K
    R = (UT @ Kt).T
    Qh = (Q.T * Gam[None, :] - WT @ M.T).T
    Uh = (UT @ M.T).T
    P = -Kt.T @ WT.T
    return P, R, Qh, Uh, Gam[-1]


def chunk_step_channel(K, Q, V, g, b, S):
    """One zero-padded chunk, per-channel gate, relative to row 31: (O, S_next)."""
    G = np.cumsum(g, axis=0)                                      # [C, Dk]
    G31 = G[31]
    Ks, Qs, Kb = K * np.exp(G - G31), Q * np.exp(G - G31), K * np.exp(G31 - G)
    A = np.tril(b[:, None] * (Ks @ Kb.T), -1)
    M = np.tril(Qs @ Kb.T, 0)
    T2 = inverse_as_kernel(A) * b[None, :]                        # T'' = T diag(beta)
    Wp, U = T2 @ Ks, T2 @ V
    Kt = Kb * np.exp(G[-1] - G31)
    Pp, Xp, R, Uh = -Kt.T @ Wp, Qs.T - Wp.T @ M.T, Kt.T @ U, M @ U
    St = np.exp(G31)[:, None] * S                                 # S~ = diag(exp G_31) S
    return Xp.T @ St + Uh, np.exp(G[-1])[:, None] * S + Pp @ St + R


def run_chunks(q, k, v, g, beta, h0, channel):
    T, Dk = q.shape
    S = h0.copy()
    o = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        n = min(C, T - c0)
        pad = lambda x: np.concatenate([x[c0:c0 + n], np.zeros((C - n,) + x.shape[1:])], 0)
        K, Q, V, gc, bc = pad(k), pad(q), pad(v), pad(g), pad(beta)
        if channel:
            O, S = chunk_step_channel(K, Q, V, gc, bc, S)
        else:
            P, R, Qh, Uh, GC = chunk_maps_scalar(K, Q, V, gc, bc)
            O, S = Qh @ S + Uh, GC * S + P @ S + R
        o[c0:c0 + n] = O[:n]
    return o, S


@pytest.mark.parametrize("channel", [False, True])
@pytest.mark.parametrize("T", [64, 150])
def test_kernel_dataflow_equals_the_token_recurrence(channel, T):
    rng = np.random.default_rng(3 + T + channel)
    Dk, Dv = 32, 16
    q = rng.standard_normal((T, Dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, Dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, Dv))
    shape = (T, Dk) if channel else (T,)
    g = -np.log1p(np.exp(-rng.normal(3.0, 1.0, shape)))           # logsigmoid(N(3, 1))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(T)))
    h0 = 0.02 * rng.standard_normal((Dk, Dv))
    o, hT = run_chunks(q, k, v, g, beta, h0, channel)
    o_ref, s_ref = oracle.recurrent(q[None, :, None], k[None, :, None], v[None, :, None],
                                    g[None, :, None], beta[None, :, None], h0[None, None])
    assert np.max(np.abs(o - o_ref[0, :, 0])) <= 1e-11 * np.max(np.abs(o_ref))
    assert np.max(np.abs(hT - s_ref[0, 0])) <= 1e-11 * np.max(np.abs(s_ref))
