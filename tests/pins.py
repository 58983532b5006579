"""Checks that pin a gated delta-rule implementation to facts fixed outside it.

Each ``pin_*`` takes ``impl(q, k, v, g, beta, h0) -> (o, hT)`` working on fp64
numpy arrays in the library layout (q,k [B,T,Hk,Dk]; v,o [B,T,Hv,Dv];
g [B,T,Hv] or [B,T,Hv,Dk]; beta [B,T,Hv]; h0,hT [B,Hv,Dk,Dv]) and raises
AssertionError when the implementation disagrees. The expected values come from
closed forms, brute force or invariants computed here, never from the
implementation under test.

The recurrence being pinned (NextTransformer, "Source notes", section "Linear
attention"): S <- alpha (I - beta k k^T) S + beta k v^T for GDN (scalar decay
before the delta update), per-key-channel decay before the delta update for
KDA, S <- S + k[beta(v - k^T S)]^T for DeltaNet, readout y = q^T S, scale 1.
"""
from fractions import Fraction

import numpy as np


def rand_case(rng, B=1, T=12, Hk=1, Hv=1, Dk=5, Dv=4, gate="scalar", h0=True,
              unit_keys=True):
    q = rng.standard_normal((B, T, Hk, Dk))
    k = rng.standard_normal((B, T, Hk, Dk))
    if unit_keys:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, Hv, Dv))
    gshape = (B, T, Hv) if gate == "scalar" else (B, T, Hv, Dk)
    g = -np.log1p(np.exp(-(rng.standard_normal(gshape) + 1.0)))  # logsigmoid(N(1,1)) < 0
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, Hv))))
    s0 = 0.5 * rng.standard_normal((B, Hv, Dk, Dv)) if h0 else None
    return q, k, v, g, beta, s0


def _rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


def _decay_vec(g, b, t, h, Dk):
    return np.exp(g[b, t, h]) * np.ones(Dk) if g.ndim == 3 else np.exp(g[b, t, h])


# --- brute force: history expansion -----------------------------------------------------
def pin_history_expansion(impl, seed=0, gate="scalar", T=12, Dk=5, Dv=4, Hk=1, Hv=1):
    """S_t = P_t...P_1 h0 + sum_{i<=t} P_t...P_{i+1} beta_i k_i v_i^T with the explicit
    Dk x Dk transition P_j = (I - beta_j k_j k_j^T) diag(exp g_j) (decay, then delta)."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, h0 = rand_case(rng, T=T, Dk=Dk, Dv=Dv, Hk=Hk, Hv=Hv, gate=gate)
    o, hT = impl(q, k, v, g, beta, h0)
    grp = Hv // Hk
    for h in range(Hv):
        hk = h // grp
        P = [(np.eye(Dk) - beta[0, j, h] * np.outer(k[0, j, hk], k[0, j, hk]))
             @ np.diag(_decay_vec(g, 0, j, h, Dk)) for j in range(T)]
        for t in range(T):
            prod = np.eye(Dk)
            for j in range(t, -1, -1):
                prod = prod @ P[j]
            S = prod @ h0[0, h]
            for i in range(t + 1):
                M = np.eye(Dk)
                for j in range(t, i, -1):
                    M = M @ P[j]
                S = S + M @ (beta[0, i, h] * np.outer(k[0, i, hk], v[0, i, h]))
            exp_o = S.T @ q[0, t, hk]
            assert _rel(o[0, t, h], exp_o) < 1e-12, ("history expansion: o", t, h)
        assert _rel(hT[0, h], S) < 1e-12, ("history expansion: hT", h)


# --- closed form: beta = 0 is pure decay of h0 -------------------------------------------
def pin_beta_zero(impl, seed=1, gate="channel"):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, h0 = rand_case(rng, T=20, Dk=6, Dv=3, gate=gate)
    beta[:] = 0.0
    o, hT = impl(q, k, v, g, beta, h0)
    G = np.cumsum(g[0, :, 0], axis=0)             # [T] or [T, Dk]
    for t in range(20):
        d = np.exp(G[t]) * np.ones(6)
        S = d[:, None] * h0[0, 0]
        assert _rel(o[0, t, 0], S.T @ q[0, t, 0]) < 1e-12, ("beta=0: o", t)
    assert _rel(hT[0, 0], S) < 1e-12, "beta=0: hT"


# --- special case: alpha = 1 is DeltaNet --------------------------------------------------
def pin_deltanet(impl, seed=2):
    """g = 0 must give the DeltaNet row: S <- S + k [beta (v - k^T S)]^T, y = q^T S."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, h0 = rand_case(rng, T=16, Dk=7, Dv=5)
    g[:] = 0.0
    o, hT = impl(q, k, v, g, beta, h0)
    S = h0[0, 0].copy()
    for t in range(16):
        kt, vt, bt = k[0, t, 0], v[0, t, 0], beta[0, t, 0]
        row = kt @ S                               # k^T S, a row over Dv
        S = S + np.outer(kt, bt * (vt - row))
        assert _rel(o[0, t, 0], q[0, t, 0] @ S) < 1e-12, ("deltanet: o", t)
    assert _rel(hT[0, 0], S) < 1e-12, "deltanet: hT"


# --- exact retrieval: beta = 1 with orthonormal keys --------------------------------------
def pin_exact_retrieval(impl, seed=3, Dk=8, Dv=5, T=8):
    """With beta = 1, orthonormal keys, h0 = 0 and a scalar gate, the state stores each
    value exactly: S_T^T k_i = (prod_{j=i+1..T} alpha_j) v_i, and reading with q_t = k_t
    right after writing gives o_t = v_t."""
    rng = np.random.default_rng(seed)
    Qm, _ = np.linalg.qr(rng.standard_normal((Dk, Dk)))
    keys = Qm[:, :T].T                             # T orthonormal rows
    k = keys[None, :, None, :].copy()
    q = k.copy()
    v = rng.standard_normal((1, T, 1, Dv))
    g = -np.abs(rng.standard_normal((1, T, 1))) * 0.3
    beta = np.ones((1, T, 1))
    o, hT = impl(q, k, v, g, beta, np.zeros((1, 1, Dk, Dv)))
    for t in range(T):
        assert np.max(np.abs(o[0, t, 0] - v[0, t, 0])) < 1e-12, ("retrieval: o_t = v_t", t)
    for i in range(T):
        decay = np.exp(np.sum(g[0, i + 1:, 0]))
        got = hT[0, 0].T @ keys[i]
        assert np.max(np.abs(got - decay * v[0, i, 0])) < 1e-12, ("retrieval: S^T k_i", i)
    g0 = np.zeros_like(g)
    _, hT0 = impl(q, k, v, g0, beta, np.zeros((1, 1, Dk, Dv)))
    for i in range(T):
        assert np.max(np.abs(hT0[0, 0].T @ keys[i] - v[0, i, 0])) < 1e-12, ("retrieval g=0", i)


# --- invariant: a scalar gate equals the same gate broadcast over key channels -------------
def pin_scalar_is_broadcast_channel(impl, seed=4):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, h0 = rand_case(rng, T=24, Dk=6, Dv=4, Hk=2, Hv=4)
    o1, s1 = impl(q, k, v, g, beta, h0)
    gc = np.repeat(g[..., None], 6, axis=-1)
    o2, s2 = impl(q, k, v, gc, beta, h0)
    assert _rel(o1, o2) < 1e-14 and _rel(s1, s2) < 1e-14, "scalar gate != broadcast channel gate"


# --- invariant: grouped value heads equal the expanded per-head form -----------------------
def pin_grouped_heads(impl, seed=5, Hk=2, Hv=6):
    """Hk key heads shared by Hv value heads == Hv key heads with q, k repeated per group
    (value head h reads key head h // (Hv // Hk))."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, h0 = rand_case(rng, B=2, T=10, Hk=Hk, Hv=Hv, Dk=4, Dv=3, gate="channel")
    o1, s1 = impl(q, k, v, g, beta, h0)
    rep = Hv // Hk
    o2, s2 = impl(np.repeat(q, rep, axis=2), np.repeat(k, rep, axis=2), v, g, beta, h0)
    assert _rel(o1, o2) < 1e-14 and _rel(s1, s2) < 1e-14, "grouped heads != expanded heads"


# --- closed form: Dk = Dv = 1 is a first-order linear recurrence ---------------------------
def pin_scalar_state(impl, seed=6, T=30):
    """s_t = a_t s_{t-1} + b_t with a_t = alpha_t (1 - beta_t k_t^2), b_t = beta_t k_t v_t,
    solved by prefix products: s_t = (prod_{j<=t} a_j) s_0 + sum_{i<=t} (prod_{i<j<=t} a_j) b_i."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, T, 1, 1))
    k = rng.uniform(-1, 1, (1, T, 1, 1))
    v = rng.standard_normal((1, T, 1, 1))
    g = -rng.uniform(0.01, 0.5, (1, T, 1))
    beta = rng.uniform(0.05, 0.95, (1, T, 1))
    s0 = np.array([[[[0.7]]]])
    o, hT = impl(q, k, v, g, beta, s0)
    a = np.exp(g[0, :, 0]) * (1.0 - beta[0, :, 0] * k[0, :, 0, 0] ** 2)
    b = beta[0, :, 0] * k[0, :, 0, 0] * v[0, :, 0, 0]
    for t in range(T):
        s = np.prod(a[:t + 1]) * 0.7 + sum(np.prod(a[i + 1:t + 1]) * b[i] for i in range(t + 1))
        assert abs(o[0, t, 0, 0] - q[0, t, 0, 0] * s) < 1e-12, ("scalar state: o", t)
    assert abs(hT[0, 0, 0, 0] - s) < 1e-12, "scalar state: hT"


# --- exact rational worked example ---------------------------------------------------------
def pin_rational_example(impl):
    """Dk = Dv = 2, three tokens with rational data, evaluated exactly with Fractions from
    S <- alpha (I - beta k k^T) S + beta k v^T, o = S^T q; alpha enters as g = log(alpha)."""
    F = Fraction
    ks = [(F(1), F(0)), (F(0), F(1)), (F(3, 5), F(4, 5))]
    qs = [(F(1), F(0)), (F(3, 5), F(4, 5)), (F(0), F(1))]
    vs = [(F(2), F(-1)), (F(1, 2), F(3)), (F(-1), F(1, 4))]
    alphas = [F(1, 2), F(3, 4), F(1)]
    betas = [F(1, 2), F(1), F(1, 4)]
    S = [[F(1, 10), F(0)], [F(0), F(-1, 5)]]
    S0 = [row[:] for row in S]
    exp_o = []
    for t in range(3):
        kk, vv, a, bt = ks[t], vs[t], alphas[t], betas[t]
        # alpha (I - beta k k^T) S
        SA = [[a * S[i][j] for j in range(2)] for i in range(2)]
        kS = [kk[0] * SA[0][j] + kk[1] * SA[1][j] for j in range(2)]
        S = [[SA[i][j] - bt * kk[i] * kS[j] + bt * kk[i] * vv[j] for j in range(2)]
             for i in range(2)]
        exp_o.append([qs[t][0] * S[0][j] + qs[t][1] * S[1][j] for j in range(2)])
    q = np.array([[[[float(x) for x in qs[t]]] for t in range(3)]])
    k = np.array([[[[float(x) for x in ks[t]]] for t in range(3)]])
    v = np.array([[[[float(x) for x in vs[t]]] for t in range(3)]])
    g = np.log(np.array([[[float(a)] for a in alphas]]))
    beta = np.array([[[float(b)] for b in betas]])
    h0 = np.array([[[[float(x) for x in row] for row in S0]]])
    o, hT = impl(q, k, v, g, beta, h0)
    for t in range(3):
        for j in range(2):
            assert abs(o[0, t, 0, j] - float(exp_o[t][j])) < 1e-14, ("rational: o", t, j)
    for i in range(2):
        for j in range(2):
            assert abs(hT[0, 0, i, j] - float(S[i][j])) < 1e-14, ("rational: hT", i, j)


# --- causality: future inputs never change past outputs -----------------------------------
def pin_causality(impl, seed=7, T=20, t0=9):
    rng = np.random.default_rng(seed)
    case = rand_case(rng, T=T, Dk=4, Dv=4, gate="channel")
    o1, _ = impl(*case)
    pert = [None if x is None else x.copy() for x in case]
    for idx in range(5):                          # q, k, v, g, beta after t0
        pert[idx][:, t0 + 1:] += 0.37
    o2, _ = impl(*pert)
    assert np.array_equal(o1[:, :t0 + 1], o2[:, :t0 + 1]), "causality: o_{<=t} changed"
    assert not np.array_equal(o1[:, t0 + 1:], o2[:, t0 + 1:]), "causality: perturbation had no effect"


# --- state passing: split a sequence and pass hT as h0 -------------------------------------
def pin_state_passing(impl, seed=8, T=26, cut=11):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, h0 = rand_case(rng, T=T, Dk=5, Dv=6, gate="channel")
    o, hT = impl(q, k, v, g, beta, h0)
    oa, sa = impl(q[:, :cut], k[:, :cut], v[:, :cut], g[:, :cut], beta[:, :cut], h0)
    ob, sb = impl(q[:, cut:], k[:, cut:], v[:, cut:], g[:, cut:], beta[:, cut:], sa)
    assert _rel(np.concatenate([oa, ob], 1), o) < 1e-13 and _rel(sb, hT) < 1e-13, "state passing"


# --- contraction: with |k| <= 1, beta in [0,1], g <= 0 the state grows at most by beta|k||v| ---
def pin_contraction(impl, seed=9, T=40):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, h0 = rand_case(rng, T=T, Dk=6, Dv=5, gate="channel")
    S = h0
    for t in range(T):
        _, S_new = impl(q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1], g[:, t:t + 1],
                        beta[:, t:t + 1], S)
        bound = (np.linalg.norm(S) + beta[0, t, 0] * np.linalg.norm(k[0, t, 0])
                 * np.linalg.norm(v[0, t, 0]))
        assert np.linalg.norm(S_new) <= bound * (1 + 1e-12), ("contraction", t)
        S = S_new


ALL_PINS = [pin_history_expansion, pin_beta_zero, pin_deltanet, pin_exact_retrieval,
            pin_scalar_is_broadcast_channel, pin_grouped_heads, pin_scalar_state,
            pin_rational_example, pin_causality, pin_state_passing, pin_contraction]


def pin_history_expansion_channel(impl):
    pin_history_expansion(impl, seed=10, gate="channel", Hk=1, Hv=2)


ALL_PINS.append(pin_history_expansion_channel)
