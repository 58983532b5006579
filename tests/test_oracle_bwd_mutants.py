"""The backward's pins are strong enough: every plausible mistake planted in a CPU copy
of the token adjoint fails at least one pin, while the unmutated copy passes them all.

The mistakes are planted on the CPU, in this file only; the oracle itself is untouched.
The pins are those of test_oracle_bwd_pins.py: central differences of the forward
oracle, beta = 0 (no k or v gradient) and grouped heads (the key-head gradients sum
over the value heads that share it, which the central differences see with Hk < Hv).
"""
import numpy as np
import pytest

import oracle


def make_impl(mut=None):
    def impl(q, k, v, g, beta, h0, do, dhT):
        B, T, Hk, Dk = q.shape
        Hv, Dv = v.shape[2], v.shape[3]
        grp = Hv // Hk
        out = {"dq": np.zeros(q.shape), "dk": np.zeros(k.shape), "dv": np.zeros(v.shape),
               "dg": np.zeros(g.shape), "dbeta": np.zeros(beta.shape), "dh0": np.zeros((B, Hv, Dk, Dv))}
        for b in range(B):
            for h in range(Hv):
                hk = h // grp
                gate = lambda t: np.exp(g[b, t, h]) * np.ones(Dk) if g.ndim == 3 else np.exp(g[b, t, h])
                S = h0[b, h].copy()
                states = []
                for t in range(T):                      # forward, keeping the state entering each token
                    states.append(S)
                    Sb = gate(t)[:, None] * S
                    e = v[b, t, h] - Sb.T @ k[b, t, hk]
                    S = Sb + beta[b, t, h] * np.outer(k[b, t, hk], e)
                dS = np.zeros((Dk, Dv)) if mut == "dhT_ignored" else dhT[b, h].copy()
                for t in reversed(range(T)):
                    a, kt, qt, bt = gate(t), k[b, t, hk], q[b, t, hk], beta[b, t, h]
                    Sb = a[:, None] * states[t]
                    e = v[b, t, h] - Sb.T @ kt
                    Sn = Sb + bt * np.outer(kt, e)
                    if mut != "no_q_term":
                        dS = dS + np.outer(qt, do[b, t, h])
                    dq = (Sb if mut == "dq_uses_Sb" else Sn) @ do[b, t, h]
                    du = dS.T @ kt
                    dp = (bt if mut == "dk_sign" else -bt) * du
                    dk = dS @ (bt * e) + (0.0 if mut == "dk_drop_Sb_dp" else Sb @ dp)
                    db = du @ (v[b, t, h] if mut == "dbeta_uses_v" else e)
                    dv = du if mut == "dv_no_beta" else bt * du
                    dSb = dS + np.outer(kt, dp)
                    rg = np.sum((dS if mut == "dg_before_update" else dSb) * Sb, axis=1)
                    if mut == "heads_not_summed":
                        out["dq"][b, t, hk] = dq
                        out["dk"][b, t, hk] = dk
                    else:
                        out["dq"][b, t, hk] += dq
                        out["dk"][b, t, hk] += dk
                    out["dv"][b, t, h] = dv
                    out["dbeta"][b, t, h] = db
                    out["dg"][b, t, h] = rg if g.ndim == 4 else rg.sum()
                    if mut == "decay_columns":
                        dS = dSb * a[None, :Dv]
                    elif mut == "dh0_undecayed" and t == 0:
                        dS = dSb
                    else:
                        dS = a[:, None] * dSb
                out["dh0"][b, h] = dS
        return out
    return impl


MUTANTS = ["no_q_term", "dq_uses_Sb", "dk_sign", "dk_drop_Sb_dp", "dbeta_uses_v", "dv_no_beta",
           "dg_before_update", "heads_not_summed", "decay_columns", "dh0_undecayed", "dhT_ignored"]


def case(rng, gate):
    B, T, Hk, Hv, Dk, Dv = 1, 5, 1, 2, 3, 3
    x = dict(q=rng.standard_normal((B, T, Hk, Dk)), k=rng.standard_normal((B, T, Hk, Dk)) * 0.5,
             v=rng.standard_normal((B, T, Hv, Dv)),
             g=-np.abs(rng.standard_normal((B, T, Hv) if gate == "scalar" else (B, T, Hv, Dk))) * 0.3,
             beta=rng.uniform(0.1, 0.9, (B, T, Hv)), h0=rng.standard_normal((B, Hv, Dk, Dv)))
    return x, rng.standard_normal((B, T, Hv, Dv)), rng.standard_normal((B, Hv, Dk, Dv))


GRAD = dict(q="dq", k="dk", v="dv", g="dg", beta="dbeta", h0="dh0")


def run_pins(impl):
    failed = set()
    for gate, seed in (("scalar", 31), ("channel", 32)):
        rng = np.random.default_rng(seed)
        x, do, dhT = case(rng, gate)
        gr = impl(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], do, dhT)

        def loss(y):
            o, hT = oracle.recurrent(y["q"], y["k"], y["v"], y["g"], y["beta"], y["h0"])
            return float((o * do).sum() + (hT * dhT).sum())
        for name in x:
            u = rng.standard_normal(x[name].shape)
            xp, xm = dict(x), dict(x)
            xp[name], xm[name] = x[name] + 1e-6 * u, x[name] - 1e-6 * u
            fd = (loss(xp) - loss(xm)) / 2e-6
            an = float((gr[GRAD[name]] * u).sum())
            if abs(fd - an) > 1e-7 * max(1.0, abs(an)):
                failed.add(f"central differences ({gate}, {name})")
        z = dict(x, beta=np.zeros_like(x["beta"]))
        g0 = impl(z["q"], z["k"], z["v"], z["g"], z["beta"], z["h0"], do, dhT)
        if np.any(g0["dv"] != 0.0) or np.any(g0["dk"] != 0.0):
            failed.add(f"beta = 0 ({gate})")
    return failed


def test_unmutated_copy_passes_every_pin():
    assert run_pins(make_impl()) == set()


@pytest.mark.parametrize("mut", MUTANTS)
def test_each_mutant_fails_a_pin(mut):
    assert run_pins(make_impl(mut)), mut
