"""The pins are strong enough: every plausible mistake planted in a CPU copy of the
recurrence fails at least one pin, while the unmutated copy passes them all.

The mistakes are planted on the CPU, in this file only; the oracle itself is untouched.
"""
import numpy as np
import pytest

from tests import pins


def make_impl(mut=None):
    def impl(q, k, v, g, beta, h0):
        B, T, Hk, Dk = q.shape
        Hv, Dv = v.shape[2], v.shape[3]
        grp = Hv // Hk
        o = np.zeros((B, T, Hv, Dv))
        hT = np.zeros((B, Hv, Dk, Dv))
        for b in range(B):
            for h in range(Hv):
                hk = (h % Hk) if mut == "strided_heads" else h // grp
                S = np.zeros((Dk, Dv)) if (h0 is None or mut == "ignore_h0") else h0[b, h].copy()
                for t in range(T):
                    kt, qt, vt, bt = k[b, t, hk], q[b, t, hk], v[b, t, h], beta[b, t, h]
                    tg = max(t - 1, 0) if mut == "gate_off_by_one" else t
                    d = np.exp(g[b, tg, h]) * np.ones(Dk) if g.ndim == 3 else np.exp(g[b, tg, h])
                    if mut == "neg_gate":
                        d = 1.0 / d
                    S_prev = S
                    if mut == "decay_columns":
                        S = S * d[None, :Dv]
                    elif mut != "decay_after":
                        S = d[:, None] * S
                    p = (S_prev if mut == "stale_prediction" else S).T @ kt
                    b_ = 1.0 if mut == "no_beta" else bt
                    sign = -1.0 if mut == "sign" else 1.0
                    S_upd = S + sign * b_ * np.outer(kt, vt - p)
                    if mut == "decay_after":
                        S_upd = d[:, None] * S_upd
                    if mut == "read_before":
                        o[b, t, h] = S.T @ qt
                    elif mut == "read_transposed":
                        o[b, t, h] = S_upd @ qt[:Dv] if Dk == Dv else S_upd.T @ qt * 1.0001
                    elif mut == "scale_rsqrt":
                        o[b, t, h] = S_upd.T @ qt / np.sqrt(Dk)
                    else:
                        o[b, t, h] = S_upd.T @ qt
                    S = S_upd
                hT[b, h] = S
        return o, hT
    return impl


MUTANTS = ["decay_after", "no_beta", "sign", "read_before", "read_transposed", "neg_gate",
           "gate_off_by_one", "stale_prediction", "strided_heads", "ignore_h0",
           "decay_columns", "scale_rsqrt"]


def run_pins(impl):
    failed = []
    for pin in pins.ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(impl)
        except (AssertionError, IndexError, ValueError):
            failed.append(pin.__name__)
    return failed


def test_unmutated_copy_passes_every_pin():
    assert run_pins(make_impl(None)) == []


@pytest.mark.parametrize("mut", MUTANTS)
def test_mutant_is_caught(mut):
    assert run_pins(make_impl(mut)), f"no pin catches the planted mistake '{mut}'"
