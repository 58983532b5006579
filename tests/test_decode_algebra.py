"""The decode kernel's single-pass step (csrc/decode.cu), restated in fp64, against the
oracle's decode steps (no GPU).

The kernel reads the state once and writes it once: with S' = diag(exp g) S it forms S'^T k
and S'^T q in the same pass, then u = beta (v - S'^T k), writes S' + k u^T and reads out
o = S'^T q + (q . k) u, which equals (S' + k u^T)^T q, the readout after the update, without
a second pass over the state.
"""
import numpy as np
import pytest

import oracle


def decode_as_kernel(q, k, v, g, beta, S):
    d = np.exp(g) if np.ndim(g) else np.full(S.shape[0], np.exp(g))
    Sp = d[:, None] * S
    Spk, Spq = Sp.T @ k, Sp.T @ q
    u = beta * (v - Spk)
    return Spq + (q @ k) * u, Sp + np.outer(k, u)


@pytest.mark.parametrize("channel", [False, True])
def test_single_pass_step_equals_the_oracle(channel):
    rng = np.random.default_rng(11 + channel)
    steps, Dk, Dv = 6, 16, 8
    q = rng.standard_normal((steps, 1, 1, Dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.standard_normal((steps, 1, 1, Dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((steps, 1, 1, Dv))
    g = -np.log1p(np.exp(-rng.normal(3.0, 1.0, (steps, 1, 1, Dk) if channel else (steps, 1, 1))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((steps, 1, 1))))
    h0 = 0.02 * rng.standard_normal((1, 1, Dk, Dv))
    o_ref, s_ref = oracle.decode_steps(q, k, v, g, beta, h0)
    S = h0[0, 0]
    for s in range(steps):
        o, S = decode_as_kernel(q[s, 0, 0], k[s, 0, 0], v[s, 0, 0], g[s, 0, 0], beta[s, 0, 0], S)
        assert np.max(np.abs(o - o_ref[s, 0, 0])) <= 1e-13
    assert np.max(np.abs(S - s_ref[0, 0])) <= 1e-13
