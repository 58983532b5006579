"""Pins of the oracle's backward (oracle.backward) that do not use its code.

The backward is the adjoint of the token loop; here it is tied to:
- central finite differences of L = sum(do * o) + sum(dhT * hT) computed with the
  forward oracle, along random directions, for every input and both gates;
- special cases: beta = 0 leaves v and k without gradient (the delta term is zero);
- invariants: the gradient is linear in the upstream gradients; a scalar gate's
  gradient is the sum over channels of the per-channel gate's when the gate is
  broadcast (NextTransformer, "Backend and numerical limits": gdn as the
  per-channel backend with a broadcast gate); grouped value heads' dq, dk equal the
  sum over the expanded heads;
- a second algorithm: the adjoint of the exact chunk map, chunk by chunk.
"""
import numpy as np
import pytest

import oracle


def case(rng, B=1, T=7, Hk=1, Hv=2, Dk=4, Dv=3, gate="scalar"):
    q = rng.standard_normal((B, T, Hk, Dk))
    k = rng.standard_normal((B, T, Hk, Dk)) * 0.5
    v = rng.standard_normal((B, T, Hv, Dv))
    gs = (B, T, Hv) if gate == "scalar" else (B, T, Hv, Dk)
    g = -np.abs(rng.standard_normal(gs)) * 0.3
    beta = rng.uniform(0.1, 0.9, (B, T, Hv))
    h0 = rng.standard_normal((B, Hv, Dk, Dv))
    do = rng.standard_normal((B, T, Hv, Dv))
    dhT = rng.standard_normal((B, Hv, Dk, Dv))
    return dict(q=q, k=k, v=v, g=g, beta=beta, h0=h0), do, dhT


def loss(x, do, dhT):
    o, hT = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
    return float((o * do).sum() + (hT * dhT).sum())


GRAD = dict(q="dq", k="dk", v="dv", g="dg", beta="dbeta", h0="dh0")


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("shape", [dict(Hk=1, Hv=2), dict(Hk=2, Hv=2, T=9, Dk=3, Dv=5)])
def test_matches_central_differences(gate, shape):
    rng = np.random.default_rng(11 if gate == "scalar" else 12)
    x, do, dhT = case(rng, gate=gate, **shape)
    gr = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], do, dhT)
    eps = 1e-6
    for name in x:
        u = rng.standard_normal(x[name].shape)
        xp, xm = dict(x), dict(x)
        xp[name] = x[name] + eps * u
        xm[name] = x[name] - eps * u
        fd = (loss(xp, do, dhT) - loss(xm, do, dhT)) / (2 * eps)
        an = float((gr[GRAD[name]] * u).sum())
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (gate, name, fd, an)


def test_no_hT_gradient_means_zero():
    rng = np.random.default_rng(13)
    x, do, _ = case(rng)
    a = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], do, None)
    b = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], do, np.zeros_like(x["h0"]))
    for n in a:
        assert np.array_equal(a[n], b[n]), n


def test_beta_zero_gives_no_v_or_k_gradient():
    rng = np.random.default_rng(14)
    x, do, dhT = case(rng)
    x["beta"] = np.zeros_like(x["beta"])
    gr = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], do, dhT)
    assert np.all(gr["dv"] == 0.0) and np.all(gr["dk"] == 0.0)


def test_linear_in_upstream_gradients():
    rng = np.random.default_rng(15)
    x, do1, dh1 = case(rng, gate="channel")
    do2, dh2 = rng.standard_normal(do1.shape), rng.standard_normal(dh1.shape)
    args = (x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"])
    a, b, ab = oracle.backward(*args, do1, dh1), oracle.backward(*args, do2, dh2), \
        oracle.backward(*args, do1 + do2, dh1 + dh2)
    for n in a:
        assert np.allclose(ab[n], a[n] + b[n], rtol=1e-12, atol=1e-12), n


def test_scalar_gate_gradient_is_the_channel_sum():
    rng = np.random.default_rng(16)
    x, do, dhT = case(rng)
    gch = np.repeat(x["g"][..., None], x["q"].shape[-1], axis=-1)
    a = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], do, dhT)
    b = oracle.backward(x["q"], x["k"], x["v"], gch, x["beta"], x["h0"], do, dhT)
    assert np.allclose(a["dg"], b["dg"].sum(-1), rtol=1e-12, atol=1e-12)
    for n in ("dq", "dk", "dv", "dbeta", "dh0"):
        assert np.allclose(a[n], b[n], rtol=1e-12, atol=1e-12), n


def test_grouped_heads_sum_over_the_expanded_heads():
    rng = np.random.default_rng(17)
    x, do, dhT = case(rng, Hk=2, Hv=4)
    grp = 2
    qe, ke = (np.repeat(x[n], grp, axis=2) for n in ("q", "k"))
    a = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], do, dhT)
    b = oracle.backward(qe, ke, x["v"], x["g"], x["beta"], x["h0"], do, dhT)
    B, T, Hk, Dk = x["q"].shape
    for n in ("dq", "dk"):
        assert np.allclose(a[n], b[n].reshape(B, T, Hk, grp, Dk).sum(3), rtol=1e-12, atol=1e-12), n
    for n in ("dv", "dg", "dbeta", "dh0"):
        assert np.allclose(a[n], b[n], rtol=1e-12, atol=1e-12), n


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("T,chunk", [(7, 1), (20, 8), (33, 16), (100, 64)])
def test_chunkwise_adjoint_matches_the_token_adjoint(gate, T, chunk):
    """A second algorithm: the adjoint of the exact chunk map (oracle/chunked.py), chunk by
    chunk in reverse, equals the token loop's adjoint within 1e-10 (max error over rms),
    with grouped heads and a ragged last chunk."""
    from oracle.chunked import chunked_backward
    rng = np.random.default_rng(100 + T)
    x, do, dhT = case(rng, B=2, T=T, Hk=1, Hv=2, Dk=6, Dv=5, gate=gate)
    a = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], do, dhT)
    b = chunked_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], do, dhT, chunk=chunk)
    for n in a:
        err = np.max(np.abs(a[n] - b[n])) / max(np.sqrt(np.mean(a[n] ** 2)), 1e-30)
        assert err <= 1e-10, (gate, T, chunk, n, err)
