"""The prologue/epilogue oracle pinned to library routines, closed forms and invariants (CPU)."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import prologue


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _torch_conv_silu(x, w, bias, state):
    """Depthwise conv1d from torch (groups = channels) over [state ; x], then x * sigmoid(x)."""
    B, T, Ch = x.shape
    W = w.shape[1]
    xt = torch.from_numpy(x).permute(0, 2, 1)                              # [B, Ch, T]
    if state is not None:
        xt = torch.cat([torch.from_numpy(state), xt], 2)                   # [B, Ch, W-1+T]
        pad = 0
    else:
        pad = W - 1
    y = F.conv1d(xt, torch.from_numpy(w)[:, None, :], None if bias is None else torch.from_numpy(bias),
                 padding=pad, groups=Ch)
    y = y[..., :T] if state is None else y
    y = y * torch.sigmoid(y)
    return y.permute(0, 2, 1).numpy()


@pytest.mark.parametrize("with_bias,with_state", [(False, False), (True, False), (True, True)])
def test_conv_matches_torch_depthwise_conv1d(with_bias, with_state):
    rng = np.random.default_rng(40)
    B, T, Ch, W = 2, 37, 12, 4
    x, w = _rand(rng, B, T, Ch), _rand(rng, Ch, W)
    bias = _rand(rng, Ch) if with_bias else None
    state = _rand(rng, B, Ch, W - 1) if with_state else None
    y, _ = prologue.causal_conv_silu(x, w, bias, state)
    ref = _torch_conv_silu(x, w, bias, state)
    assert np.max(np.abs(y - ref)) < 1e-12


def test_conv_impulse_response_is_the_reversed_taps():
    """A unit impulse at token t0 of channel c gives SiLU(w[c, W-1-j]) at t0 + j, SiLU(0) = 0 elsewhere."""
    rng = np.random.default_rng(41)
    T, Ch, W, t0, c = 20, 3, 4, 7, 1
    w = _rand(rng, Ch, W)
    x = np.zeros((1, T, Ch))
    x[0, t0, c] = 1.0
    y, _ = prologue.causal_conv_silu(x, w)
    expect = np.zeros((1, T, Ch))
    for j in range(W):
        a = w[c, W - 1 - j]
        expect[0, t0 + j, c] = a / (1.0 + np.exp(-a))
    assert np.array_equal(y, expect)


def test_conv_state_carries_a_split_sequence():
    rng = np.random.default_rng(42)
    B, T, Ch, W = 2, 29, 5, 4
    x, w, bias = _rand(rng, B, T, Ch), _rand(rng, Ch, W), _rand(rng, Ch)
    y, s = prologue.causal_conv_silu(x, w, bias)
    for T1 in (1, 2, 3, 11):
        ya, sa = prologue.causal_conv_silu(x[:, :T1], w, bias)
        yb, sb = prologue.causal_conv_silu(x[:, T1:], w, bias, sa)
        assert np.array_equal(np.concatenate([ya, yb], 1), y) and np.array_equal(sb, s)


def test_conv_final_state_of_short_sequences_reaches_into_the_given_state():
    rng = np.random.default_rng(43)
    Ch, W = 4, 4
    w, state = _rand(rng, Ch, W), _rand(rng, 1, Ch, W - 1)
    for T in (1, 2, 3, 5):
        x = _rand(rng, 1, T, Ch)
        _, s = prologue.causal_conv_silu(x, w, None, state)
        hist = np.concatenate([state[0].T, x[0]], 0)   # [W-1+T, Ch], oldest first
        assert np.array_equal(s[0], hist[-(W - 1):].T)


def test_conv_packed_sequences_equal_separate_calls():
    rng = np.random.default_rng(44)
    Ch, W = 6, 4
    lens = [5, 1, 0, 17, 2]
    cu = np.concatenate([[0], np.cumsum(lens)])
    x, w, bias = _rand(rng, 1, cu[-1], Ch), _rand(rng, Ch, W), _rand(rng, Ch)
    state = _rand(rng, len(lens), Ch, W - 1)
    y, s = prologue.causal_conv_silu(x, w, bias, state, cu_seqlens=cu)
    for n in range(len(lens)):
        yn, sn = prologue.causal_conv_silu(x[:, cu[n]:cu[n + 1]], w, bias, state[n:n + 1])
        assert np.array_equal(y[:, cu[n]:cu[n + 1]], yn) and np.array_equal(s[n:n + 1], sn)


def test_l2norm_matches_torch_normalize_and_is_scale_free():
    rng = np.random.default_rng(45)
    x = _rand(rng, 7, 128)
    y = prologue.l2norm(x)
    ref = F.normalize(torch.from_numpy(x), p=2.0, dim=-1).numpy()   # x / max(|x|, 1e-12)
    # the two differ only by eps = 1e-6 inside the root: relative 5e-7 / |x|^2
    assert np.max(np.abs(y - ref)) < 1e-8
    assert np.max(np.abs(prologue.l2norm(3.0 * x) - y)) < 1e-8
    assert np.allclose(np.linalg.norm(y, axis=-1), 1.0, atol=1e-8)


def test_rmsnorm_gated_matches_torch_rms_norm_times_silu():
    rng = np.random.default_rng(46)
    o, z, wt = _rand(rng, 9, 128), _rand(rng, 9, 128), _rand(rng, 128)
    y = prologue.rmsnorm_gated(o, z, wt)
    ref = F.rms_norm(torch.from_numpy(o), (128,), torch.from_numpy(wt), eps=1e-5) * F.silu(torch.from_numpy(z))
    assert np.max(np.abs(y - ref.numpy())) < 1e-12


def test_rmsnorm_gated_of_a_constant_row():
    """o = c (every channel): rms = sqrt(c^2 + eps), so y = c / sqrt(c^2 + eps) * weight * SiLU(z)."""
    z = np.linspace(-3, 3, 16)[None]
    wt = np.linspace(0.5, 2.0, 16)
    for c in (-2.0, 0.25, 10.0):
        y = prologue.rmsnorm_gated(np.full((1, 16), c), z, wt)
        expect = c / np.sqrt(c * c + 1e-5) * wt * (z / (1.0 + np.exp(-z)))
        assert np.max(np.abs(y - expect)) < 1e-14
