"""fp64 oracle of the layer's prologue and epilogue around the recurrence.

TEST INFRASTRUCTURE ONLY (the same rule as the rest of ``oracle/``).

What the pages fix, and the readings taken where they do not:

- ``causal_conv_silu``: the short causal convolution with SiLU applied to the
  q/k/v projections before the recurrence. NextTransformer "Source notes",
  section "Linear attention" (rows deltanet and kda: causal conv + SiLU, short
  conv), "Backend and numerical limits" (a causal convolution with SiLU
  activation), and the Atlas entry 03 Gated DeltaNet (a four-token causal
  convolution). Reading: depthwise over channels, W = 4 taps, tap W-1 on the
  current token, an optional per-channel bias, history before a sequence's first
  token taken from a caller's conv state (else zero), SiLU(y) = y / (1 + e^-y).
- ``l2norm``: L2-normalized q and k (same rows deltanet and kda). Reading:
  x / sqrt(sum x^2 + eps) over the head dimension, eps = 1e-6 (the pages give no
  eps).
- ``rmsnorm_gated``: the GDN output, RMSNorm x gain x SiLU gate (row gdn;
  "Backend and numerical limits": a gated RMSNorm). Reading: per head over Dv,
  o / sqrt(mean(o^2) + eps) * weight * SiLU(z), eps = 1e-5.

Each function is the definition written out, one token or row at a time.
"""
import numpy as np


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def silu(y):
    return y / (1.0 + np.exp(-y))


def causal_conv_silu(x, w, bias=None, conv_state=None, cu_seqlens=None):
    """x: [B, T, Ch] (or [1, T_total, Ch] with cu_seqlens of N + 1 offsets);
    w: [Ch, W]; bias: [Ch] or None; conv_state: [B or N, Ch, W - 1] inputs
    preceding each sequence (oldest first) or None for zeros.

    Returns (y [same shape as x], final_state [B or N, Ch, W - 1]): y[t, c] =
    SiLU(bias[c] + sum_j w[c, j] x[t - (W - 1) + j, c]), and final_state the
    last W - 1 inputs of each sequence (reaching into conv_state when the
    sequence is shorter than W - 1).
    """
    x, w, bias, conv_state = (_f64(a) for a in (x, w, bias, conv_state))
    Bx, T, Ch = x.shape
    W = w.shape[1]
    if cu_seqlens is None:
        spans = [(b, 0, T) for b in range(Bx)]
    else:
        cu = [int(c) for c in np.asarray(cu_seqlens).reshape(-1)]
        assert Bx == 1
        spans = [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    y = np.zeros_like(x)
    final = np.zeros((len(spans), Ch, W - 1))
    for n, (b, s0, s1) in enumerate(spans):
        hist = np.zeros((W - 1, Ch)) if conv_state is None else conv_state[n].T.copy()
        for t in range(s0, s1):
            window = np.concatenate([hist, x[b, t][None]], 0)   # [W, Ch], oldest first
            acc = np.zeros(Ch) if bias is None else bias.copy()
            for j in range(W):
                acc += w[:, j] * window[j]
            y[b, t] = silu(acc)
            hist = window[1:]
        final[n] = hist.T
    return y, final


def l2norm(x, eps=1e-6):
    """x / sqrt(sum(x^2) + eps) over the last axis."""
    x = _f64(x)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def rmsnorm_gated(o, z, weight, eps=1e-5):
    """o / sqrt(mean(o^2) + eps) * weight * SiLU(z) over the last axis."""
    o, z, weight = (_f64(a) for a in (o, z, weight))
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    return o / rms * weight * silu(z)
