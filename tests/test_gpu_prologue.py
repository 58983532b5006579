"""GPU parity of the causal conv + SiLU and the gated RMSNorm against the fp64 oracle."""
import numpy as np
import pytest
import torch

import gated_delta_rule_68_b200 as gdr
from oracle import prologue

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def err(got, ref):
    """max|got - ref| / rms(ref), not counting the round-to-nearest of a bf16 output: half an
    ulp of ref, 2^(floor(log2 |ref|) - 8). What is left is the fp32 arithmetic, so both
    dtypes meet 1e-4."""
    g = got.detach().double().cpu().numpy()
    ref = np.asarray(ref, np.float64)
    allow = 0.0
    if got.dtype == torch.bfloat16:
        allow = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 8)
    rms = np.sqrt(np.mean(ref ** 2))
    return float(np.max(np.maximum(np.abs(g - ref) - allow, 0.0)) / max(rms, 1e-30))


TOL = 1e-4


def _gen(seed):
    return torch.Generator().manual_seed(seed)


def _conv_inputs(B, T, Ch, dtype, seed, packed=False):
    g = _gen(seed)
    shape = (T, Ch) if packed else (B, T, Ch)
    x = torch.randn(shape, generator=g).to(dtype)
    w = (0.5 * torch.randn(Ch, 4, generator=g)).float()
    bias = (0.1 * torch.randn(Ch, generator=g)).float()
    state = torch.randn(B, Ch, 3, generator=g).to(dtype)
    return x, w, bias, state


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("B,T,Ch", [(2, 100, 48), (1, 1, 8), (3, 16, 64), (2, 2, 16), (1, 47, 128)])
@pytest.mark.parametrize("with_state", [False, True])
def test_conv_matches_oracle(dtype, B, T, Ch, with_state):
    x, w, bias, state = _conv_inputs(B, T, Ch, dtype, seed=B * 1000 + T + Ch)
    st = state if with_state else None
    y, s_out = gdr.gdr_causal_conv_silu(x.to(DEV), w.to(DEV), bias.to(DEV),
                                        None if st is None else st.to(DEV), want_state=True)
    torch.cuda.synchronize()
    y_ref, s_ref = prologue.causal_conv_silu(x, w, bias, st)
    assert err(y, y_ref) <= TOL
    # the final state is a copy of inputs: exact
    assert np.array_equal(s_out.double().cpu().numpy(), s_ref)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_conv_packed_sequences(dtype):
    lens = [5, 0, 1, 37, 2, 64, 0, 17]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    N, Ch = len(lens), 40
    x, w, bias, state = _conv_inputs(N, int(cu[-1]), Ch, dtype, seed=7, packed=True)
    y, s_out = gdr.gdr_causal_conv_silu(x.to(DEV), w.to(DEV), bias.to(DEV), state.to(DEV), cu.to(DEV),
                                        want_state=True)
    torch.cuda.synchronize()
    y_ref, s_ref = prologue.causal_conv_silu(x[None], w, bias, state, cu_seqlens=cu.numpy())
    assert err(y, y_ref[0]) <= TOL
    assert np.array_equal(s_out.double().cpu().numpy(), s_ref)


def test_conv_split_sequence_through_the_state():
    """One call over T tokens equals two calls over [0, T1) and [T1, T) joined by the state."""
    x, w, bias, _ = _conv_inputs(2, 90, 32, torch.bfloat16, seed=8)
    xd, wd, bd = x.to(DEV), w.to(DEV), bias.to(DEV)
    y, s = gdr.gdr_causal_conv_silu(xd, wd, bd, want_state=True)
    ya, sa = gdr.gdr_causal_conv_silu(xd[:, :33].contiguous(), wd, bd, want_state=True)
    yb, sb = gdr.gdr_causal_conv_silu(xd[:, 33:].contiguous(), wd, bd, sa, want_state=True)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([ya, yb], 1), y) and torch.equal(sb, s)


def test_conv_full_layer_projection_sampled():
    """The q/k/v projections of the nanochat GDN layer packed as channels (2*16*128 + 16*128 =
    6144) over B=8, T=2048; the oracle checks 64 sampled channels of every token."""
    B, T, Ch = 8, 2048, 6144
    x, w, bias, _ = _conv_inputs(B, T, Ch, torch.bfloat16, seed=9)
    y, _ = gdr.gdr_causal_conv_silu(x.to(DEV), w.to(DEV), bias.to(DEV))
    torch.cuda.synchronize()
    ch = torch.from_numpy(np.random.default_rng(9).choice(Ch, 64, replace=False))
    y_ref, _ = prologue.causal_conv_silu(x[:, :, ch], w[ch], bias[ch])
    assert err(y[:, :, ch.to(DEV)], y_ref) <= TOL


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("D", [64, 128])
def test_rmsnorm_gated_matches_oracle(dtype, D):
    g = _gen(D)
    o = (3.0 * torch.randn(1000, D, generator=g)).to(dtype)
    z = torch.randn(1000, D, generator=g).to(dtype)
    wt = (1.0 + 0.1 * torch.randn(D, generator=g)).float()
    y = gdr.gdr_rmsnorm_gated(o.to(DEV), z.to(DEV), wt.to(DEV))
    torch.cuda.synchronize()
    assert err(y, prologue.rmsnorm_gated(o, z, wt)) <= TOL


def test_rmsnorm_gated_in_place():
    g = _gen(5)
    o = torch.randn(3, 7, 16, 128, generator=g).to(torch.bfloat16).to(DEV)
    z = torch.randn(3, 7, 16, 128, generator=g).to(torch.bfloat16).to(DEV)
    wt = torch.ones(128).to(DEV)
    ref = gdr.gdr_rmsnorm_gated(o, z, wt)
    y = gdr.gdr_rmsnorm_gated(o, z, wt, y=o)
    torch.cuda.synchronize()
    assert y.data_ptr() == o.data_ptr() and torch.equal(y, ref)
