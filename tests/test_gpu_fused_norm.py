"""The fused kernel's in-kernel q/k L2 normalisation and gated output RMSNorm
(gdr_fwd_chunked_norm) against the oracle composition: l2norm, the fp64
recurrence, then rmsnorm_gated."""
import numpy as np
import pytest
import torch

import gated_delta_rule_68_b200 as gdr
import oracle
from gated_delta_rule_68_b200.workloads import WORKLOADS, make_inputs
from oracle import prologue
from tests.gpu_util import TOL, oracle_units, rel_err, sample_units

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def layer_inputs(w, device, scale_qk=True):
    """The workload's inputs, with q and k rows scaled by 0.5..4 (so that only an L2 norm
    brings them back to the unit keys the delta rule needs) when scale_qk, a gate
    z ~ N(0, 1) shaped like o, and a norm weight near 1."""
    inp = make_inputs(w, "cpu")
    gen = torch.Generator().manual_seed(w.seed + 500)
    for n in ("q", "k"):
        scale = 0.5 + 3.5 * torch.rand(inp[n].shape[:-1] + (1,), generator=gen)
        if scale_qk:
            inp[n] = (inp[n].float() * scale).to(inp[n].dtype)
    inp["z"] = torch.randn(inp["v"].shape, generator=gen).to(torch.bfloat16)
    inp["nw"] = (1.0 + 0.2 * torch.randn(inp["v"].shape[-1], generator=gen)).float()
    return {n: (None if t is None else t.to(device)) for n, t in inp.items()}


def reference(inp, l2, gated, eps=1e-5):
    q, k = inp["q"], inp["k"]
    if l2:
        q, k = prologue.l2norm(q), prologue.l2norm(k)
    o, hT = oracle.recurrent(q, k, inp["v"], inp["g"], inp["beta"], inp["h0"])
    if gated:
        o = prologue.rmsnorm_gated(o, inp["z"], inp["nw"], eps)
    return o, hT


def run(inp, l2, gated, out_dtype=torch.float32, cu=None):
    return gdr.gdr_fwd_chunked_norm(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                                    cu_seqlens=cu, qk_l2norm=l2, z=inp["z"] if gated else None,
                                    norm_weight=inp["nw"] if gated else None, out_dtype=out_dtype)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("l2,gated", [(True, False), (False, True), (True, True)])
@pytest.mark.parametrize("T,Hk,Hv", [(130, 2, 4), (64, 1, 1), (1, 1, 2)])
def test_fused_norms_match_oracle(gate, l2, gated, T, Hk, Hv):
    w = WORKLOADS["gdn_bf16"].with_(B=2, T=T, Hk=Hk, Hv=Hv, gate=gate,
                                    g_mu=4.0 if gate == "channel" else 3.0, seed=60 + T)
    inp = layer_inputs(w, DEV, scale_qk=l2)
    o, hT = run(inp, l2, gated)
    torch.cuda.synchronize()
    o_ref, s_ref = reference(inp, l2, gated)
    eo, es = rel_err(o, o_ref), rel_err(hT, s_ref)
    assert eo <= TOL["bf16"] and es <= TOL["bf16"], (eo, es)


def test_without_options_equals_the_plain_call():
    w = WORKLOADS["gdn_bf16"].with_(B=2, T=100, Hk=2, Hv=4, seed=70)
    inp = layer_inputs(w, DEV, scale_qk=False)
    o1, h1 = run(inp, False, False)
    o2, h2 = gdr.gdr_fwd_chunked(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"],
                                 out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


def test_l2norm_in_kernel_equals_normalised_inputs_within_rounding():
    """Normalising in the kernel or before it gives the same result up to the bf16 rounding of
    the normalised inputs (which only the second path has)."""
    w = WORKLOADS["gdn_bf16"].with_(B=2, T=200, Hk=2, Hv=2, seed=71)
    inp = layer_inputs(w, DEV)
    o1, h1 = run(inp, True, False)
    qn = torch.nn.functional.normalize(inp["q"].float(), dim=-1, eps=1e-12).to(torch.bfloat16)
    kn = torch.nn.functional.normalize(inp["k"].float(), dim=-1, eps=1e-12).to(torch.bfloat16)
    o2, h2 = gdr.gdr_fwd_chunked(qn, kn, inp["v"], inp["g"], inp["beta"], inp["h0"], out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert rel_err(o1, o2.double().cpu().numpy()) <= 2e-2 and rel_err(h1, h2.double().cpu().numpy()) <= 2e-2


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_fused_norms_packed_sequences(gate):
    lengths = [70, 1, 128, 0, 33]
    w = WORKLOADS["gdn_bf16"].with_(B=1, T=sum(lengths), Hk=2, Hv=4, gate=gate,
                                    g_mu=4.0 if gate == "channel" else 3.0, seed=72)
    inp = layer_inputs(w, "cpu")
    N = len(lengths)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    flat = {n: inp[n][0].contiguous() for n in ("q", "k", "v", "g", "beta", "z")}
    flat["nw"] = inp["nw"]
    flat["h0"] = torch.randn(N, 4, 128, 128, generator=torch.Generator().manual_seed(3)) * 0.02
    dflat = {n: t.to(DEV) for n, t in flat.items()}
    o, hT = run(dflat, True, True, cu=cu.to(DEV))
    torch.cuda.synchronize()
    for s in range(N):
        a, b = int(cu[s]), int(cu[s + 1])
        sub = {n: flat[n][a:b][None] for n in ("q", "k", "v", "g", "beta", "z")}
        sub["nw"], sub["h0"] = flat["nw"], flat["h0"][s:s + 1]
        o_ref, s_ref = reference(sub, True, True)
        if b > a:
            assert rel_err(o[a:b], o_ref[0]) <= TOL["bf16"]
        assert rel_err(hT[s], s_ref[0]) <= TOL["bf16"]


@pytest.mark.parametrize("name", ["gdn_bf16", "kda_bf16"])
def test_fused_norms_full_workload_sampled(name):
    """The full workload with both options and a bf16 o; sampled (b, h) units against the oracle."""
    w = WORKLOADS[name]
    inp = layer_inputs(w, "cpu")
    dinp = {n: (None if t is None else t.to(DEV)) for n, t in inp.items()}
    o, hT = run(dinp, True, True, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    units = sample_units(w.B, w.Hv, 3, seed=w.seed)
    normed = dict(inp)
    normed["q"] = torch.from_numpy(prologue.l2norm(inp["q"]))
    normed["k"] = torch.from_numpy(prologue.l2norm(inp["k"]))
    o_ref, s_ref = oracle_units(normed, units)
    for i, (b, h) in enumerate(units):
        og = prologue.rmsnorm_gated(o_ref[i], inp["z"][b, :, h], inp["nw"])
        assert rel_err(o[b, :, h].float(), og) <= TOL["bf16"] + 2.0 ** -8 * np.max(np.abs(og)) / np.sqrt(np.mean(og ** 2))
        assert rel_err(hT[b, h], s_ref[i]) <= TOL["bf16"]


def test_warp_level_kernel_mixed_launch_with_channel_gate():
    """The per-channel gate with the layer's options runs the warp-level kernel. With 160
    (batch row, value head) units on a 148-SM B200 its launch mixes whole units and units
    split over two CTAs by value columns; every unit is checked."""
    w = WORKLOADS["gdn_bf16"].with_(B=10, T=130, Hk=16, Hv=16, gate="channel", g_mu=4.0, seed=77)
    inp = layer_inputs(w, DEV, scale_qk=True)
    o, hT = run(inp, True, False)
    torch.cuda.synchronize()
    o_ref, s_ref = reference(inp, True, False)
    eo, es = rel_err(o, o_ref), rel_err(hT, s_ref)
    assert eo <= TOL["bf16"] and es <= TOL["bf16"], (eo, es)
