"""Edge cases of the scalar-gate tensor-core path (bf16 inputs, Dk = Dv = 128) against the
fp64 oracle, through the C ABI (needs a B200).

This path keeps the state map of each 64-token chunk in affine form and hands each
chunk from one warp group to another, so the cases here aim at chunk boundaries,
partial chunks, grouped value heads, more CTAs than one wave of SMs, in-place states,
decays strong enough to underflow the in-chunk gate products, and the two output dtypes.
Tolerances as in test_gpu_parity.py.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_68_b200 as gdr
import oracle
from gated_delta_rule_68_b200.workloads import WORKLOADS, make_inputs
from tests.gpu_util import TOL, oracle_units, rel_err, rel_err_excess, sample_units

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def run_fwd(inp, **kw):
    return gdr.gdr_fwd_chunked(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], **kw)


def check_all(w, out_dtype=None):
    """Every element against the oracle. A bf16-o call is also repeated with an fp32 o,
    which must meet the plain bound (no allowance for rounding o to bf16) and round to
    the bf16 o bit for bit; neither call may report an fp16 range error."""
    inp = make_inputs(w, DEV)
    _, r0 = gdr.gdr_fused_error_counts()
    o, hT = run_fwd(inp, **({} if out_dtype is None else {"out_dtype": out_dtype}))
    o32, hT32 = (o, hT) if out_dtype == torch.float32 else run_fwd(inp, out_dtype=torch.float32)
    torch.cuda.synchronize()
    _, r1 = gdr.gdr_fused_error_counts()
    assert r1 == r0
    o_ref, s_ref = oracle.recurrent(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    eo = rel_err(o, o_ref) if out_dtype == torch.float32 else rel_err_excess(o, o_ref, "bf16")
    eo32 = rel_err(o32, o_ref)
    es = rel_err(hT, s_ref)
    assert eo <= TOL["bf16"] and eo32 <= TOL["bf16"] and es <= TOL["bf16"], (w, eo, eo32, es)
    if out_dtype != torch.float32:
        assert torch.equal(o, o32.to(torch.bfloat16)) and torch.equal(hT, hT32)
    return inp, o, hT


@pytest.mark.parametrize("T", [1, 63, 64, 65, 128, 191])
def test_chunk_boundaries_grouped_heads(T):
    check_all(WORKLOADS["gva_gdn_bf16"].with_(B=2, T=T, Hk=2, Hv=6, seed=100 + T))


@pytest.mark.parametrize("Hk,Hv", [(1, 4), (4, 4), (2, 8)])
def test_head_groupings(Hk, Hv):
    check_all(WORKLOADS["gdn_bf16"].with_(B=2, T=150, Hk=Hk, Hv=Hv, seed=200 + Hk * 10 + Hv))


def test_fp32_output_and_bf16_output_agree():
    """The bf16-o launch is round-to-nearest bf16 of the fp32-o launch, bit for bit (both
    run the same arithmetic and round only at the store)."""
    w = WORKLOADS["gdn_bf16"].with_(B=2, T=200, Hk=2, Hv=4, seed=300)
    inp, o32, h32 = check_all(w, out_dtype=torch.float32)
    o16, h16 = run_fwd(inp)
    torch.cuda.synchronize()
    assert torch.equal(o16, o32.to(torch.bfloat16))
    assert torch.equal(h16, h32)


def test_more_ctas_than_two_waves_of_sms():
    """B * Hv = 320 units, one CTA each: more than two waves of 148 SMs."""
    w = WORKLOADS["gdn_bf16"].with_(B=20, T=130, Hk=4, Hv=16, seed=400)
    inp = make_inputs(w, DEV)
    o, hT = run_fwd(inp, out_dtype=torch.float32)
    torch.cuda.synchronize()
    units = sample_units(w.B, w.Hv, 8, seed=1)
    o_ref, s_ref = oracle_units(inp, units)
    for n, (b, h) in enumerate(units):
        assert rel_err(o[b, :, h], o_ref[n]) <= TOL["bf16"], (b, h)
        assert rel_err(hT[b, h], s_ref[n]) <= TOL["bf16"], (b, h)


def test_in_place_state():
    """hT may alias h0: the state is read at the start and written at the end."""
    w = WORKLOADS["gdn_bf16"].with_(B=2, T=100, Hk=2, Hv=2, seed=500)
    inp = make_inputs(w, DEV)
    o_ref, s_ref = oracle.recurrent(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    state = inp["h0"].clone()
    o, hT = gdr.gdr_fwd_chunked(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], state, hT=state,
                                out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert hT.data_ptr() == state.data_ptr()
    assert rel_err(o, o_ref) <= TOL["bf16"] and rel_err(state, s_ref) <= TOL["bf16"]


@pytest.mark.parametrize("g_mu", [-1.0, 8.0])
def test_strong_and_weak_decay(g_mu):
    """g = logsigmoid(N(mu, 1)): mu = -1 decays by about e^-80 over a chunk, so the
    in-chunk Gamma underflows; mu = 8 keeps the state nearly undamped over the sequence."""
    check_all(WORKLOADS["gdn_bf16"].with_(B=2, T=260, Hk=2, Hv=4, g_mu=g_mu, seed=600 + int(g_mu)),
              out_dtype=torch.float32)


def test_repeated_calls_are_bitwise_identical():
    w = WORKLOADS["gdn_bf16"].with_(B=3, T=333, Hk=2, Hv=6, seed=700)
    inp = make_inputs(w, DEV)
    o1, h1 = run_fwd(inp)
    o2, h2 = run_fwd(inp)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


def _growing_state_inputs(v_scale, T=320, seed=800):
    """g = 0 and beta = 1 with v scaled up (kept inside fp16's range): the state grows
    with the sequence, to about 7.5e4 by token 192 at v_scale = 2e4."""
    w = WORKLOADS["gdn_bf16"].with_(B=1, T=T, Hk=1, Hv=1, seed=seed)
    inp = make_inputs(w, DEV)
    inp["g"] = torch.zeros_like(inp["g"])
    inp["beta"] = torch.ones_like(inp["beta"])
    inp["v"] = (inp["v"].float() * v_scale).clamp(-6e4, 6e4).to(torch.bfloat16)
    return inp


def test_state_past_fp16_range_is_counted():
    """A state that outgrows fp16 (its copy is an operand of the next chunk's products)
    makes the call count one range error for its unit; the call itself still succeeds."""
    inp = _growing_state_inputs(2e4)
    _, before = gdr.gdr_fused_error_counts()
    run_fwd(inp)
    torch.cuda.synchronize()
    _, after = gdr.gdr_fused_error_counts()
    assert after == before + 1


def test_initial_state_past_fp16_range_is_counted():
    w = WORKLOADS["gdn_bf16"].with_(B=2, T=70, Hk=1, Hv=2, seed=801)
    inp = make_inputs(w, DEV)
    inp["h0"][1, 0, 3, 5] = 1e5   # one unit: batch row 1, value head 0
    _, before = gdr.gdr_fused_error_counts()
    run_fwd(inp)
    torch.cuda.synchronize()
    _, after = gdr.gdr_fused_error_counts()
    assert after == before + 1


def test_large_values_inside_fp16_range_are_not_counted():
    """The same growth with v 20 times smaller stays inside fp16 and meets the tolerance."""
    inp = _growing_state_inputs(1e3)
    _, before = gdr.gdr_fused_error_counts()
    o, hT = run_fwd(inp, out_dtype=torch.float32)
    torch.cuda.synchronize()
    _, after = gdr.gdr_fused_error_counts()
    assert after == before
    o_ref, s_ref = oracle.recurrent(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
    assert rel_err(o, o_ref) <= TOL["bf16"] and rel_err(hT, s_ref) <= TOL["bf16"]


# ------------------------------------------------------------------ per-channel gate (KDA)
@pytest.mark.parametrize("T", [1, 31, 32, 63, 64, 65, 191])
def test_channel_gate_chunk_boundaries_grouped_heads(T):
    """The per-channel gate on the tcgen05 kernel: partial chunks on both sides of the
    in-chunk reference row 31, three value heads per key head."""
    check_all(WORKLOADS["kda_bf16"].with_(B=2, T=T, Hk=2, Hv=6, seed=900 + T))


@pytest.mark.parametrize("g_mu", [2.0, 8.0])
def test_channel_gate_strong_and_weak_decay(g_mu):
    """g = logsigmoid(N(mu, 1)) per key channel: mu = 2 decays by about e^-4 per 32 tokens
    (the factors exp(+-(G - G_31)) stay inside fp16), mu = 8 barely decays at all."""
    check_all(WORKLOADS["kda_bf16"].with_(B=2, T=300, Hk=2, Hv=4, g_mu=g_mu, seed=950 + int(g_mu)),
              out_dtype=torch.float32)


def test_channel_gate_repeated_calls_are_bitwise_identical():
    w = WORKLOADS["kda_bf16"].with_(B=2, T=333, Hk=2, Hv=4, seed=990)
    inp = make_inputs(w, DEV)
    o1, h1 = run_fwd(inp)
    o2, h2 = run_fwd(inp)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


# ------------------------------------------------------------------ more units than SMs
@pytest.mark.parametrize("gate,T", [("scalar", 200), ("channel", 200), ("scalar", 130), ("scalar", 64)])
def test_units_spread_over_the_sms_equal_one_cta_per_unit(gate, T):
    """More (batch row, value head) units than SMs: with the workspace gdr_fwd_workspace_size
    asks for, the kernel spreads the units' chunks evenly over the SMs, cutting some units
    between two CTAs (the first part hands its state to the second through the workspace);
    with none it runs one CTA per unit. Both do each chunk's arithmetic the same way and the
    hand-off is an exact fp32 copy, so the results are equal bit for bit; sampled units also
    meet the oracle."""
    w = WORKLOADS["gdn_bf16"].with_(B=11, T=T, Hk=4, Hv=16, gate=gate,
                                    g_mu=4.0 if gate == "channel" else 3.0, seed=1100 + T)
    need = gdr.gdr_fwd_workspace_size(w.B, w.T, w.Hk, w.Hv, w.Dk, w.Dv, w.gate_mode, gdr.GDR_BF16)
    assert need > 0   # 176 units on 148 SMs
    inp = make_inputs(w, DEV)
    o1, h1 = run_fwd(inp, out_dtype=torch.float32)   # the binding passes the workspace
    none = torch.empty(0, dtype=torch.uint8, device=DEV)
    o2, h2 = run_fwd(inp, out_dtype=torch.float32, workspace=none)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(h1, h2)
    units = sample_units(w.B, w.Hv, 6, seed=3)
    o_ref, s_ref = oracle_units(inp, units)
    for n, (b, h) in enumerate(units):
        assert rel_err(o1[b, :, h], o_ref[n]) <= TOL["bf16"], (b, h)
        assert rel_err(h1[b, h], s_ref[n]) <= TOL["bf16"], (b, h)
