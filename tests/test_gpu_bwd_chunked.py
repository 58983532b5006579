"""The chunked tensor-core backward (gdr_bwd_chunked) against the fp64 oracle backward.

Its products take fp16 operands with fp32 accumulation, as the forward's do, so every
gradient is held to the bf16 workloads' bound: max|gpu - oracle| / rms(oracle) <= 2e-2
(an fp64 emulation of this arithmetic gives 1e-3 to 4e-3). Small and ragged cases
compare every element; the full-size shapes are checked on sampled units.
"""
import pytest
import torch

import gated_delta_rule_68_b200 as gdr
import oracle
from gated_delta_rule_68_b200.workloads import WORKLOADS, make_inputs
from tests.gpu_util import rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL = 2e-2
NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dh0")


def upstream(w, seed):
    gen = torch.Generator().manual_seed(seed)
    do = torch.randn((w.B, w.T, w.Hv, w.Dv), generator=gen)
    dhT = torch.randn((w.B, w.Hv, w.Dk, w.Dv), generator=gen) * 0.1
    return do.to(torch.bfloat16).to(DEV), dhT.to(DEV)


def run(w, seed, with_dhT=True):
    inp = make_inputs(w, DEV)
    do, dhT = upstream(w, seed)
    dhT = dhT if with_dhT else None
    got = gdr.gdr_bwd_chunked(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], do, dhT)
    torch.cuda.synchronize()
    return inp, do, dhT, got


def check(w, seed, with_dhT=True):
    before = gdr.gdr_fused_error_counts()
    inp, do, dhT, got = run(w, seed, with_dhT)
    assert gdr.gdr_fused_error_counts() == before, "wait timeouts or range errors counted"
    ref = oracle.backward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], do, dhT)
    for n in NAMES:
        err = rel_err(got[n], ref[n])
        assert err <= TOL, (w, n, err)


@pytest.mark.parametrize("T", [1, 17, 63, 64, 65, 130, 200])
def test_small_and_ragged_cases(T):
    """Grouped heads (two value heads per key head), h0 and dhT, chunk boundaries on both
    sides of 64 and a partial last chunk."""
    w = WORKLOADS["gdn_bf16"].with_(B=2, T=T, Hk=2, Hv=4, seed=900 + T)
    check(w, seed=T)


def test_without_h0_and_dhT():
    w = WORKLOADS["gdn_bf16"].with_(B=1, T=100, Hk=1, Hv=2, h0_std=0.0, seed=910)
    check(w, seed=3, with_dhT=False)


def test_strong_and_weak_decay():
    for mu, seed in ((-1.0, 911), (8.0, 912)):
        w = WORKLOADS["gdn_bf16"].with_(B=1, T=150, Hk=1, Hv=2, g_mu=mu, seed=seed)
        check(w, seed=seed)


def test_empty_sequence_passes_dhT_to_dh0():
    w = WORKLOADS["gdn_bf16"].with_(B=2, T=0, Hk=1, Hv=2, seed=913)
    inp = make_inputs(w, DEV)
    do, dhT = upstream(w, 4)
    got = gdr.gdr_bwd_chunked(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], do, dhT)
    torch.cuda.synchronize()
    assert torch.equal(got["dh0"], dhT)


def test_agrees_with_the_fp32_backward():
    """On a mid-size case both backward paths meet the oracle; here they are compared with
    each other at the same bound."""
    w = WORKLOADS["gdn_bf16"].with_(B=2, T=333, Hk=2, Hv=2, seed=914)
    inp, do, dhT, got = run(w, 5)
    ref = gdr.gdr_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], do, dhT)
    torch.cuda.synchronize()
    for n in NAMES:
        err = rel_err(got[n], ref[n].double().cpu().numpy())
        assert err <= TOL, (n, err)


def test_repeatable():
    """dv, dg, dbeta and dh0 are written once per element: bit for bit equal over calls;
    dq and dk are sums of atomics: equal to rounding."""
    w = WORKLOADS["gdn_bf16"].with_(B=2, T=256, Hk=1, Hv=2, seed=915)
    inp, do, dhT, a = run(w, 6)
    b = gdr.gdr_bwd_chunked(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], do, dhT)
    torch.cuda.synchronize()
    for n in ("dv", "dg", "dbeta", "dh0"):
        assert torch.equal(a[n], b[n]), n
    for n in ("dq", "dk"):
        assert rel_err(a[n], b[n].double().cpu().numpy()) <= 1e-5, n


def test_repeatable_with_one_value_head_per_key_head():
    """With Hv == Hk every dq and dk row has one writer (plain stores, no atomics): every
    gradient repeats bit for bit, ragged last chunk included."""
    w = WORKLOADS["gdn_bf16"].with_(B=2, T=200, Hk=2, Hv=2, seed=917)
    inp, do, dhT, a = run(w, 7)
    b = gdr.gdr_bwd_chunked(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], do, dhT)
    torch.cuda.synchronize()
    for n in NAMES:
        assert torch.equal(a[n], b[n]), n


def test_fp16_overflow_is_counted():
    """dout beyond the fp16 range (bf16 holds it) overflows the fp16 operands: the non-finite
    gradients are counted as range errors, one per reverse-scan unit (its dh0) and one per
    chunk work item, while the same inputs at unit scale count none."""
    w = WORKLOADS["gdn_bf16"].with_(B=1, T=128, Hk=1, Hv=1, seed=918)
    inp = make_inputs(w, DEV)
    do, dhT = upstream(w, 8)
    t0, r0 = gdr.gdr_fused_error_counts()
    gdr.gdr_bwd_chunked(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], do, dhT)
    torch.cuda.synchronize()
    assert gdr.gdr_fused_error_counts() == (t0, r0)
    big = (do.float() * 3.0e4).to(torch.bfloat16)   # |x| up to about 1.2e5 > 65504
    got = gdr.gdr_bwd_chunked(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], big, dhT)
    torch.cuda.synchronize()
    t1, r1 = gdr.gdr_fused_error_counts()
    assert t1 == t0
    assert r1 - r0 == 1 + 2, (r0, r1)   # the unit's scan and its two chunks
    assert not torch.isfinite(got["dh0"]).all()


def test_rejects_the_per_channel_gate():
    w = WORKLOADS["gdn_bf16"].with_(B=1, T=16, Hk=1, Hv=1, gate="channel", seed=916)
    inp = make_inputs(w, DEV)
    do, dhT = upstream(w, 7)
    with pytest.raises(gdr.GdrError) as ei:
        gdr.gdr_bwd_chunked(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], do, dhT)
    assert ei.value.status == gdr.GDR_ERR_UNSUPPORTED


def sampled_unit_check(w, units, seed):
    """Gradients of a full-size workload against the oracle on sampled (b, key head)
    groups, each with every value head sharing that key head (so dq and dk are complete)."""
    inp, do, dhT, got = run(w, seed)
    grp = w.Hv // w.Hk
    for b, hk in units:
        hv = slice(hk * grp, (hk + 1) * grp)
        sk = lambda x: x[b:b + 1, :, hk:hk + 1].cpu()
        sv = lambda x: x[b:b + 1, :, hv].cpu()
        ref = oracle.backward(sk(inp["q"]), sk(inp["k"]), sv(inp["v"]), sv(inp["g"]), sv(inp["beta"]),
                              inp["h0"][b:b + 1, hv].cpu(), sv(do), dhT[b:b + 1, hv].cpu())
        sel = {"dq": got["dq"][b:b + 1, :, hk:hk + 1], "dk": got["dk"][b:b + 1, :, hk:hk + 1],
               "dv": got["dv"][b:b + 1, :, hv], "dg": got["dg"][b:b + 1, :, hv],
               "dbeta": got["dbeta"][b:b + 1, :, hv], "dh0": got["dh0"][b:b + 1, hv]}
        for n in NAMES:
            err = rel_err(sel[n], ref[n])
            assert err <= TOL, (w.name, b, hk, n, err)


def test_nanochat_gdn_shape_sampled_units():
    """B=8, T=2048, H=16, d=128: the bench's backward workload."""
    sampled_unit_check(WORKLOADS["gdn_bwd_bf16"], [(0, 0), (7, 15)], seed=11)


def test_grouped_value_shape_sampled_units():
    """B=4, T=4096, Hk=16, Hv=48: three value heads per key head, 192 units."""
    sampled_unit_check(WORKLOADS["gva_gdn_bf16"], [(0, 0), (3, 15)], seed=12)
