"""Backward of the recurrence on the GPU (gdr_bwd) against the fp64 oracle backward.

The arithmetic is fp32 on both dtypes (bf16 inputs convert exactly), so every
gradient must match the fp64 adjoint within max|gpu - oracle| / rms(oracle) <= 1e-4.
Small cases compare every element; the nanochat GDN shape is checked on sampled
(batch row, value head) units.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_68_b200 as gdr
import oracle
from gated_delta_rule_68_b200.workloads import WORKLOADS, make_inputs
from tests.gpu_util import rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL = 1e-4
NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dh0")


def upstream(w, seed):
    gen = torch.Generator().manual_seed(seed)
    do = torch.randn((w.B, w.T, w.Hv, w.Dv), generator=gen)
    dhT = torch.randn((w.B, w.Hv, w.Dk, w.Dv), generator=gen) * 0.1
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    return do.to(dt).to(DEV), dhT.to(DEV)


def check(w, seed, with_dhT=True):
    inp = make_inputs(w, DEV)
    do, dhT = upstream(w, seed)
    dhT = dhT if with_dhT else None
    got = gdr.gdr_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], do, dhT)
    torch.cuda.synchronize()
    ref = oracle.backward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], do, dhT)
    for n in NAMES:
        err = rel_err(got[n], ref[n])
        assert err <= TOL, (w, n, err)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("T,D", [(1, 64), (9, 128), (100, 64), (130, 128)])
def test_small_cases(dtype, gate, T, D):
    w = WORKLOADS["gdn_bf16"].with_(B=2, T=T, Hk=2, Hv=4, Dk=D, Dv=D, gate=gate, dtype=dtype,
                                    g_mu=4.0 if gate == "channel" else 3.0, seed=800 + T)
    check(w, seed=T)


def test_without_h0_and_dhT():
    w = WORKLOADS["gdn_bf16"].with_(B=1, T=40, Hk=1, Hv=2, h0_std=0.0, seed=810)
    check(w, seed=3, with_dhT=False)


def test_empty_sequence_passes_dhT_to_dh0():
    w = WORKLOADS["gdn_bf16"].with_(B=2, T=0, Hk=1, Hv=2, seed=811)
    inp = make_inputs(w, DEV)
    do, dhT = upstream(w, 4)
    got = gdr.gdr_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], do, dhT)
    torch.cuda.synchronize()
    assert torch.equal(got["dh0"], dhT)


def test_nanochat_gdn_shape_sampled_units():
    """The bench shape (B=8, T=2048, H=16, d=128, bf16): gradients of sampled units against
    the oracle run on those units alone (Hk = Hv, so no key-head sums cross units)."""
    w = WORKLOADS["gdn_bf16"]
    inp = make_inputs(w, DEV)
    do, dhT = upstream(w, 5)
    got = gdr.gdr_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], do, dhT)
    torch.cuda.synchronize()
    for b, h in [(0, 0), (3, 9), (7, 15)]:
        sel = lambda x: x[b:b + 1, :, h:h + 1].cpu()
        ref = oracle.backward(sel(inp["q"]), sel(inp["k"]), sel(inp["v"]), sel(inp["g"]), sel(inp["beta"]),
                              inp["h0"][b:b + 1, h:h + 1].cpu(), sel(do), dhT[b:b + 1, h:h + 1].cpu())
        for n in NAMES:
            g = got[n][b:b + 1, :, h:h + 1] if n not in ("dh0",) else got[n][b:b + 1, h:h + 1]
            err = rel_err(g, ref[n])
            assert err <= TOL, (b, h, n, err)


def test_rejects_unsupported_and_small_workspace():
    w = WORKLOADS["gdn_bf16"].with_(B=1, T=16, Hk=1, Hv=1, seed=812)
    inp = make_inputs(w, DEV)
    do, dhT = upstream(w, 6)
    with pytest.raises(gdr.GdrError) as ei:
        gdr.gdr_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], do, dhT,
                    workspace=torch.empty(16, dtype=torch.uint8, device=DEV))
    assert ei.value.status == gdr.GDR_ERR_WORKSPACE


@pytest.mark.parametrize("T", [3, 7, 11])
def test_lengths_that_leave_a_partial_checkpoint_block(T):
    w = WORKLOADS["gdn_bf16"].with_(B=2, T=T, Hk=1, Hv=2, gate="channel", g_mu=2.0, seed=820 + T)
    check(w, seed=20 + T)


@pytest.mark.parametrize("Dk,Dv", [(64, 128), (128, 64)])
def test_rectangular_states(Dk, Dv):
    w = WORKLOADS["gdn_bf16"].with_(B=1, T=50, Hk=2, Hv=4, Dk=Dk, Dv=Dv, dtype="fp32", seed=830 + Dk)
    check(w, seed=7)


def test_strong_decay():
    """g = logsigmoid(N(-1, 1)): the state forgets within a few tokens, and a = exp(g)
    spans several orders of magnitude inside one checkpoint block."""
    w = WORKLOADS["gdn_bf16"].with_(B=2, T=70, Hk=2, Hv=2, g_mu=-1.0, seed=840)
    check(w, seed=8)


def sampled_unit_check(w, units, seed):
    """Gradients of the full-size workload against the oracle run on the sampled (b, key head)
    groups: each group carries every value head that shares its key head, so dq and dk
    (summed over those heads) are complete."""
    inp = make_inputs(w, DEV)
    do, dhT = upstream(w, seed)
    got = gdr.gdr_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], do, dhT)
    torch.cuda.synchronize()
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


def test_grouped_value_shape_sampled_units():
    """B=4, T=4096, Hk=16, Hv=48: three value heads per key head."""
    sampled_unit_check(WORKLOADS["gva_gdn_bf16"], [(0, 0), (3, 15)], seed=9)


def test_kda_shape_sampled_units():
    """B=2, T=16384, H=32, per-channel gate (a 17 GB checkpoint workspace)."""
    sampled_unit_check(WORKLOADS["kda_bf16"], [(0, 0), (1, 31)], seed=10)
