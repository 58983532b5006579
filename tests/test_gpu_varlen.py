"""Packed variable-length sequences (gdr_fwd_chunked_varlen) on the GPU.

Each packed sequence must equal a gdr_fwd_chunked call on that sequence alone,
bit for bit, and the fp64 oracle within the bf16 bound: the recurrent state
restarts at every sequence start.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_68_b200 as gdr
import oracle
from gated_delta_rule_68_b200.workloads import WORKLOADS, make_inputs
from tests.gpu_util import TOL, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def packed_case(lengths, gate, Hk=2, Hv=4, seed=31):
    """One packed batch: each sequence drawn as its own B=1 workload, then concatenated."""
    seqs = [make_inputs(WORKLOADS["gdn_bf16"].with_(B=1, T=L, Hk=Hk, Hv=Hv, gate=gate,
                                                    g_mu=4.0 if gate == "channel" else 3.0, seed=seed + i), DEV)
            for i, L in enumerate(lengths)]
    cat = {n: torch.cat([s[n][0] for s in seqs], 0).contiguous() for n in ("q", "k", "v", "g", "beta")}
    cat["h0"] = torch.cat([s["h0"] for s in seqs], 0).contiguous()
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device=DEV)
    return seqs, cat, cu


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("lengths", [[64, 1, 130, 0, 200], [257, 63, 65]])
def test_packed_equals_separate_calls_and_oracle(gate, lengths):
    seqs, cat, cu = packed_case(lengths, gate)
    o, hT = gdr.gdr_fwd_chunked_varlen(cat["q"], cat["k"], cat["v"], cat["g"], cat["beta"], cu, cat["h0"],
                                       out_dtype=torch.float32)
    torch.cuda.synchronize()
    start = 0
    for i, (L, s) in enumerate(zip(lengths, seqs)):
        o1, h1 = gdr.gdr_fwd_chunked(s["q"], s["k"], s["v"], s["g"], s["beta"], s["h0"], out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(o[start:start + L], o1[0]), (gate, i)
        assert torch.equal(hT[i], h1[0]), (gate, i)
        if L > 0:
            o_ref, s_ref = oracle.recurrent(s["q"], s["k"], s["v"], s["g"], s["beta"], s["h0"])
            assert rel_err(o1[0], o_ref[0]) <= TOL["bf16"] and rel_err(h1[0], s_ref[0]) <= TOL["bf16"]
        start += L


def test_packed_rejects_unsupported_shapes():
    _, cat, cu = packed_case([70, 30], "scalar")
    with pytest.raises(gdr.GdrError) as ei:
        gdr.gdr_fwd_chunked_varlen(cat["q"].float(), cat["k"].float(), cat["v"].float(), cat["g"], cat["beta"],
                                   cu, cat["h0"])
    assert ei.value.status == gdr.GDR_ERR_UNSUPPORTED
