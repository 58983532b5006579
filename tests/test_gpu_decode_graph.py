"""Decode steps captured in a CUDA graph: the entry point allocates nothing and does not
synchronise, so a serving loop can capture it. A replay of the captured steps gives the eager
loop's state and outputs bit for bit, and a second replay from the same starting state
repeats them."""
import pytest
import torch

import gated_delta_rule_68_b200 as gdr
from gated_delta_rule_68_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_graph_replay_matches_eager(gate):
    w = WORKLOADS["decode_bf16"].with_(B=4, T=12, Hk=2, Hv=4, gate=gate, g_mu=4.0 if gate == "channel" else 3.0,
                                       seed=950)
    d = make_inputs(w, DEV)
    st_e = d["h0"].clone()
    o_e = torch.stack([gdr.gdr_decode_step(d["q"][s], d["k"][s], d["v"][s], d["g"][s], d["beta"][s], st_e)
                       for s in range(w.T)])
    torch.cuda.synchronize()

    st_g = d["h0"].clone()
    o_g = torch.empty_like(o_e)
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap):
        for s in range(w.T):
            gdr.gdr_decode_step(d["q"][s], d["k"][s], d["v"][s], d["g"][s], d["beta"][s], st_g, o=o_g[s], stream=cap)
    for _ in range(2):
        st_g.copy_(d["h0"])
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(st_g, st_e)
        assert torch.equal(o_g, o_e)
