"""gdr_fwd_chunked_noalloc: the chunked forward for callers that cannot allocate device
memory (engines that own all device memory in their own pool, serving loops that may not
allocate after start-up). It runs on a fixed scratch array inside the library.

Called through the C ABI with raw pointers and checked against gdr_fwd_chunked (which
takes a caller-allocated workspace) on two calls in a row, so the second call also shows
that scratch contents left by the first do not leak into its results. Both entry points
run the same kernels on the same inputs, so the results must agree bit for bit. The
shapes are ones whose forward needs scratch (fp32 inputs, Dk or Dv of 64, rectangular
states: the CUDA-core kernels), plus one that needs none. This file is named to be
collected last.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_68_b200 as gdr
from gated_delta_rule_68_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def noalloc_call(inp, o, hT, dtype_code):
    q, k, v, g, beta, h0 = (inp[n] for n in ("q", "k", "v", "g", "beta", "h0"))
    B, T, Hk, Dk = q.shape
    Hv, Dv = v.shape[2], v.shape[3]
    gate = gdr.GDR_GATE_CHANNEL if g.dim() == 4 else gdr.GDR_GATE_SCALAR
    vp = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return gdr.lib().gdr_fwd_chunked_noalloc(vp(q), vp(k), vp(v), vp(g), vp(beta), vp(h0), vp(o), vp(hT),
                                             B, T, Hk, Hv, Dk, Dv, gate, dtype_code, stream)


# (dtype, gate, Dk, Dv, needs scratch)
CASES = [("fp32", "scalar", 64, 64, True), ("fp32", "channel", 128, 64, True),
         ("bf16", "channel", 64, 128, True), ("bf16", "scalar", 128, 128, False)]


@pytest.mark.parametrize("dtype,gate,Dk,Dv,uses_scratch", CASES)
def test_noalloc_matches_fwd_chunked_on_two_calls(dtype, gate, Dk, Dv, uses_scratch):
    code = gdr.GDR_BF16 if dtype == "bf16" else gdr.GDR_FP32
    gmode = gdr.GDR_GATE_CHANNEL if gate == "channel" else gdr.GDR_GATE_SCALAR
    base = WORKLOADS["gva_gdn_bf16"].with_(B=2, T=200, Hk=2, Hv=4, Dk=Dk, Dv=Dv, dtype=dtype, gate=gate,
                                           g_mu=4.0 if gate == "channel" else 3.0)
    for call, seed in enumerate((41, 42)):
        w = base.with_(seed=seed, T=200 if call == 0 else 137)
        need = gdr.gdr_fwd_workspace_size(w.B, w.T, w.Hk, w.Hv, Dk, Dv, gmode, code)
        assert (need > 0) == uses_scratch and need <= gdr.GDR_NOALLOC_SCRATCH_BYTES, need
        inp = make_inputs(w, DEV)
        o_ref, s_ref = gdr.gdr_fwd_chunked(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
        o = torch.full_like(o_ref, float("nan"))
        hT = torch.full_like(s_ref, float("nan"))
        st = noalloc_call(inp, o, hT, code)
        assert st == gdr.GDR_OK, gdr.gdr_last_error()
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref), (call, dtype, gate, Dk, Dv)
        assert torch.equal(hT, s_ref), (call, dtype, gate, Dk, Dv)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # fp32 inputs (the CUDA-core path), B=2, T=16384, 32 heads: a workspace far beyond the scratch.
    w = WORKLOADS["kda_bf16"].with_(dtype="fp32")
    need = gdr.gdr_fwd_workspace_size(w.B, w.T, w.Hk, w.Hv, w.Dk, w.Dv, gdr.GDR_GATE_CHANNEL, gdr.GDR_FP32)
    assert need > gdr.GDR_NOALLOC_SCRATCH_BYTES
    inp = make_inputs(w.with_(T=64), DEV)   # real buffers; the call must not touch them
    o = torch.empty((w.B, 64, w.Hv, w.Dv), dtype=torch.float32, device=DEV)
    vp = lambda t: ctypes.c_void_p(t.data_ptr())
    st = gdr.lib().gdr_fwd_chunked_noalloc(vp(inp["q"]), vp(inp["k"]), vp(inp["v"]), vp(inp["g"]),
                                           vp(inp["beta"]), None, vp(o), None, w.B, w.T, w.Hk, w.Hv,
                                           w.Dk, w.Dv, gdr.GDR_GATE_CHANNEL, gdr.GDR_FP32, None)
    assert st == gdr.GDR_ERR_WORKSPACE
    assert "scratch" in gdr.gdr_last_error()
