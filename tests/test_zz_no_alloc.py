"""gdr_fwd_chunked_noalloc: the chunked forward for callers that cannot allocate device
memory (engines that own all device memory in their own pool, serving loops that may not
allocate after start-up). It runs on a fixed scratch array inside the library.

Called through the C ABI with raw pointers and checked against gdr_fwd_chunked (which
takes a caller-allocated workspace) on two calls in a row, so the second call also shows
that scratch contents left by the first do not leak into its results. This file is named
to be collected last.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_68_b200 as gdr
from gated_delta_rule_68_b200.workloads import WORKLOADS, make_inputs
from tests.gpu_util import TOL, rel_err, rel_err_excess

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


@pytest.mark.parametrize("dtype,gate", [("bf16", "scalar"), ("bf16", "channel"), ("fp32", "scalar")])
def test_noalloc_matches_fwd_chunked_on_two_calls(dtype, gate):
    code = gdr.GDR_BF16 if dtype == "bf16" else gdr.GDR_FP32
    base = WORKLOADS["gva_gdn_bf16"].with_(B=2, T=200, Hk=2, Hv=4, dtype=dtype, gate=gate,
                                           g_mu=4.0 if gate == "channel" else 3.0)
    for call, seed in enumerate((41, 42)):
        w = base.with_(seed=seed, T=200 if call == 0 else 137)
        inp = make_inputs(w, DEV)
        o_ref, s_ref = gdr.gdr_fwd_chunked(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"])
        o = torch.full_like(o_ref, float("nan"))
        hT = torch.full_like(s_ref, float("nan"))
        st = noalloc_call(inp, o, hT, code)
        assert st == gdr.GDR_OK, gdr.gdr_last_error()
        torch.cuda.synchronize()
        ref_o = o_ref.double().cpu().numpy()
        assert rel_err_excess(o, ref_o, dtype) <= TOL[dtype], (call, dtype, gate)
        assert rel_err(hT, s_ref.double().cpu().numpy()) <= TOL[dtype], (call, dtype, gate)


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
