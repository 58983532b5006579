"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
symbol include/gdr.h declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_68_b200 as gdr
from gated_delta_rule_68_b200 import build as gbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    gbuild.build()
    return gdr.lib()


def declared_symbols():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"GDR_API\s+[\w\s\*]+?\b(gdr_\w+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_binding_exports():
    assert set(declared_symbols()) == set(gdr.EXPORTS)


def test_library_resolves_every_symbol_at_load(L):
    """Binding every symbol at load time (RTLD_NOW) fails on any reference the library leaves
    undefined, such as an internal function declared with the wrong linkage, which a lazy load
    would only reveal at its first call."""
    ctypes.CDLL(gdr.LIB_PATH, mode=os.RTLD_NOW | os.RTLD_LOCAL)


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
    assert L.gdr_version() >= 100


# Fake, never-dereferenced device addresses: every case below fails validation first.
A = 1 << 20          # 16- and 256-byte aligned
MIS = A + 8          # not 16-byte aligned


def fwd(L, q=A, k=A, v=A, g=A, beta=A, h0=0, o=A, hT=0, B=1, T=64, Hk=1, Hv=1, Dk=128, Dv=128,
        gate=0, dtype=0, ws=0, ws_bytes=0):
    vp = ctypes.c_void_p
    return L.gdr_fwd_chunked(vp(q), vp(k), vp(v), vp(g), vp(beta), vp(h0 or None), vp(o),
                             vp(hT or None), B, T, Hk, Hv, Dk, Dv, gate, dtype, vp(ws or None),
                             ws_bytes, None)


def dec(L, q=A, k=A, v=A, g=A, beta=A, state=A, o=A, B=1, Hk=1, Hv=1, Dk=128, Dv=128, gate=0, dtype=0):
    vp = ctypes.c_void_p
    return L.gdr_decode_step(vp(q), vp(k), vp(v), vp(g), vp(beta), vp(state), vp(o), B, Hk, Hv, Dk,
                             Dv, gate, dtype, None)


@pytest.mark.parametrize("kw,status", [
    (dict(Hk=2, Hv=3), gdr.GDR_ERR_INVALID_ARG),
    (dict(Dk=96), gdr.GDR_ERR_UNSUPPORTED),
    (dict(Dv=256), gdr.GDR_ERR_UNSUPPORTED),
    (dict(T=-1), gdr.GDR_ERR_INVALID_ARG),
    (dict(Hk=0), gdr.GDR_ERR_INVALID_ARG),
    (dict(gate=2), gdr.GDR_ERR_INVALID_ARG),
    (dict(dtype=7), gdr.GDR_ERR_INVALID_ARG),
    (dict(q=0), gdr.GDR_ERR_INVALID_ARG),
    (dict(beta=0), gdr.GDR_ERR_INVALID_ARG),
    (dict(o=0), gdr.GDR_ERR_INVALID_ARG),
    (dict(k=MIS), gdr.GDR_ERR_MISALIGNED),
    (dict(h0=MIS), gdr.GDR_ERR_MISALIGNED),
    (dict(ws=A + 16, ws_bytes=1 << 30), gdr.GDR_ERR_MISALIGNED),
    (dict(o=A, q=A), gdr.GDR_ERR_INVALID_ARG),       # o aliases q
])
def test_fwd_rejects(L, kw, status):
    base = dict(q=A, k=A + 4096, v=A + 8192, g=A + 12288, beta=A + 16384, o=A + 20480)
    base.update(kw)
    assert fwd(L, **base) == status
    assert len(gdr.gdr_last_error()) > 0


def test_fwd_rejects_small_workspace(L):
    need = L.gdr_fwd_workspace_size(2, 200, 1, 2, 128, 128, 0, gdr.GDR_FP32)
    assert need > 0
    st = fwd(L, k=A + 4096, v=A + 8192, g=A + 12288, beta=A + 16384, o=A + 20480, B=2, T=200, Hv=2,
             dtype=gdr.GDR_FP32, ws=A + 1 << 24, ws_bytes=need - 1)
    assert st == gdr.GDR_ERR_WORKSPACE
    st = fwd(L, k=A + 4096, v=A + 8192, g=A + 12288, beta=A + 16384, o=A + 20480, B=2, T=200, Hv=2,
             dtype=gdr.GDR_FP32)
    assert st == gdr.GDR_ERR_WORKSPACE


def test_empty_inputs_are_a_no_op(L):
    # No GPU work: B = 0 or T = 0 with no hT to write.
    assert fwd(L, q=0, k=0, v=0, g=0, beta=0, o=0, B=0) == gdr.GDR_OK
    assert fwd(L, q=0, k=0, v=0, g=0, beta=0, o=0, T=0) == gdr.GDR_OK
    assert dec(L, B=0, q=0) == gdr.GDR_OK


def test_workspace_size_rules(L):
    assert L.gdr_fwd_workspace_size(1, 64, 1, 3, 128, 128, 0, gdr.GDR_BF16) == 0   # tensor-core path
    assert L.gdr_fwd_workspace_size(1, 64, 1, 3, 64, 64, 0, gdr.GDR_BF16) > 0      # CUDA-core path
    assert L.gdr_fwd_workspace_size(1, 64, 2, 3, 128, 128, 0, 0) == 0    # invalid -> 0
    assert L.gdr_fwd_workspace_size(0, 64, 1, 1, 128, 128, 0, 0) == 0    # empty -> 0
    a = L.gdr_fwd_workspace_size(1, 64, 1, 1, 128, 128, 0, 1)
    b = L.gdr_fwd_workspace_size(1, 128, 1, 1, 128, 128, 0, 1)
    assert b >= a


@pytest.mark.parametrize("kw,status", [
    (dict(Hk=2, Hv=3), gdr.GDR_ERR_INVALID_ARG),
    (dict(Dk=32), gdr.GDR_ERR_UNSUPPORTED),
    (dict(state=0), gdr.GDR_ERR_INVALID_ARG),
    (dict(state=MIS), gdr.GDR_ERR_MISALIGNED),
    (dict(g=A + 2), gdr.GDR_ERR_MISALIGNED),
    (dict(q=A + 1), gdr.GDR_ERR_MISALIGNED),
    (dict(gate=5), gdr.GDR_ERR_INVALID_ARG),
])
def test_decode_rejects(L, kw, status):
    assert dec(L, **kw) == status


def conv(L, x=A, w=A, bias=0, sin=0, sout=0, y=A + (1 << 16), cu=0, B=1, T=16, Ch=64, width=4, dtype=0):
    vp = ctypes.c_void_p
    return L.gdr_causal_conv_silu(vp(x), vp(w), vp(bias or None), vp(sin or None), vp(sout or None), vp(y),
                                  vp(cu or None), B, T, Ch, width, dtype, None)


@pytest.mark.parametrize("kw,status", [
    (dict(width=3), gdr.GDR_ERR_UNSUPPORTED),
    (dict(Ch=12), gdr.GDR_ERR_UNSUPPORTED),
    (dict(dtype=2), gdr.GDR_ERR_INVALID_ARG),
    (dict(B=-1), gdr.GDR_ERR_INVALID_ARG),
    (dict(x=0), gdr.GDR_ERR_INVALID_ARG),
    (dict(y=A), gdr.GDR_ERR_INVALID_ARG),          # y aliases x
    (dict(x=MIS), gdr.GDR_ERR_MISALIGNED),
    (dict(w=MIS), gdr.GDR_ERR_MISALIGNED),
    (dict(cu=A + 2), gdr.GDR_ERR_MISALIGNED),
    (dict(cu=A, B=0), gdr.GDR_ERR_INVALID_ARG),    # packed tokens with no sequence
])
def test_conv_rejects_bad_arguments(L, kw, status):
    before = L.gdr_kernel_launches()
    assert conv(L, **kw) == status
    assert L.gdr_kernel_launches() == before


def norm(L, o=A, z=A, w=A, y=A, rows=4, D=128, eps=1e-5, dtype=0):
    vp = ctypes.c_void_p
    return L.gdr_rmsnorm_gated(vp(o), vp(z), vp(w), vp(y), rows, D, ctypes.c_float(eps), dtype, None)


@pytest.mark.parametrize("kw,status", [
    (dict(D=96), gdr.GDR_ERR_UNSUPPORTED),
    (dict(dtype=2), gdr.GDR_ERR_INVALID_ARG),
    (dict(rows=-1), gdr.GDR_ERR_INVALID_ARG),
    (dict(eps=-1.0), gdr.GDR_ERR_INVALID_ARG),
    (dict(z=0), gdr.GDR_ERR_INVALID_ARG),
    (dict(o=A + 1), gdr.GDR_ERR_MISALIGNED),
    (dict(w=A + 2), gdr.GDR_ERR_MISALIGNED),
])
def test_rmsnorm_gated_rejects_bad_arguments(L, kw, status):
    before = L.gdr_kernel_launches()
    assert norm(L, **kw) == status
    assert L.gdr_kernel_launches() == before


def test_empty_calls_launch_nothing(L):
    before = L.gdr_kernel_launches()
    assert norm(L, rows=0) == gdr.GDR_OK
    assert conv(L, T=0) == gdr.GDR_OK    # no tokens, no state_out: nothing to do
    assert L.gdr_kernel_launches() == before


def bwd(L, q=A, k=A + 4096, v=A + 8192, g=A + 12288, beta=A + 16384, h0=0, do=A + 20480, dhT=0,
        dq=A + 24576, dk=A + 28672, dv=A + 32768, dg=A + 36864, dbeta=A + 40960, dh0=A + 45056,
        B=1, T=16, Hk=1, Hv=1, Dk=128, Dv=128, gate=0, dtype=0, ws=0, ws_bytes=0, fn="gdr_bwd"):
    vp = ctypes.c_void_p
    ptrs = [q, k, v, g, beta, h0, do, dhT, dq, dk, dv, dg, dbeta, dh0]
    return getattr(L, fn)(*(vp(p or None) for p in ptrs), B, T, Hk, Hv, Dk, Dv, gate, dtype, vp(ws or None),
                          ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(Hk=2, Hv=3), gdr.GDR_ERR_INVALID_ARG),
    (dict(Dk=96), gdr.GDR_ERR_UNSUPPORTED),
    (dict(Dv=32), gdr.GDR_ERR_UNSUPPORTED),
    (dict(gate=3), gdr.GDR_ERR_INVALID_ARG),
    (dict(dtype=9), gdr.GDR_ERR_INVALID_ARG),
    (dict(dh0=0), gdr.GDR_ERR_INVALID_ARG),
    (dict(do=0), gdr.GDR_ERR_INVALID_ARG),
    (dict(dq=0), gdr.GDR_ERR_INVALID_ARG),
    (dict(dbeta=MIS), gdr.GDR_ERR_MISALIGNED),
    (dict(dhT=MIS), gdr.GDR_ERR_MISALIGNED),
    (dict(), gdr.GDR_ERR_WORKSPACE),                          # no workspace given
    (dict(ws=A + (1 << 24), ws_bytes=16), gdr.GDR_ERR_WORKSPACE),
])
def test_bwd_rejects(L, kw, status):
    assert bwd(L, **kw) == status
    assert len(gdr.gdr_last_error()) > 0


@pytest.mark.parametrize("kw,status", [
    (dict(gate=1), gdr.GDR_ERR_UNSUPPORTED),                 # the per-channel gate: gdr_bwd
    (dict(dtype=gdr.GDR_FP32), gdr.GDR_ERR_UNSUPPORTED),     # fp32 inputs: gdr_bwd
    (dict(Dk=64, Dv=64), gdr.GDR_ERR_UNSUPPORTED),
    (dict(Hk=2, Hv=3), gdr.GDR_ERR_INVALID_ARG),
    (dict(dh0=0), gdr.GDR_ERR_INVALID_ARG),
    (dict(do=0), gdr.GDR_ERR_INVALID_ARG),
    (dict(dk=0), gdr.GDR_ERR_INVALID_ARG),
    (dict(dg=MIS), gdr.GDR_ERR_MISALIGNED),
    (dict(), gdr.GDR_ERR_WORKSPACE),
    (dict(ws=A + (1 << 24), ws_bytes=16), gdr.GDR_ERR_WORKSPACE),
])
def test_bwd_chunked_rejects(L, kw, status):
    before = L.gdr_kernel_launches()
    assert bwd(L, fn="gdr_bwd_chunked", **kw) == status
    assert len(gdr.gdr_last_error()) > 0
    assert L.gdr_kernel_launches() == before


def test_bwd_chunked_workspace_size_rules(L):
    # S^T, P and the state gradient [128][128], Qh^T [128][64] and T [64][64], fp16, per chunk
    per_chunk = (3 * 128 * 128 + 128 * 64 + 64 * 64) * 2
    assert L.gdr_bwd_chunked_workspace_size(2, 130, 1, 3, 128, 128, 0, 0) == 2 * 3 * 3 * per_chunk
    assert L.gdr_bwd_chunked_workspace_size(1, 64, 2, 2, 128, 128, 0, 2) == 2 * per_chunk
    assert L.gdr_bwd_chunked_workspace_size(1, 64, 1, 1, 128, 128, 1, 0) == 0   # unsupported
    assert L.gdr_bwd_chunked_workspace_size(0, 64, 1, 1, 128, 128, 0, 0) == 0
    assert L.gdr_bwd_chunked_workspace_size(1, 0, 1, 1, 128, 128, 0, 0) == 0


def test_bwd_workspace_size_rules(L):
    # the state before every 4th token, fp32, per (batch row, value head)
    assert L.gdr_bwd_workspace_size(2, 10, 1, 3, 128, 64, 0, 0) == 2 * 3 * 3 * 128 * 64 * 4
    assert L.gdr_bwd_workspace_size(1, 8, 1, 1, 64, 64, 1, 1) == 2 * 64 * 64 * 4
    assert L.gdr_bwd_workspace_size(0, 8, 1, 1, 64, 64, 0, 0) == 0
    assert L.gdr_bwd_workspace_size(1, 0, 1, 1, 64, 64, 0, 0) == 0


def test_grid_limits_are_reported_before_launch(L):
    # the backward's (batch row, value head) axis and the CUDA-core path's batch axis
    assert bwd(L, B=70000, Hv=1, ws=A + (1 << 24), ws_bytes=1 << 62) == gdr.GDR_ERR_UNSUPPORTED
    assert "65535" in gdr.gdr_last_error()
    st = fwd(L, k=A + 4096, v=A + 8192, g=A + 12288, beta=A + 16384, o=A + 20480, B=70000, dtype=gdr.GDR_FP32,
             ws=A + (1 << 24), ws_bytes=1 << 62)
    assert st == gdr.GDR_ERR_UNSUPPORTED and "65535" in gdr.gdr_last_error()
