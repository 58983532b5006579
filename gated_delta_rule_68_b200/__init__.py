"""Python binding of libgdr, the B200 (sm_100a) gated delta-rule library.

The functions here carry the C ABI's names (include/gdr.h) and only marshal
arguments: they check dtypes and shapes, take raw device pointers from torch
tensors, pass the current CUDA stream, and turn a non-zero status into a
``GdrError``. Every step of the computation runs in the library's CUDA kernels;
there is no CPU fallback. If libgdr.so is missing the first call raises.

Layouts (row-major, contiguous): q,k [B,T,Hk,Dk]; v,o [B,T,Hv,Dv]; g [B,T,Hv]
(scalar gate) or [B,T,Hv,Dk] (per-channel gate) in fp32; beta [B,T,Hv] fp32;
h0, hT, state [B,Hv,Dk,Dv] fp32. Decode drops the T axis; packed sequences
(gdr_fwd_chunked_varlen) drop the B axis and add cu_seqlens.
"""
import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgdr.so")

GDR_OK, GDR_ERR_INVALID_ARG, GDR_ERR_UNSUPPORTED, GDR_ERR_MISALIGNED, GDR_ERR_WORKSPACE, GDR_ERR_CUDA = range(6)
GDR_GATE_SCALAR, GDR_GATE_CHANNEL = 0, 1
GDR_BF16, GDR_FP32, GDR_BF16_OUT_F32 = 0, 1, 2

# Every symbol include/gdr.h declares.
EXPORTS = ("gdr_version", "gdr_last_error", "gdr_kernel_launches", "gdr_fwd_workspace_size",
           "gdr_fwd_chunked", "gdr_decode_step", "gdr_fwd_chunked_noalloc", "gdr_fused_error_counts",
           "gdr_fwd_chunked_varlen", "gdr_causal_conv_silu", "gdr_rmsnorm_gated",
           "gdr_fwd_chunked_norm", "gdr_bwd_workspace_size", "gdr_bwd",
           "gdr_bwd_chunked_workspace_size", "gdr_bwd_chunked")

# Scratch held by gdr_fwd_chunked_noalloc (GDR_NOALLOC_SCRATCH_BYTES in include/gdr.h).
GDR_NOALLOC_SCRATCH_BYTES = 64 << 20

_lib = None


class GdrError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"libgdr status {status}: {message}")
        self.status = status


def lib():
    """Load libgdr.so (built in-tree by ``python -m gated_delta_rule_68_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m gated_delta_rule_68_b200.build` (no fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        vp, fp, i, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.gdr_version.restype = i
        L.gdr_version.argtypes = []
        L.gdr_last_error.restype = ctypes.c_char_p
        L.gdr_last_error.argtypes = []
        L.gdr_kernel_launches.restype = ctypes.c_ulonglong
        L.gdr_kernel_launches.argtypes = []
        L.gdr_fwd_workspace_size.restype = sz
        L.gdr_fwd_workspace_size.argtypes = [i] * 8
        L.gdr_fwd_chunked.restype = i
        L.gdr_fwd_chunked.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp] + [i] * 8 + [vp, sz, vp]
        L.gdr_decode_step.restype = i
        L.gdr_decode_step.argtypes = [vp, vp, vp, fp, fp, fp, vp] + [i] * 7 + [vp]
        L.gdr_fwd_chunked_noalloc.restype = i
        L.gdr_fwd_chunked_noalloc.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp] + [i] * 8 + [vp]
        L.gdr_fwd_chunked_varlen.restype = i
        L.gdr_fwd_chunked_varlen.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, vp] + [i] * 8 + [vp]
        L.gdr_fused_error_counts.restype = ctypes.c_uint
        L.gdr_fused_error_counts.argtypes = [vp, vp]
        L.gdr_causal_conv_silu.restype = i
        L.gdr_causal_conv_silu.argtypes = [vp, fp, fp, vp, vp, vp, vp] + [i] * 5 + [vp]
        L.gdr_fwd_chunked_norm.restype = i
        L.gdr_fwd_chunked_norm.argtypes = ([vp, vp, vp, fp, fp, fp, vp, fp, vp] + [i] * 9 + [vp, fp, ctypes.c_float, vp])
        L.gdr_rmsnorm_gated.restype = i
        L.gdr_rmsnorm_gated.argtypes = [vp, vp, fp, vp, ctypes.c_long, i, ctypes.c_float, i, vp]
        L.gdr_bwd_workspace_size.restype = sz
        L.gdr_bwd_workspace_size.argtypes = [i] * 8
        L.gdr_bwd.restype = i
        L.gdr_bwd.argtypes = [vp] * 14 + [i] * 8 + [vp, sz, vp]
        L.gdr_bwd_chunked_workspace_size.restype = sz
        L.gdr_bwd_chunked_workspace_size.argtypes = [i] * 8
        L.gdr_bwd_chunked.restype = i
        L.gdr_bwd_chunked.argtypes = [vp] * 14 + [i] * 8 + [vp, sz, vp]
        _lib = L
    return _lib


def gdr_version() -> int:
    return int(lib().gdr_version())


def gdr_last_error() -> str:
    return lib().gdr_last_error().decode()


def gdr_kernel_launches() -> int:
    return int(lib().gdr_kernel_launches())


def gdr_fused_error_counts():
    """(load_timeouts, range_errors) of the tensor-core chunked forward and backward kernels on the
    current device; see include/gdr.h."""
    t, r = ctypes.c_uint(0), ctypes.c_uint(0)
    lib().gdr_fused_error_counts(ctypes.byref(t), ctypes.byref(r))
    return int(t.value), int(r.value)


def _check(status):
    if status != GDR_OK:
        raise GdrError(status, gdr_last_error())


def _dtype_code(t, out_dtype):
    if t.dtype == torch.bfloat16:
        if out_dtype in (None, torch.bfloat16):
            return GDR_BF16, torch.bfloat16
        if out_dtype == torch.float32:
            return GDR_BF16_OUT_F32, torch.float32
    elif t.dtype == torch.float32 and out_dtype in (None, torch.float32):
        return GDR_FP32, torch.float32
    raise TypeError(f"unsupported q/k/v dtype {t.dtype} with output dtype {out_dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype=None, shape=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def gdr_fwd_workspace_size(B, T, Hk, Hv, Dk, Dv, gate_mode, dtype) -> int:
    return int(lib().gdr_fwd_workspace_size(B, T, Hk, Hv, Dk, Dv, gate_mode, dtype))


def gdr_bwd_workspace_size(B, T, Hk, Hv, Dk, Dv, gate_mode, dtype) -> int:
    return int(lib().gdr_bwd_workspace_size(B, T, Hk, Hv, Dk, Dv, gate_mode, dtype))


def gdr_bwd_chunked_workspace_size(B, T, Hk, Hv, Dk, Dv, gate_mode, dtype) -> int:
    return int(lib().gdr_bwd_chunked_workspace_size(B, T, Hk, Hv, Dk, Dv, gate_mode, dtype))


def gdr_bwd(q, k, v, g, beta, h0, dout, dhT=None, *, workspace=None, stream=None, out=None):
    """Backward of the recurrence: fp32 gradients of sum(dout * o) + sum(dhT * hT) with respect
    to q, k, v, g, beta and h0, as a dict (dq, dk, dv, dg, dbeta, dh0). dout has q's dtype.
    out, if given, is such a dict of preallocated fp32 tensors to write into."""
    return _bwd_call("gdr_bwd", gdr_bwd_workspace_size, q, k, v, g, beta, h0, dout, dhT, workspace, stream, out)


def gdr_bwd_chunked(q, k, v, g, beta, h0, dout, dhT=None, *, workspace=None, stream=None, out=None):
    """The same gradients by the tensor-core chunked backward (scalar gate, bf16 inputs,
    Dk = Dv = 128; fp16 operands, so of the forward's accuracy rather than fp32)."""
    return _bwd_call("gdr_bwd_chunked", gdr_bwd_chunked_workspace_size, q, k, v, g, beta, h0, dout, dhT,
                     workspace, stream, out)


def _bwd_call(fn, ws_size, q, k, v, g, beta, h0, dout, dhT, workspace, stream, out):
    B, T, Hk, Dk = q.shape
    Hv, Dv = v.shape[2], v.shape[3]
    dt, _ = _dtype_code(q, None)
    gate_mode = GDR_GATE_CHANNEL if g.dim() == 4 else GDR_GATE_SCALAR
    _need(q, "q", q.dtype)
    _need(k, "k", q.dtype, q.shape)
    _need(v, "v", q.dtype, (B, T, Hv, Dv))
    _need(dout, "dout", q.dtype, (B, T, Hv, Dv))
    _need(g, "g", torch.float32, (B, T, Hv) if gate_mode == 0 else (B, T, Hv, Dk))
    _need(beta, "beta", torch.float32, (B, T, Hv))
    for t, n in ((h0, "h0"), (dhT, "dhT")):
        if t is not None:
            _need(t, n, torch.float32, (B, Hv, Dk, Dv))
    f32 = dict(dtype=torch.float32, device=q.device)
    shapes = {"dq": (B, T, Hk, Dk), "dk": (B, T, Hk, Dk), "dv": (B, T, Hv, Dv), "dg": tuple(g.shape),
              "dbeta": (B, T, Hv), "dh0": (B, Hv, Dk, Dv)}
    if out is None:
        out = {n: torch.empty(s, **f32) for n, s in shapes.items()}
    for n, s in shapes.items():
        _need(out[n], n, torch.float32, s)
    need = ws_size(B, T, Hk, Hv, Dk, Dv, gate_mode, dt)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(getattr(lib(), fn)(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(dout), _ptr(dhT),
                         *(_ptr(out[n]) for n in ("dq", "dk", "dv", "dg", "dbeta", "dh0")),
                         B, T, Hk, Hv, Dk, Dv, gate_mode, dt, _ptr(workspace), ws_bytes, _stream(stream)))
    return out


def gdr_fwd_chunked(q, k, v, g, beta, h0=None, *, o=None, hT=None, want_hT=True,
                    workspace=None, stream=None, out_dtype=None):
    """Chunked forward. Returns (o, hT); hT is None when want_hT is False and no hT is given.
    o has q's dtype unless out_dtype=torch.float32 is asked for with bf16 inputs."""
    B, T, Hk, Dk = q.shape
    Hv, Dv = v.shape[2], v.shape[3]
    if o is not None and out_dtype is None:
        out_dtype = o.dtype
    dt, odt = _dtype_code(q, out_dtype)
    gate_mode = GDR_GATE_CHANNEL if g.dim() == 4 else GDR_GATE_SCALAR
    _need(q, "q", q.dtype)
    _need(k, "k", q.dtype, q.shape)
    _need(v, "v", q.dtype, (B, T, Hv, Dv))
    _need(g, "g", torch.float32, (B, T, Hv) if gate_mode == 0 else (B, T, Hv, Dk))
    _need(beta, "beta", torch.float32, (B, T, Hv))
    if h0 is not None:
        _need(h0, "h0", torch.float32, (B, Hv, Dk, Dv))
    if o is None:
        o = torch.empty((B, T, Hv, Dv), dtype=odt, device=q.device)
    _need(o, "o", odt, (B, T, Hv, Dv))
    if hT is None and want_hT:
        hT = torch.empty((B, Hv, Dk, Dv), dtype=torch.float32, device=q.device)
    if hT is not None:
        _need(hT, "hT", torch.float32, (B, Hv, Dk, Dv))
    need = gdr_fwd_workspace_size(B, T, Hk, Hv, Dk, Dv, gate_mode, dt)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().gdr_fwd_chunked(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(o),
                                 _ptr(hT), B, T, Hk, Hv, Dk, Dv, gate_mode, dt, _ptr(workspace),
                                 ws_bytes, _stream(stream)))
    return o, hT


def gdr_fwd_chunked_varlen(q, k, v, g, beta, cu_seqlens, h0=None, *, o=None, hT=None, want_hT=True,
                           stream=None, out_dtype=None):
    """Chunked forward over packed sequences: q, k [T_total, Hk, Dk], v [T_total, Hv, Dv],
    g [T_total, Hv] or [T_total, Hv, Dk], beta [T_total, Hv], cu_seqlens int32 [N + 1] on the
    device. Returns (o [T_total, Hv, Dv], hT [N, Hv, Dk, Dv] or None)."""
    T_total, Hk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    N = cu_seqlens.numel() - 1
    if o is not None and out_dtype is None:
        out_dtype = o.dtype
    dt, odt = _dtype_code(q, out_dtype)
    gate_mode = GDR_GATE_CHANNEL if g.dim() == 3 else GDR_GATE_SCALAR
    _need(q, "q", q.dtype)
    _need(k, "k", q.dtype, q.shape)
    _need(v, "v", q.dtype, (T_total, Hv, Dv))
    _need(g, "g", torch.float32, (T_total, Hv) if gate_mode == 0 else (T_total, Hv, Dk))
    _need(beta, "beta", torch.float32, (T_total, Hv))
    _need(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,))
    if h0 is not None:
        _need(h0, "h0", torch.float32, (N, Hv, Dk, Dv))
    if o is None:
        o = torch.empty((T_total, Hv, Dv), dtype=odt, device=q.device)
    _need(o, "o", odt, (T_total, Hv, Dv))
    if hT is None and want_hT:
        hT = torch.empty((N, Hv, Dk, Dv), dtype=torch.float32, device=q.device)
    if hT is not None:
        _need(hT, "hT", torch.float32, (N, Hv, Dk, Dv))
    _check(lib().gdr_fwd_chunked_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(o),
                                        _ptr(hT), _ptr(cu_seqlens), N, T_total, Hk, Hv, Dk, Dv, gate_mode, dt,
                                        _stream(stream)))
    return o, hT


def gdr_decode_step(q, k, v, g, beta, state, *, o=None, stream=None, out_dtype=None):
    """One decode step; ``state`` is updated in place. Returns o [B,Hv,Dv]."""
    B, Hk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    if o is not None and out_dtype is None:
        out_dtype = o.dtype
    dt, odt = _dtype_code(q, out_dtype)
    gate_mode = GDR_GATE_CHANNEL if g.dim() == 3 else GDR_GATE_SCALAR
    _need(q, "q", q.dtype)
    _need(k, "k", q.dtype, q.shape)
    _need(v, "v", q.dtype, (B, Hv, Dv))
    _need(g, "g", torch.float32, (B, Hv) if gate_mode == 0 else (B, Hv, Dk))
    _need(beta, "beta", torch.float32, (B, Hv))
    _need(state, "state", torch.float32, (B, Hv, Dk, Dv))
    if o is None:
        o = torch.empty((B, Hv, Dv), dtype=odt, device=q.device)
    _need(o, "o", odt, (B, Hv, Dv))
    _check(lib().gdr_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), _ptr(o),
                                 B, Hk, Hv, Dk, Dv, gate_mode, dt, _stream(stream)))
    return o


def gdr_fwd_chunked_noalloc(q, k, v, g, beta, h0=None, *, o=None, hT=None, want_hT=True, stream=None,
                            out_dtype=None):
    """Chunked forward on the library's own fixed scratch (no workspace, no allocation by the
    library). For callers that must not allocate device memory; see include/gdr.h. Outputs o
    and hT are allocated here by torch only when the caller does not pass them."""
    B, T, Hk, Dk = q.shape
    Hv, Dv = v.shape[2], v.shape[3]
    if o is not None and out_dtype is None:
        out_dtype = o.dtype
    dt, odt = _dtype_code(q, out_dtype)
    gate_mode = GDR_GATE_CHANNEL if g.dim() == 4 else GDR_GATE_SCALAR
    _need(q, "q", q.dtype)
    _need(k, "k", q.dtype, q.shape)
    _need(v, "v", q.dtype, (B, T, Hv, Dv))
    _need(g, "g", torch.float32, (B, T, Hv) if gate_mode == 0 else (B, T, Hv, Dk))
    _need(beta, "beta", torch.float32, (B, T, Hv))
    if h0 is not None:
        _need(h0, "h0", torch.float32, (B, Hv, Dk, Dv))
    if o is None:
        o = torch.empty((B, T, Hv, Dv), dtype=odt, device=q.device)
    _need(o, "o", odt, (B, T, Hv, Dv))
    if hT is None and want_hT:
        hT = torch.empty((B, Hv, Dk, Dv), dtype=torch.float32, device=q.device)
    if hT is not None:
        _need(hT, "hT", torch.float32, (B, Hv, Dk, Dv))
    _check(lib().gdr_fwd_chunked_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                                         _ptr(o), _ptr(hT), B, T, Hk, Hv, Dk, Dv, gate_mode, dt,
                                         _stream(stream)))
    return o, hT


def gdr_causal_conv_silu(x, w, bias=None, state_in=None, cu_seqlens=None, *, y=None, state_out=None,
                         want_state=False, stream=None):
    """Short causal convolution (4 taps) + SiLU; see include/gdr.h. x: [B, T, Ch] (or [T, Ch]
    with cu_seqlens int32 [N + 1]); w: [Ch, 4] fp32; bias: [Ch] fp32; state_in: [B or N, Ch, 3]
    in x's dtype. Returns (y, state_out or None)."""
    if x.dtype == torch.bfloat16:
        dt = GDR_BF16
    elif x.dtype == torch.float32:
        dt = GDR_FP32
    else:
        raise TypeError(f"unsupported x dtype {x.dtype}")
    if cu_seqlens is None:
        B, T, Ch = x.shape
    else:
        T, Ch = x.shape
        B = cu_seqlens.numel() - 1
        _need(cu_seqlens, "cu_seqlens", torch.int32, (B + 1,))
    _need(x, "x", x.dtype)
    _need(w, "w", torch.float32, (Ch, w.shape[1]))
    if bias is not None:
        _need(bias, "bias", torch.float32, (Ch,))
    if state_in is not None:
        _need(state_in, "state_in", x.dtype, (B, Ch, 3))
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", x.dtype, tuple(x.shape))
    if state_out is None and want_state:
        state_out = torch.empty((B, Ch, 3), dtype=x.dtype, device=x.device)
    if state_out is not None:
        _need(state_out, "state_out", x.dtype, (B, Ch, 3))
    _check(lib().gdr_causal_conv_silu(_ptr(x), _ptr(w), _ptr(bias), _ptr(state_in), _ptr(state_out), _ptr(y),
                                      _ptr(cu_seqlens), B, T, Ch, w.shape[1], dt, _stream(stream)))
    return y, state_out


def gdr_rmsnorm_gated(o, z, weight, eps=1e-5, *, y=None, stream=None):
    """y = o / sqrt(mean(o^2) + eps) * weight * SiLU(z) over the last axis (64 or 128);
    o, z, y in one dtype (bf16 or fp32); y may be o (in place)."""
    if o.dtype == torch.bfloat16:
        dt = GDR_BF16
    elif o.dtype == torch.float32:
        dt = GDR_FP32
    else:
        raise TypeError(f"unsupported o dtype {o.dtype}")
    D = o.shape[-1]
    _need(o, "o", o.dtype)
    _need(z, "z", o.dtype, tuple(o.shape))
    _need(weight, "weight", torch.float32, (D,))
    if y is None:
        y = torch.empty_like(o)
    _need(y, "y", o.dtype, tuple(o.shape))
    rows = o.numel() // D if D else 0
    _check(lib().gdr_rmsnorm_gated(_ptr(o), _ptr(z), _ptr(weight), _ptr(y), rows, D, float(eps), dt,
                                   _stream(stream)))
    return y


def gdr_fwd_chunked_norm(q, k, v, g, beta, h0=None, *, cu_seqlens=None, qk_l2norm=False, z=None,
                         norm_weight=None, norm_eps=1e-5, o=None, hT=None, want_hT=True, stream=None,
                         out_dtype=None):
    """Chunked forward with in-kernel q/k L2 normalisation and/or the gated output RMSNorm
    (see include/gdr.h). Shapes as gdr_fwd_chunked, or as gdr_fwd_chunked_varlen when
    cu_seqlens is given; z like o (bf16), norm_weight [Dv] fp32. Returns (o, hT)."""
    packed = cu_seqlens is not None
    if packed:
        T, Hk, Dk = q.shape
        Hv, Dv = v.shape[1], v.shape[2]
        B = cu_seqlens.numel() - 1
        tok = (T,)
        _need(cu_seqlens, "cu_seqlens", torch.int32, (B + 1,))
    else:
        B, T, Hk, Dk = q.shape
        Hv, Dv = v.shape[2], v.shape[3]
        tok = (B, T)
    if o is not None and out_dtype is None:
        out_dtype = o.dtype
    dt, odt = _dtype_code(q, out_dtype)
    gate_mode = GDR_GATE_CHANNEL if g.dim() == len(tok) + 2 else GDR_GATE_SCALAR
    _need(q, "q", q.dtype)
    _need(k, "k", q.dtype, q.shape)
    _need(v, "v", q.dtype, tok + (Hv, Dv))
    _need(g, "g", torch.float32, tok + ((Hv,) if gate_mode == 0 else (Hv, Dk)))
    _need(beta, "beta", torch.float32, tok + (Hv,))
    if h0 is not None:
        _need(h0, "h0", torch.float32, (B, Hv, Dk, Dv))
    if z is not None:
        _need(z, "z", torch.bfloat16, tok + (Hv, Dv))
        _need(norm_weight, "norm_weight", torch.float32, (Dv,))
    if o is None:
        o = torch.empty(tok + (Hv, Dv), dtype=odt, device=q.device)
    _need(o, "o", odt, tok + (Hv, Dv))
    if hT is None and want_hT:
        hT = torch.empty((B, Hv, Dk, Dv), dtype=torch.float32, device=q.device)
    if hT is not None:
        _need(hT, "hT", torch.float32, (B, Hv, Dk, Dv))
    _check(lib().gdr_fwd_chunked_norm(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(o),
                                      _ptr(hT), _ptr(cu_seqlens), B, T, Hk, Hv, Dk, Dv, gate_mode, dt,
                                      int(bool(qk_l2norm)), _ptr(z), _ptr(norm_weight), float(norm_eps),
                                      _stream(stream)))
    return o, hT
