"""fp64 CPU oracle for the gated delta rule.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The CUDA library
(``gated_delta_rule_68_b200``) never imports it and shares no code with it.

Functions:

``recurrent``  the plain definition: the token-by-token recurrence in fp64
               (C, ``gdr_oracle.c``), following NextTransformer "Source notes",
               section "Linear attention" (rows gdn, kda, deltanet) and
               "Backend and numerical limits" (scale 1, FP64 recurrent reference).
``chunked``    the exact chunkwise (UT/WY) form in fp64 numpy
               (``chunked.py``), the algebra the CUDA kernels implement, pinned
               against ``recurrent`` as the SinkProbe README describes for its
               delta-rule layer (chunk sizes 1, 8, 16, 64; agreement 1e-10).
``backward``   the gradients of the recurrence: the adjoint of each step of the
               token loop, in reverse order, in fp64 (C, ``gdr_oracle.c``).

Pins (tests/test_oracle_pins.py) tie ``recurrent`` to closed forms, brute
force and invariants that do not use this code. The GQA/GVA head-mapping
convention (value head h reads key head h // (Hv // Hk)) is a declared
convention the pages do not fix: parity unpinned for that choice alone.
"""
import ctypes
import os

import numpy as np

from .build import build as _build
from .chunked import chunked  # noqa: F401

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.gdr_oracle_recurrent.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp] + [ctypes.c_int] * 8
        lib.gdr_oracle_recurrent.restype = ctypes.c_int
        lib.gdr_oracle_threads.argtypes = [ctypes.c_int, ctypes.c_long]
        lib.gdr_oracle_threads.restype = ctypes.c_int
        lib.gdr_oracle_backward.argtypes = [dp] * 14 + [ctypes.c_int] * 8
        lib.gdr_oracle_backward.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor -> fp64 numpy (exact upcast of bf16/fp32)
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def threads_used(nthreads: int, units: int) -> int:
    return int(_load().gdr_oracle_threads(int(nthreads), int(units)))


def recurrent(q, k, v, g, beta, h0=None, gate_mode=None, nthreads=0, want_o=True):
    """Token-by-token fp64 recurrence.

    q, k: [B,T,Hk,Dk]; v: [B,T,Hv,Dv]; g: [B,T,Hv] (scalar gate) or
    [B,T,Hv,Dk] (per-channel gate); beta: [B,T,Hv]; h0: [B,Hv,Dk,Dv] or None.
    Inputs may be numpy arrays or CPU/GPU torch tensors; they are upcast to fp64
    exactly. Returns (o [B,T,Hv,Dv] or None, hT [B,Hv,Dk,Dv]) as fp64 numpy.
    """
    q, k, v, g, beta, h0 = (_f64(x) for x in (q, k, v, g, beta, h0))
    B, T, Hk, Dk = q.shape
    Hv, Dv = v.shape[2], v.shape[3]
    if gate_mode is None:
        gate_mode = 1 if g.ndim == 4 else 0
    assert k.shape == q.shape and v.shape[:2] == (B, T)
    assert beta.shape == (B, T, Hv)
    assert g.shape == ((B, T, Hv) if gate_mode == 0 else (B, T, Hv, Dk))
    if h0 is not None:
        assert h0.shape == (B, Hv, Dk, Dv)
    o = np.zeros((B, T, Hv, Dv), dtype=np.float64) if want_o else None
    hT = np.zeros((B, Hv, Dk, Dv), dtype=np.float64)
    rc = _load().gdr_oracle_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                                      _ptr(o), _ptr(hT), B, T, Hk, Hv, Dk, Dv, gate_mode,
                                      int(nthreads))
    if rc != 0:
        raise ValueError("gdr_oracle_recurrent rejected its arguments")
    return o, hT


def decode_steps(q, k, v, g, beta, h0, nthreads=0):
    """Repeated single-token steps: inputs are [steps, B, H, D] (g: [steps,B,Hv] or
    [steps,B,Hv,Dk]); returns (o [steps,B,Hv,Dv], final state [B,Hv,Dk,Dv]).

    One decode step is the recurrence with T = 1, so this feeds each step to
    ``recurrent`` with the previous step's final state as its h0.
    """
    q, k, v, g, beta, h0 = (_f64(x) for x in (q, k, v, g, beta, h0))
    steps = q.shape[0]
    S = h0
    outs = []
    for s in range(steps):
        o, S = recurrent(q[s][:, None], k[s][:, None], v[s][:, None], g[s][:, None],
                         beta[s][:, None], S, nthreads=nthreads)
        outs.append(o[:, 0])
    return np.stack(outs, 0), S


def backward(q, k, v, g, beta, h0, do, dhT=None, gate_mode=None, nthreads=0):
    """Gradients of L = sum(do * o) + sum(dhT * hT) through the token recurrence, fp64.

    Shapes as in ``recurrent``; do [B,T,Hv,Dv]; dhT [B,Hv,Dk,Dv] or None (zero).
    Returns a dict with dq, dk [B,T,Hk,Dk], dv [B,T,Hv,Dv], dg (g's shape),
    dbeta [B,T,Hv] and dh0 [B,Hv,Dk,Dv] as fp64 numpy arrays.
    """
    q, k, v, g, beta, h0, do, dhT = (_f64(x) for x in (q, k, v, g, beta, h0, do, dhT))
    B, T, Hk, Dk = q.shape
    Hv, Dv = v.shape[2], v.shape[3]
    if gate_mode is None:
        gate_mode = 1 if g.ndim == 4 else 0
    assert do.shape == v.shape and beta.shape == (B, T, Hv)
    out = {"dq": np.zeros(q.shape), "dk": np.zeros(k.shape), "dv": np.zeros(v.shape),
           "dg": np.zeros(g.shape), "dbeta": np.zeros(beta.shape), "dh0": np.zeros((B, Hv, Dk, Dv))}
    rc = _load().gdr_oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(do),
                                     _ptr(dhT), *(_ptr(out[n]) for n in ("dq", "dk", "dv", "dg", "dbeta", "dh0")),
                                     B, T, Hk, Hv, Dk, Dv, gate_mode, int(nthreads))
    if rc != 0:
        raise ValueError("gdr_oracle_backward rejected its arguments")
    return out
