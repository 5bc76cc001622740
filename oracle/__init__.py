"""KDA oracle -- TEST INFRASTRUCTURE ONLY.

A plain fp64 CPU statement of the Kimi Delta Attention recurrence
(``kda_oracle.c``), wrapped with ctypes.  Only ``tests/``, the package's
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference leg
may import this module.  The CUDA product path never imports it.

Sources: "Kimi Delta Attention 徹底解説" (tech-tide.dev), sections
"なぜ今「線形アテンション」なのか" and "Kimi Delta Attention の仕組み"; "Kimi
Linear、独自の土俵でFull Attentionを上回る" (remio.ai), section "Kimi Linearが
より賢いRecurrent Memoryを使う方法".  The recurrence, per (sequence, head)::

    S'  = Diag(alpha_t) S          alpha_t = exp(log_alpha_t), on the key axis
    S   = S' + beta_t k_t (v_t - S'^T k_t)^T
    o_t = S^T q_t

Every function here is pinned by ``tests/test_oracle_pins.py`` against
closed forms, special cases (DeltaNet, Gated DeltaNet), brute force and a
hand-worked fixture; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build_oracle, library_path

__all__ = ["forward", "backward", "prologue", "unrolled", "step", "max_threads", "library_path", "build_oracle"]

_lib = None


def _load():
    global _lib
    if _lib is None:
        # KDA_ORACLE_LIB lets the mutation test load a deliberately broken copy.
        path = os.environ.get("KDA_ORACLE_LIB") or library_path()
        src = os.path.join(os.path.dirname(__file__), "kda_oracle.c")
        if "KDA_ORACLE_LIB" not in os.environ and (
                not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(src)):
            build_oracle()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        c_int = ctypes.c_int
        lib.kda_oracle_forward.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, ip] + [c_int] * 7
        lib.kda_oracle_forward.restype = c_int
        lib.kda_oracle_backward.argtypes = [dp] * 14 + [ip] + [c_int] * 7
        lib.kda_oracle_backward.restype = c_int
        lib.kda_oracle_unrolled.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp] + [c_int] * 5
        lib.kda_oracle_unrolled.restype = c_int
        lib.kda_oracle_step.argtypes = [dp, dp, dp, dp, dp, dp, dp] + [c_int] * 5
        lib.kda_oracle_step.restype = c_int
        lib.kda_oracle_max_threads.argtypes = []
        lib.kda_oracle_max_threads.restype = c_int
        _lib = lib
    return _lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def max_threads() -> int:
    """Number of OpenMP threads the oracle uses by default."""
    return int(_load().kda_oracle_max_threads())


def forward(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, nthreads=0):
    """Token-by-token fp64 recurrence.

    q, k, log_alpha: [B, T, H, dk]; v: [B, T, H, dv]; beta: [B, T, H];
    init_state: [N, H, dk, dv] or None (zeros); cu_seqlens: [N+1] int or None
    (then N = B).  Returns (o [B, T, H, dv], final_state [N, H, dk, dv]),
    both float64.
    """
    q, k, v, g, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or g.shape != q.shape or v.shape[:3] != q.shape[:3] or b.shape != q.shape[:3]:
        raise ValueError("oracle.forward: inconsistent shapes")
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        N = cu.shape[0] - 1
    else:
        N = B
    s0 = None if init_state is None else _f64(init_state)
    if s0 is not None and s0.shape != (N, H, dk, dv):
        raise ValueError("oracle.forward: init_state shape")
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    fs = np.zeros((N, H, dk, dv), dtype=np.float64)
    cu_p = None if cu is None else cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    rc = _load().kda_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(s0),
                                    _ptr(o), _ptr(fs), cu_p, B, T, H, dk, dv, N, int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle.forward failed with code {rc}")
    return o, fs


def backward(q, k, v, log_alpha, beta, d_o, init_state=None, dfinal=None, cu_seqlens=None, nthreads=0):
    """Gradients of L = sum <d_o, o> + <dfinal, final_state> by reverse-mode
    differentiation of the token recurrence (fp64).

    Shapes as in :func:`forward`; d_o is [B, T, H, dv], dfinal is
    [N, H, dk, dv] or None (zero).  Returns a dict with dq, dk, dv,
    dlog_alpha, dbeta and dinit_state (dL/dS_0, also when init_state is None).
    """
    q, k, v, g, b, do = (_f64(x) for x in (q, k, v, log_alpha, beta, d_o))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if (k.shape != q.shape or g.shape != q.shape or v.shape[:3] != q.shape[:3]
            or b.shape != q.shape[:3] or do.shape != v.shape):
        raise ValueError("oracle.backward: inconsistent shapes")
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        N = cu.shape[0] - 1
    else:
        N = B
    s0 = None if init_state is None else _f64(init_state)
    dS = None if dfinal is None else _f64(dfinal)
    for name, x in (("init_state", s0), ("dfinal", dS)):
        if x is not None and x.shape != (N, H, dk, dv):
            raise ValueError(f"oracle.backward: {name} shape")
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v),
               dlog_alpha=np.zeros_like(g), dbeta=np.zeros_like(b),
               dinit_state=np.zeros((N, H, dk, dv), dtype=np.float64))
    cu_p = None if cu is None else cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    rc = _load().kda_oracle_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(s0), _ptr(do), _ptr(dS),
        _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dlog_alpha"]),
        _ptr(out["dbeta"]), _ptr(out["dinit_state"]), cu_p, B, T, H, dk, dv, N, int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle.backward failed with code {rc}")
    return out


def prologue(q_raw, k_raw, gate_x, eps=1e-6):
    """Input prologue of the operator, fp64 (numpy), for the fused-prologue entry
    points: q and k scaled to unit L2 norm over the key axis, and the per-channel
    log-decay from the gate pre-activation x,

        q = q_raw / max(|q_raw|_2, eps),   k likewise,   log_alpha = -softplus(x)

    ("Kimi Linear、独自の土俵でFull Attentionを上回る" (remio.ai), § "Kimi Linearが
    より賢いRecurrent Memoryを使う方法": the decay gate is computed per channel from
    the current token; the pages leave its parametrisation open, so this module
    takes the plainest form with alpha in (0, 1): alpha = exp(-softplus(x)) =
    1 / (1 + e^x)).  softplus is evaluated as max(x, 0) + log1p(exp(-|x|)).
    Shapes: q_raw, k_raw, gate_x [..., dk]; returns (q, k, log_alpha) float64.
    """
    q = _f64(q_raw)
    k = _f64(k_raw)
    x = _f64(gate_x)
    qn = np.maximum(np.sqrt((q * q).sum(axis=-1, keepdims=True)), eps)
    kn = np.maximum(np.sqrt((k * k).sum(axis=-1, keepdims=True)), eps)
    log_alpha = -(np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x))))
    return q / qn, k / kn, log_alpha


def unrolled(q, k, v, log_alpha, beta, init_state=None):
    """Brute-force transition-matrix product form (tiny sizes only)."""
    q, k, v, g, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    s0 = None if init_state is None else _f64(init_state)
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    fs = np.zeros((B, H, dk, dv), dtype=np.float64)
    rc = _load().kda_oracle_unrolled(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(s0),
                                     _ptr(o), _ptr(fs), B, T, H, dk, dv)
    if rc != 0:
        raise ValueError(f"oracle.unrolled failed with code {rc}")
    return o, fs


def step(q, k, v, log_alpha, beta, state, nthreads=0):
    """One decode step for [N, H] states.  Returns (o [N, H, dv], new_state)."""
    q, k, v, g, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    N, H, dk = q.shape
    dv = v.shape[-1]
    s = _f64(state).copy()
    o = np.zeros((N, H, dv), dtype=np.float64)
    rc = _load().kda_oracle_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(s), _ptr(o),
                                 N, H, dk, dv, int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle.step failed with code {rc}")
    return o, s
