"""B200-native Kimi Delta Attention (KDA) operator: Python binding of libkda.

Thin ctypes marshalling over the C ABI in include/kda.h: every step of the
operator runs in the CUDA kernels of libkda.so; PyTorch only provides device
memory and the current stream.  There is no CPU fallback: calling an operator
without the built library, or without a CUDA device, raises.

    o, S = chunk_forward(q, k, v, log_alpha, beta, init_state, cu_seqlens=None)
    o    = recurrent_step(q, k, v, log_alpha, beta, state)      # state in place
    g    = chunk_backward(q, k, v, log_alpha, beta, d_o, init_state)   # dict of gradients

The recurrence ("Kimi Delta Attention 徹底解説" (tech-tide.dev), § "Kimi Delta
Attention の仕組み"), per (sequence, head), with a dk x dv fp32 state S:
    S' = Diag(exp(log_alpha_t)) S;  S = S' + beta_t k_t (v_t - S'^T k_t)^T;  o_t = S^T q_t
"""
from __future__ import annotations

import ctypes
import os
from types import SimpleNamespace

import torch

__all__ = [
    "chunk_forward", "chunk_backward", "gdn_chunk_backward", "backward_workspace_size", "chunk_forward_prologue",
    "recurrent_step_prologue", "chunk_forward_simt", "chunk_forward_static_ws", "chunk_forward_slots", "recurrent_step",
    "recurrent_step_slots", "gdn_chunk_forward", "gdn_recurrent_step", "workspace_size", "set_auto_workspace_limit",
    "device_status",
    "debug_wait_timeout", "last_error", "library_path", "load_library", "KDAError", "KDA_BF16", "KDA_F32", "CHUNK",
    "DEV_WAIT_TIMEOUT", "DEV_DECAY_RANGE", "DEV_BAD_SLOT", "ALGOS",
]

KDA_BF16 = 0
KDA_F32 = 1
CHUNK = 64
DEV_WAIT_TIMEOUT = 0x1
DEV_DECAY_RANGE = 0x2
DEV_BAD_SLOT = 0x4
# tensor-core prefill schedules (KDA_ALGO_* in include/kda.h)
ALGOS = {"auto": 0, "fused": 1, "two_pass": 2}
# size of the built-in scratch of kda_chunk_forward_static_ws (KDA_STATIC_WS_BYTES)
STATIC_WS_BYTES = 64 << 20

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None


class KDAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"kda error {code}: {msg}")
        self.code = code


def library_path() -> str:
    return os.path.join(_HERE, "libkda.so")


def load_library():
    """Load libkda.so (built by gated_delta_rule_85_b200/build.py); raise if absent."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"libkda.so is not built ({path}); run gated_delta_rule_85_b200/build.py")
    lib = ctypes.CDLL(path)
    vp, fp, ip = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
    ci, sz = ctypes.c_int, ctypes.c_size_t
    lib.kda_chunk_forward.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, ip] + [ci] * 8 + [vp, sz, vp]
    lib.kda_chunk_forward.restype = ci
    lib.kda_chunk_forward_simt.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, ip] + [ci] * 8 + [vp]
    lib.kda_chunk_forward_simt.restype = ci
    lib.kda_chunk_forward_workspace_size.argtypes = [ci] * 8
    lib.kda_chunk_forward_workspace_size.restype = sz
    lib.kda_chunk_forward_ex.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, ip] + [ci] * 9 + [vp, sz, vp]
    lib.kda_chunk_forward_ex.restype = ci
    lib.kda_chunk_forward_workspace_size_ex.argtypes = [ci] * 9
    lib.kda_chunk_forward_workspace_size_ex.restype = sz
    lib.kda_chunk_forward_static_ws.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, ip] + [ci] * 8 + [vp]
    lib.kda_chunk_forward_static_ws.restype = ci
    lib.kda_chunk_forward_slots.argtypes = [vp, vp, vp, fp, fp, fp, ip, vp, ip] + [ci] * 10 + [vp, sz, vp]
    lib.kda_chunk_forward_slots.restype = ci
    lib.kda_recurrent_step_slots.argtypes = [vp, vp, vp, fp, fp, fp, ip, vp] + [ci] * 6 + [vp]
    lib.kda_recurrent_step_slots.restype = ci
    lib.kda_gdn_chunk_forward.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, ip] + [ci] * 9 + [vp, sz, vp]
    lib.kda_gdn_chunk_forward.restype = ci
    lib.kda_gdn_recurrent_step.argtypes = [vp, vp, vp, fp, fp, fp, vp] + [ci] * 5 + [vp]
    lib.kda_gdn_recurrent_step.restype = ci
    lib.kda_recurrent_step.argtypes = [vp, vp, vp, fp, fp, fp, vp] + [ci] * 5 + [vp]
    lib.kda_recurrent_step.restype = ci
    lib.kda_chunk_forward_prologue.argtypes = [vp, vp, vp, vp, fp, fp, vp, fp, ip] + [ci] * 9 + [vp, sz, vp]
    lib.kda_chunk_forward_prologue.restype = ci
    lib.kda_recurrent_step_prologue.argtypes = [vp, vp, vp, vp, fp, fp, vp] + [ci] * 5 + [vp]
    lib.kda_recurrent_step_prologue.restype = ci
    lib.kda_chunk_backward.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, vp, vp, vp, fp, fp, fp, ip] + \
        [ci] * 8 + [vp, sz, vp]
    lib.kda_chunk_backward.restype = ci
    lib.kda_gdn_chunk_backward.argtypes = lib.kda_chunk_backward.argtypes
    lib.kda_gdn_chunk_backward.restype = ci
    lib.kda_chunk_backward_workspace_size.argtypes = [ci] * 6
    lib.kda_chunk_backward_workspace_size.restype = sz
    lib.kda_chunk_backward_workspace_size_ex.argtypes = [ci] * 8
    lib.kda_chunk_backward_workspace_size_ex.restype = sz
    lib.kda_chunk_backward_ex.argtypes = lib.kda_chunk_backward.argtypes + [ci]
    lib.kda_chunk_backward_ex.restype = ci
    lib.kda_gdn_chunk_backward_ex.argtypes = lib.kda_chunk_backward_ex.argtypes
    lib.kda_gdn_chunk_backward_ex.restype = ci
    lib.kda_last_error.argtypes = []
    lib.kda_last_error.restype = ctypes.c_char_p
    lib.kda_get_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint), ci, vp]
    lib.kda_get_device_status.restype = ci
    lib.kda_debug_wait_timeout.argtypes = [ctypes.c_longlong, vp]
    lib.kda_debug_wait_timeout.restype = ci
    lib.kda_api_version.argtypes = []
    lib.kda_api_version.restype = ci
    lib.kda_set_auto_workspace_limit.argtypes = [sz]
    lib.kda_set_auto_workspace_limit.restype = sz
    _lib = lib
    return lib


def last_error() -> str:
    return load_library().kda_last_error().decode()


def _check(rc: int):
    if rc != 0:
        raise KDAError(rc, last_error())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError(f"unsupported dtype {t.dtype}; q/k/v must be bfloat16 or float32")


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be on the same CUDA device")
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous in the documented layouts")


def _algo_code(algo: str) -> int:
    if algo not in ALGOS:
        raise ValueError(f"algo must be one of {sorted(ALGOS)}, got {algo!r}")
    return ALGOS[algo]


def set_auto_workspace_limit(nbytes: int) -> int:
    """AUTO's workspace budget in bytes (kda_set_auto_workspace_limit; 0 restores the
    1 GiB default).  Returns the previous budget."""
    return int(load_library().kda_set_auto_workspace_limit(int(nbytes)))


def workspace_size(B, T, H, dk, dv, num_seqs, dtype=KDA_BF16, algo="auto") -> int:
    return int(load_library().kda_chunk_forward_workspace_size_ex(B, T, H, dk, dv, num_seqs, dtype, CHUNK,
                                                                  _algo_code(algo)))


def _prefill_args(q, k, v, log_alpha, beta, init_state, cu_seqlens):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or log_alpha.shape != q.shape or v.shape[:3] != q.shape[:3] or beta.shape != q.shape[:3]:
        raise ValueError("shape mismatch among q, k, v, log_alpha, beta")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k and v must share a dtype")
    if log_alpha.dtype != torch.float32 or beta.dtype != torch.float32:
        raise ValueError("log_alpha and beta must be float32")
    N = B if cu_seqlens is None else cu_seqlens.shape[0] - 1
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    if init_state is not None and (init_state.shape != (N, H, dk, dv) or init_state.dtype != torch.float32):
        raise ValueError("init_state must be float32 [N, H, dk, dv]")
    return B, T, H, dk, dv, N


def _to_device(ts, device):
    return [None if t is None else t.to(device, non_blocking=True) for t in ts]


def chunk_forward(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, *, o=None,
                  final_state=True, workspace=None, simt=False, algo="auto"):
    """Chunked KDA prefill (64-token chunks) through kda_chunk_forward_ex.

    Tensors are in the include/kda.h layouts.  `final_state` may be True
    (allocate and return), False (skip) or a preallocated float32 tensor.
    `algo` picks the tensor-core schedule ("auto", "fused", "two_pass"); the
    workspace it needs is allocated here unless `workspace` (uint8, CUDA) is
    given.  "auto" takes the two-pass schedule for few (sequence, head) chains
    within AUTO's workspace budget (1 GiB, set_auto_workspace_limit), running a
    single long sequence in windows that fit it (the two-pass records are 58 KB per
    64-token chunk and head, 3.8 GB unwindowed at 131072 tokens x 32 heads); pass a
    reusable `workspace` (workspace_size(..., algo=...)) to keep it across calls,
    or algo="fused" to need none.  With `simt=True` the fp32 CUDA-core path (kda_chunk_forward_simt)
    runs instead.  Host (CPU) inputs are copied to the current CUDA device and
    the results copied back, all inside this call.
    Returns (o, final_state or None).
    """
    if not q.is_cuda:
        dev = torch.device("cuda", torch.cuda.current_device())
        args = _to_device([q, k, v, log_alpha, beta, init_state, cu_seqlens], dev)
        fs_dev = final_state if isinstance(final_state, bool) else True
        o_d, s_d = chunk_forward(*args, final_state=fs_dev, workspace=workspace, simt=simt, algo=algo)
        o_h = o if o is not None else torch.empty(o_d.shape, dtype=o_d.dtype, pin_memory=True)
        o_h.copy_(o_d, non_blocking=True)
        s_h = None
        if s_d is not None:
            s_h = final_state if isinstance(final_state, torch.Tensor) else \
                torch.empty(s_d.shape, dtype=s_d.dtype, pin_memory=True)
            s_h.copy_(s_d, non_blocking=True)
        torch.cuda.current_stream(dev).synchronize()
        return o_h, s_h
    B, T, H, dk, dv, N = _prefill_args(q, k, v, log_alpha, beta, init_state, cu_seqlens)
    _need_cuda(q, k, v, log_alpha, beta, init_state, cu_seqlens)
    lib = load_library()
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is True:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    elif final_state is False:
        final_state = None
    _need_cuda(o, final_state)
    dt = _dtype_code(q)
    ac = _algo_code(algo)
    st = _stream(q.device)
    if simt:
        rc = lib.kda_chunk_forward_simt(_p(q), _p(k), _p(v), _p(log_alpha), _p(beta), _p(init_state), _p(o),
                                        _p(final_state), _p(cu_seqlens), B, T, H, dk, dv, N, dt, CHUNK, st)
    else:
        need = int(lib.kda_chunk_forward_workspace_size_ex(B, T, H, dk, dv, N, dt, CHUNK, ac))
        if need and workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        rc = lib.kda_chunk_forward_ex(_p(q), _p(k), _p(v), _p(log_alpha), _p(beta), _p(init_state), _p(o),
                                      _p(final_state), _p(cu_seqlens), B, T, H, dk, dv, N, dt, CHUNK, ac,
                                      _p(workspace), ws_bytes, st)
    _check(rc)
    return o, final_state


def chunk_forward_prologue(q_raw, k_raw, v, gate_x, beta, init_state=None, cu_seqlens=None, *, o=None,
                           final_state=True, workspace=None, algo="auto"):
    """Chunked prefill on raw inputs (kda_chunk_forward_prologue): q and k are
    scaled to unit norm over dk and log_alpha = -softplus(gate_x) inside the
    kernels.  gate_x has q's shape and dtype.  Returns (o, final_state or None)."""
    # the shared shape checks, with a metadata-only stand-in for an fp32 log_alpha
    B, T, H, dk, dv, N = _prefill_args(q_raw, k_raw, v, SimpleNamespace(shape=gate_x.shape, dtype=torch.float32),
                                       beta, init_state, cu_seqlens)
    if gate_x.shape != q_raw.shape or gate_x.dtype != q_raw.dtype:
        raise ValueError("gate_x must have q's shape and dtype")
    _need_cuda(q_raw, k_raw, v, gate_x, beta, init_state, cu_seqlens)
    lib = load_library()
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q_raw.dtype, device=q_raw.device)
    if final_state is True:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q_raw.device)
    elif final_state is False:
        final_state = None
    dt = _dtype_code(q_raw)
    need = 0 if dt == KDA_F32 else int(lib.kda_chunk_forward_workspace_size_ex(B, T, H, dk, dv, N, dt, CHUNK,
                                                                                ALGOS["two_pass"]))
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q_raw.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib.kda_chunk_forward_prologue(_p(q_raw), _p(k_raw), _p(v), _p(gate_x), _p(beta), _p(init_state), _p(o),
                                        _p(final_state), _p(cu_seqlens), B, T, H, dk, dv, N, dt, CHUNK,
                                        _algo_code(algo), _p(workspace), ws_bytes, _stream(q_raw.device))
    _check(rc)
    return o, final_state


def recurrent_step_prologue(q_raw, k_raw, v, gate_x, beta, state, o=None):
    """One decode step on raw inputs (kda_recurrent_step_prologue); state updated in place."""
    N, H, dk = q_raw.shape
    dv = v.shape[-1]
    if k_raw.shape != q_raw.shape or gate_x.shape != q_raw.shape or gate_x.dtype != q_raw.dtype:
        raise ValueError("q_raw, k_raw and gate_x must share shape and dtype")
    if state.shape != (N, H, dk, dv) or state.dtype != torch.float32:
        raise ValueError("state must be float32 [N, H, dk, dv]")
    _need_cuda(q_raw, k_raw, v, gate_x, beta, state)
    if o is None:
        o = torch.empty((N, H, dv), dtype=q_raw.dtype, device=q_raw.device)
    rc = load_library().kda_recurrent_step_prologue(_p(q_raw), _p(k_raw), _p(v), _p(gate_x), _p(beta), _p(state),
                                                    _p(o), N, H, dk, dv, _dtype_code(q_raw), _stream(q_raw.device))
    _check(rc)
    return o


BACKWARD_ALGOS = {"auto": 0, "tensor": 1, "simt": 2}   # KDA_BWD_AUTO, KDA_BWD_TENSOR, KDA_BWD_SIMT


def backward_workspace_size(B, T, H, dk, dv, num_seqs, dtype=None, algo="auto") -> int:
    """Workspace bytes of kda_chunk_backward: enough for any schedule when dtype is
    None, else what the schedule `algo` takes for that dtype (torch dtype)."""
    lib = load_library()
    if dtype is None:
        return int(lib.kda_chunk_backward_workspace_size(B, T, H, dk, dv, num_seqs))
    code = {torch.bfloat16: KDA_BF16, torch.float32: KDA_F32}[dtype]
    return int(lib.kda_chunk_backward_workspace_size_ex(B, T, H, dk, dv, num_seqs, code, BACKWARD_ALGOS[algo]))


def gdn_chunk_backward(q, k, v, log_alpha, beta, d_o, init_state=None, dfinal_state=None, cu_seqlens=None, *,
                       dinit_state=True, workspace=None, out=None, algo="auto"):
    """Gradients through the Gated DeltaNet prefill (kda_gdn_chunk_backward_ex):
    log_alpha and the returned dlog_alpha are [B, T, H]; otherwise as chunk_backward."""
    if log_alpha.shape != q.shape[:3]:
        raise ValueError("log_alpha must be [B, T, H] (one rate per token-head)")
    return chunk_backward(q, k, v, log_alpha, beta, d_o, init_state, dfinal_state, cu_seqlens,
                          dinit_state=dinit_state, workspace=workspace, out=out, algo=algo, _gate_scalar=True)


def chunk_backward(q, k, v, log_alpha, beta, d_o, init_state=None, dfinal_state=None, cu_seqlens=None, *,
                   dinit_state=True, workspace=None, out=None, algo="auto", _gate_scalar=False):
    """Gradients of sum <d_o, o> + <dfinal_state, final_state> through the chunked
    prefill (kda_chunk_backward): a dict with dq, dk, dv (in q's dtype),
    dlog_alpha, dbeta and dinit_state (float32; None when dinit_state=False).

    Inputs are the forward call's, in the include/kda.h layouts; d_o has o's
    shape and dtype, dfinal_state is float32 [N, H, dk, dv] or None (zero).
    The workspace (uint8, CUDA) and the outputs (`out`, a dict with any of the
    keys above) are allocated here unless given.  algo: "auto", "tensor" or
    "simt" (kda_chunk_backward_ex).
    Device tensors only.
    """
    gate = SimpleNamespace(shape=q.shape, dtype=log_alpha.dtype) if _gate_scalar else log_alpha
    B, T, H, dk, dv, N = _prefill_args(q, k, v, gate, beta, init_state, cu_seqlens)
    if d_o.shape != v.shape or d_o.dtype != q.dtype:
        raise ValueError("d_o must have o's shape and dtype")
    if dfinal_state is not None and (dfinal_state.shape != (N, H, dk, dv) or dfinal_state.dtype != torch.float32):
        raise ValueError("dfinal_state must be float32 [N, H, dk, dv]")
    _need_cuda(q, k, v, log_alpha, beta, init_state, d_o, dfinal_state, cu_seqlens)
    lib = load_library()
    g = dict(out or {})
    dev = q.device
    g.setdefault("dq", torch.empty_like(q))
    g.setdefault("dk", torch.empty_like(k))
    g.setdefault("dv", torch.empty_like(v))
    g.setdefault("dlog_alpha", torch.empty_like(log_alpha))
    g.setdefault("dbeta", torch.empty_like(beta))
    if dinit_state:
        g.setdefault("dinit_state", torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev))
    else:
        g["dinit_state"] = None
    _need_cuda(*g.values())
    if algo not in BACKWARD_ALGOS:
        raise ValueError(f"unknown backward algo {algo!r}")
    need = int(lib.kda_chunk_backward_workspace_size_ex(B, T, H, dk, dv, N, _dtype_code(q), BACKWARD_ALGOS[algo]))
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    args = (_p(q), _p(k), _p(v), _p(log_alpha), _p(beta), _p(init_state), _p(d_o), _p(dfinal_state), _p(g["dq"]),
            _p(g["dk"]), _p(g["dv"]), _p(g["dlog_alpha"]), _p(g["dbeta"]), _p(g["dinit_state"]), _p(cu_seqlens),
            B, T, H, dk, dv, N, _dtype_code(q), CHUNK, _p(workspace), ws_bytes, _stream(dev))
    entry = lib.kda_gdn_chunk_backward_ex if _gate_scalar else lib.kda_chunk_backward_ex
    rc = entry(*args, BACKWARD_ALGOS[algo])
    _check(rc)
    return g


def chunk_forward_static_ws(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, *, o=None,
                            final_state=True):
    """kda_chunk_forward_static_ws: the two-pass prefill on the library's built-in
    scratch (no workspace argument, nothing allocated by the library).  Device
    tensors only; the caller's outputs are allocated here unless given."""
    B, T, H, dk, dv, N = _prefill_args(q, k, v, log_alpha, beta, init_state, cu_seqlens)
    _need_cuda(q, k, v, log_alpha, beta, init_state, cu_seqlens)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is True:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    elif final_state is False:
        final_state = None
    _need_cuda(o, final_state)
    rc = load_library().kda_chunk_forward_static_ws(
        _p(q), _p(k), _p(v), _p(log_alpha), _p(beta), _p(init_state), _p(o), _p(final_state), _p(cu_seqlens),
        B, T, H, dk, dv, N, _dtype_code(q), CHUNK, _stream(q.device))
    _check(rc)
    return o, final_state


def chunk_forward_simt(*args, **kw):
    """kda_chunk_forward_simt: the fp32 CUDA-core prefill path."""
    return chunk_forward(*args, simt=True, **kw)


def recurrent_step(q, k, v, log_alpha, beta, state, o=None):
    """One KDA decode step (kda_recurrent_step); `state` [N, H, dk, dv] fp32 is updated in place."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or log_alpha.shape != q.shape or v.shape[:2] != q.shape[:2] or beta.shape != q.shape[:2]:
        raise ValueError("shape mismatch among q, k, v, log_alpha, beta")
    if state.shape != (N, H, dk, dv) or state.dtype != torch.float32:
        raise ValueError("state must be float32 [N, H, dk, dv]")
    _need_cuda(q, k, v, log_alpha, beta, state)
    if o is None:
        o = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    rc = load_library().kda_recurrent_step(_p(q), _p(k), _p(v), _p(log_alpha), _p(beta), _p(state), _p(o),
                                           N, H, dk, dv, _dtype_code(q), _stream(q.device))
    _check(rc)
    return o


def _check_slots(slots, n):
    if slots.dtype != torch.int32 or slots.shape != (n,) or not slots.is_cuda:
        raise ValueError(f"slots must be a CUDA int32 tensor of shape ({n},)")


def chunk_forward_slots(q, k, v, log_alpha, beta, state_pool, slots, cu_seqlens=None, *, o=None, workspace=None,
                        algo="auto"):
    """Prefill from and into a state pool (kda_chunk_forward_slots): sequence n
    starts from state_pool[slots[n]] and its final state is written back there
    (slot -1: start from zeros, write nothing).  Device tensors; returns o."""
    B, T, H, dk, dv, N = _prefill_args(q, k, v, log_alpha, beta, None, cu_seqlens)
    if state_pool.dim() != 4 or state_pool.shape[1:] != (H, dk, dv) or state_pool.dtype != torch.float32:
        raise ValueError("state_pool must be float32 [num_slots, H, dk, dv]")
    _check_slots(slots, N)
    _need_cuda(q, k, v, log_alpha, beta, state_pool, slots, cu_seqlens)
    lib = load_library()
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    dt = _dtype_code(q)
    ac = _algo_code(algo)
    need = int(lib.kda_chunk_forward_workspace_size_ex(B, T, H, dk, dv, N, dt, CHUNK, ac))
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib.kda_chunk_forward_slots(_p(q), _p(k), _p(v), _p(log_alpha), _p(beta), _p(state_pool), _p(slots),
                                     _p(o), _p(cu_seqlens), B, T, H, dk, dv, N, state_pool.shape[0], dt, CHUNK,
                                     ac, _p(workspace), ws_bytes, _stream(q.device))
    _check(rc)
    return o


def recurrent_step_slots(q, k, v, log_alpha, beta, state_pool, slots, o=None):
    """One decode step on a state pool (kda_recurrent_step_slots): sequence n uses
    and updates state_pool[slots[n]] in place (slot -1: padding, o row zero)."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or log_alpha.shape != q.shape or v.shape[:2] != q.shape[:2] or beta.shape != q.shape[:2]:
        raise ValueError("shape mismatch among q, k, v, log_alpha, beta")
    if state_pool.dim() != 4 or state_pool.shape[1:] != (H, dk, dv) or state_pool.dtype != torch.float32:
        raise ValueError("state_pool must be float32 [num_slots, H, dk, dv]")
    _check_slots(slots, N)
    _need_cuda(q, k, v, log_alpha, beta, state_pool, slots)
    if o is None:
        o = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    rc = load_library().kda_recurrent_step_slots(_p(q), _p(k), _p(v), _p(log_alpha), _p(beta), _p(state_pool),
                                                 _p(slots), _p(o), N, H, dk, dv, state_pool.shape[0],
                                                 _dtype_code(q), _stream(q.device))
    _check(rc)
    return o


def gdn_chunk_forward(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, *, o=None, final_state=True,
                      workspace=None, algo="auto"):
    """Gated DeltaNet prefill (kda_gdn_chunk_forward): log_alpha is one scalar per
    (token, head), shape [B, T, H].  Device tensors; returns (o, final_state or None)."""
    B, T, H, dk = q.shape
    if log_alpha.shape != q.shape[:3] or log_alpha.dtype != torch.float32:
        raise ValueError("log_alpha must be float32 [B, T, H] for the scalar gate")
    _, _, _, _, dv, N = _prefill_args(q, k, v, log_alpha.unsqueeze(-1).expand(q.shape), beta, init_state, cu_seqlens)
    _need_cuda(q, k, v, log_alpha, beta, init_state, cu_seqlens)
    lib = load_library()
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is True:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    elif final_state is False:
        final_state = None
    dt = _dtype_code(q)
    ac = _algo_code(algo)
    need = int(lib.kda_chunk_forward_workspace_size_ex(B, T, H, dk, dv, N, dt, CHUNK, ac))
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib.kda_gdn_chunk_forward(_p(q), _p(k), _p(v), _p(log_alpha), _p(beta), _p(init_state), _p(o),
                                   _p(final_state), _p(cu_seqlens), B, T, H, dk, dv, N, dt, CHUNK, ac,
                                   _p(workspace), ws_bytes, _stream(q.device))
    _check(rc)
    return o, final_state


def gdn_recurrent_step(q, k, v, log_alpha, beta, state, o=None):
    """One Gated DeltaNet decode step (kda_gdn_recurrent_step); log_alpha [N, H]."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    if log_alpha.shape != q.shape[:2] or log_alpha.dtype != torch.float32:
        raise ValueError("log_alpha must be float32 [N, H] for the scalar gate")
    if state.shape != (N, H, dk, dv) or state.dtype != torch.float32:
        raise ValueError("state must be float32 [N, H, dk, dv]")
    _need_cuda(q, k, v, log_alpha, beta, state)
    if o is None:
        o = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    rc = load_library().kda_gdn_recurrent_step(_p(q), _p(k), _p(v), _p(log_alpha), _p(beta), _p(state), _p(o),
                                               N, H, dk, dv, _dtype_code(q), _stream(q.device))
    _check(rc)
    return o


def debug_wait_timeout(limit_cycles: int = 2_000_000) -> None:
    """Test hook: one CTA waits (bounded by `limit_cycles` SM cycles) on an mbarrier
    nothing completes, so the device status word gets DEV_WAIT_TIMEOUT; asynchronous
    on the current stream of the current device."""
    _check(load_library().kda_debug_wait_timeout(int(limit_cycles), _stream(torch.cuda.current_device())))


def device_status(clear: bool = True) -> int:
    """Device status word (KDA_DEV_* bits) of the current device; synchronises."""
    bits = ctypes.c_uint(0)
    rc = load_library().kda_get_device_status(ctypes.byref(bits), int(clear),
                                              _stream(torch.cuda.current_device()))
    if rc not in (0, -6):
        _check(rc)
    return int(bits.value)
