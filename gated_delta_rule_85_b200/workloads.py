"""Seeded synthetic inputs for the KDA operator.

This module holds no KDA arithmetic: it only draws the operator's inputs with
the distributions and shapes of the workloads the tests and the benchmark use,
so the CUDA path and the fp64 oracle can be fed the exact same tensors.

Distributions (per the workload definitions):
  q, k      ~ N(0, 1), then L2-normalised over dk per (token, head) in fp32,
              then cast to the input dtype (bf16 or fp32)
  v         ~ N(0, 1), cast to the input dtype
  log_alpha = -softplus(x), x ~ N(-2, 1), fp32, one value per channel (KDA), or
              one per (token, head) for the scalar gate of Gated DeltaNet
  beta      = sigmoid(x), x ~ N(0, 1), fp32, one value per (token, head)
  states    ~ N(0, 0.01^2) fp32 (std 0.01), or zeros
  backward cotangents: d_o ~ N(0, 1) in the input dtype, dfinal_state ~ N(0, 1) fp32
  raw inputs (fused-prologue entry points): q, k ~ N(0, 1) not normalised, and the
              gate pre-activation gate_x ~ N(-2, 1), all in the input dtype
  strong decay (strong_decay): parts of a gate tensor overwritten with fast
              forgetting -- single-token hard resets (log_alpha = -100), whole
              64-token chunks at log_alpha = -2, channels at -10 -- or, for a
              gate pre-activation, the values x whose -softplus(x) is about those
Every tensor is drawn from its own generator seeded with (seed, stream id), so
one tensor's draw does not depend on another's size.  Large tensors are drawn
in token slices of fixed size so device memory for temporaries stays bounded.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

_STREAM = {"q": 1, "k": 2, "v": 3, "log_alpha": 4, "beta": 5, "init_state": 6, "d_o": 7, "dfinal_state": 8,
           "gate_x": 9}
_SLICE_TOKENS = 1 << 15


@dataclass(frozen=True)
class PrefillShape:
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: torch.dtype = torch.bfloat16
    init_state: str = "normal"          # "normal" (std 0.01) or "zeros"
    cu_seqlens: tuple | None = None      # packed layout when set (B must be 1)
    gate: str = "channel"                # "channel": log_alpha [B, T, H, dk]; "scalar": [B, T, H]
    inputs: str = "prepared"             # "raw": q, k unnormalised and gate_x instead of log_alpha

    @property
    def num_seqs(self) -> int:
        return self.B if self.cu_seqlens is None else len(self.cu_seqlens) - 1


@dataclass(frozen=True)
class DecodeShape:
    N: int
    H: int
    dk: int
    dv: int
    steps: int
    dtype: torch.dtype = torch.bfloat16
    gate: str = "channel"                # "channel": log_alpha [N, H, dk]; "scalar": [N, H]
    inputs: str = "prepared"             # "raw": q, k unnormalised and gate_x instead of log_alpha


def _gen(device, seed: int, stream: int, sub: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + stream * 7919 + sub) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _normal(shape, device, seed, stream, mean=0.0, std=1.0):
    """fp32 normal draw, generated in token slices along dim 0*dim1 rows."""
    out = torch.empty(shape, dtype=torch.float32, device=device)
    flat = out.view(-1, shape[-1]) if len(shape) > 1 else out.view(-1, 1)
    rows = flat.shape[0]
    per = max(1, _SLICE_TOKENS * 32)
    for i, r0 in enumerate(range(0, rows, per)):
        r1 = min(rows, r0 + per)
        flat[r0:r1].normal_(mean, std, generator=_gen(device, seed, stream, i))
    return out


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    """L2-normalise the last axis in fp32 (input preparation, not KDA math)."""
    n = torch.linalg.vector_norm(x, dim=-1, keepdim=True).clamp_min(1e-6)
    return x / n


def draw_qk(shape, device, seed, stream, dtype):
    """[..., dk] keys/queries: normal, unit rows in fp32, then cast, sliced to bound memory."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat_out = out.view(-1, shape[-1])
    rows = flat_out.shape[0]
    per = _SLICE_TOKENS * 32
    for i, r0 in enumerate(range(0, rows, per)):
        r1 = min(rows, r0 + per)
        x = torch.empty((r1 - r0, shape[-1]), dtype=torch.float32, device=device)
        x.normal_(0.0, 1.0, generator=_gen(device, seed, stream, i))
        flat_out[r0:r1] = _unit_rows(x).to(dtype)
    return out


def draw_v(shape, device, seed, stream, dtype):
    out = torch.empty(shape, dtype=dtype, device=device)
    flat_out = out.view(-1, shape[-1])
    rows = flat_out.shape[0]
    per = _SLICE_TOKENS * 32
    for i, r0 in enumerate(range(0, rows, per)):
        r1 = min(rows, r0 + per)
        x = torch.empty((r1 - r0, shape[-1]), dtype=torch.float32, device=device)
        x.normal_(0.0, 1.0, generator=_gen(device, seed, stream, i))
        flat_out[r0:r1] = x.to(dtype)
    return out


def draw_raw(shape, device, seed, stream, dtype, mean=0.0):
    """N(mean, 1) drawn in fp32, then cast (raw q, k or gate pre-activation)."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat_out = out.view(-1, shape[-1])
    rows = flat_out.shape[0]
    per = _SLICE_TOKENS * 32
    for i, r0 in enumerate(range(0, rows, per)):
        r1 = min(rows, r0 + per)
        x = torch.empty((r1 - r0, shape[-1]), dtype=torch.float32, device=device)
        x.normal_(mean, 1.0, generator=_gen(device, seed, stream, i))
        flat_out[r0:r1] = x.to(dtype)
    return out


def draw_log_alpha(shape, device, seed, stream):
    """-softplus(N(-2, 1)) per channel, fp32."""
    out = torch.empty(shape, dtype=torch.float32, device=device)
    flat = out.view(-1, shape[-1])
    rows = flat.shape[0]
    per = _SLICE_TOKENS * 32
    for i, r0 in enumerate(range(0, rows, per)):
        r1 = min(rows, r0 + per)
        x = flat[r0:r1]
        x.normal_(-2.0, 1.0, generator=_gen(device, seed, stream, i))
        torch.nn.functional.softplus(x, out=x)
        x.neg_()
    return out


def draw_beta(shape, device, seed, stream):
    """sigmoid(N(0, 1)) per (token, head), fp32."""
    x = torch.empty(shape, dtype=torch.float32, device=device)
    x.normal_(0.0, 1.0, generator=_gen(device, seed, stream))
    return torch.sigmoid(x)


def draw_state(shape, device, seed, stream, kind="normal"):
    if kind == "zeros":
        return torch.zeros(shape, dtype=torch.float32, device=device)
    x = torch.empty(shape, dtype=torch.float32, device=device)
    x.normal_(0.0, 0.01, generator=_gen(device, seed, stream))
    return x


def prefill_inputs(shape: PrefillShape, seed: int = 0, device="cpu") -> dict:
    """All prefill inputs of one workload, drawn in the order q, k, v, log_alpha, beta, init_state."""
    B, T, H, dk, dv = shape.B, shape.T, shape.H, shape.dk, shape.dv
    if shape.inputs == "raw":
        d = {
            "q": draw_raw((B, T, H, dk), device, seed, _STREAM["q"], shape.dtype),
            "k": draw_raw((B, T, H, dk), device, seed, _STREAM["k"], shape.dtype),
            "v": draw_v((B, T, H, dv), device, seed, _STREAM["v"], shape.dtype),
            "gate_x": draw_raw((B, T, H, dk), device, seed, _STREAM["gate_x"], shape.dtype, mean=-2.0),
            "beta": draw_beta((B, T, H), device, seed, _STREAM["beta"]),
        }
        N = shape.num_seqs
        d["init_state"] = (None if shape.init_state == "none"
                           else draw_state((N, H, dk, dv), device, seed, _STREAM["init_state"], shape.init_state))
        d["cu_seqlens"] = (None if shape.cu_seqlens is None
                           else torch.tensor(shape.cu_seqlens, dtype=torch.int32, device=device))
        return d
    d = {
        "q": draw_qk((B, T, H, dk), device, seed, _STREAM["q"], shape.dtype),
        "k": draw_qk((B, T, H, dk), device, seed, _STREAM["k"], shape.dtype),
        "v": draw_v((B, T, H, dv), device, seed, _STREAM["v"], shape.dtype),
        "log_alpha": draw_log_alpha((B, T, H, dk) if shape.gate == "channel" else (B, T, H), device, seed,
                                    _STREAM["log_alpha"]),
        "beta": draw_beta((B, T, H), device, seed, _STREAM["beta"]),
    }
    N = shape.num_seqs
    d["init_state"] = (None if shape.init_state == "none"
                       else draw_state((N, H, dk, dv), device, seed, _STREAM["init_state"], shape.init_state))
    d["cu_seqlens"] = (None if shape.cu_seqlens is None
                       else torch.tensor(shape.cu_seqlens, dtype=torch.int32, device=device))
    return d


STRONG_KINDS = ("reset", "minus2", "mixed")
_STREAM_STRONG = 10


def strong_decay(g: torch.Tensor, kind: str, seed: int, raw: bool = False) -> torch.Tensor:
    """Overwrite parts of a gate tensor (in place; returned) with fast forgetting.

    g is log_alpha [B, T, H, dk] (per channel) or [B, T, H] (one rate per
    token-head), or with raw=True the gate pre-activation x [B, T, H, dk] of the
    fused prologue, where x = 100, 10, 2 give -softplus(x) ~ -100, -10, -2.13.
      reset   each entry independently with probability 1/32 becomes a hard reset (-100)
      minus2  tokens [64, 192) of every row become -2 (whole chunks, summed -128 per chunk)
      mixed   per channel gate: the first half of the channels -2 on every token, the next
              eight -10, and resets with probability 1/64 in the rest; one rate per
              token-head: tokens [0, 64) at -2 and resets with probability 1/16
    """
    if kind not in STRONG_KINDS:
        raise ValueError(kind)
    reset, m2, m10 = (100.0, 2.0, 10.0) if raw else (-100.0, -2.0, -10.0)
    gen = _gen(g.device, seed, _STREAM_STRONG)
    u = torch.empty(g.shape, dtype=torch.float32, device=g.device).uniform_(0.0, 1.0, generator=gen)
    per_channel = g.dim() == 4
    if kind == "reset":
        g[u < 1 / 32] = reset
    elif kind == "minus2":
        g[:, 64:192] = m2
    else:
        if per_channel:
            dk = g.shape[-1]
            rest = torch.zeros(g.shape, dtype=torch.bool, device=g.device)
            rest[..., dk // 2 + 8:] = True
            g[rest & (u < 1 / 64)] = reset
            g[..., : dk // 2] = m2
            g[..., dk // 2: dk // 2 + 8] = m10
        else:
            g[u < 1 / 16] = reset
            g[:, :64] = m2
    return g


def backward_cotangents(shape: PrefillShape, seed: int = 0, device="cpu", dfinal: bool = True) -> dict:
    """dL/do [B, T, H, dv] (input dtype) and dL/dfinal_state [N, H, dk, dv] fp32 (or None)."""
    B, T, H, dk, dv = shape.B, shape.T, shape.H, shape.dk, shape.dv
    d_o = draw_v((B, T, H, dv), device, seed, _STREAM["d_o"], shape.dtype)
    dS = None
    if dfinal:
        dS = torch.empty((shape.num_seqs, H, dk, dv), dtype=torch.float32, device=device)
        dS.normal_(0.0, 1.0, generator=_gen(device, seed, _STREAM["dfinal_state"]))
    return {"d_o": d_o, "dfinal_state": dS}


def decode_step_inputs(shape: DecodeShape, step: int, seed: int = 0, device="cpu") -> dict:
    """Per-step decode inputs (q, k, v [N, H, d], log_alpha [N, H, dk], beta [N, H])."""
    N, H, dk, dv = shape.N, shape.H, shape.dk, shape.dv
    base = seed * 65_537 + 100 + step
    if shape.inputs == "raw":
        return {
            "q": draw_raw((N, H, dk), device, base, _STREAM["q"], shape.dtype),
            "k": draw_raw((N, H, dk), device, base, _STREAM["k"], shape.dtype),
            "v": draw_v((N, H, dv), device, base, _STREAM["v"], shape.dtype),
            "gate_x": draw_raw((N, H, dk), device, base, _STREAM["gate_x"], shape.dtype, mean=-2.0),
            "beta": draw_beta((N, H), device, base, _STREAM["beta"]),
        }
    return {
        "q": draw_qk((N, H, dk), device, base, _STREAM["q"], shape.dtype),
        "k": draw_qk((N, H, dk), device, base, _STREAM["k"], shape.dtype),
        "v": draw_v((N, H, dv), device, base, _STREAM["v"], shape.dtype),
        "log_alpha": draw_log_alpha((N, H, dk) if shape.gate == "channel" else (N, H), device, base,
                                    _STREAM["log_alpha"]),
        "beta": draw_beta((N, H), device, base, _STREAM["beta"]),
    }


def decode_all_steps(shape: DecodeShape, seed: int = 0, device="cpu") -> dict:
    """Every step's inputs stacked on a leading [steps] axis, plus the initial states."""
    N, H, dk, dv, S = shape.N, shape.H, shape.dk, shape.dv, shape.steps
    out = {
        "q": torch.empty((S, N, H, dk), dtype=shape.dtype, device=device),
        "k": torch.empty((S, N, H, dk), dtype=shape.dtype, device=device),
        "v": torch.empty((S, N, H, dv), dtype=shape.dtype, device=device),
        "log_alpha": torch.empty((S, N, H, dk) if shape.gate == "channel" else (S, N, H), dtype=torch.float32,
                                 device=device),
        "beta": torch.empty((S, N, H), dtype=torch.float32, device=device),
    }
    for s in range(S):
        one = decode_step_inputs(shape, s, seed, device)
        for key in out:
            out[key][s].copy_(one[key])
    out["state"] = draw_state((N, H, dk, dv), device, seed, _STREAM["init_state"])
    return out


def varlen_lengths(total: int = 1 << 20, lo: int = 1024, hi: int = 262_144, seed: int = 0) -> list[int]:
    """Log-uniform sequence lengths in [lo, hi] that fill `total` tokens.

    Draw floor(exp(U(ln lo, ln hi))) in order with numpy PCG64(seed); stop when
    the next draw would overflow `total`; extend the last kept sequence by the
    remainder so the lengths sum to `total` exactly.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    lens: list[int] = []
    used = 0
    while True:
        L = int(math.floor(math.exp(rng.uniform(math.log(lo), math.log(hi)))))
        if used + L > total:
            break
        lens.append(L)
        used += L
    if not lens:
        return [total]
    lens[-1] += total - used
    return lens


def cu_from_lengths(lengths) -> tuple:
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    return tuple(cu)


# The five workloads the operator is measured and checked on.
CONFIGS = {
    "tiny_f32": PrefillShape(B=1, T=256, H=2, dk=64, dv=64, dtype=torch.float32, init_state="zeros"),
    "prefill_8k": PrefillShape(B=1, T=8192, H=32, dk=128, dv=128, dtype=torch.bfloat16),
    "prefill_128k": PrefillShape(B=1, T=131072, H=32, dk=128, dv=128, dtype=torch.bfloat16),
    "decode_b256": DecodeShape(N=256, H=32, dk=128, dv=128, steps=1024, dtype=torch.bfloat16),
}


def varlen_1m_shape() -> PrefillShape:
    cu = cu_from_lengths(varlen_lengths())
    return PrefillShape(B=1, T=cu[-1], H=32, dk=128, dv=128, dtype=torch.bfloat16, cu_seqlens=cu)


def to_f64(x: torch.Tensor | None):
    """Exact values of a tensor as a float64 numpy array (bf16 widens exactly)."""
    if x is None:
        return None
    return x.detach().to("cpu", torch.float64).numpy()
