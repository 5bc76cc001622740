#!/usr/bin/env python
"""KDA operator benchmark: chunked-prefill and decode tokens/s on B200.

One step = one chunked prefill (kda_chunk_forward, tcgen05 kernel) of the
"prefill_8k" workload: B=1, T=8192, H=32, dk=dv=128, bf16 q/k/v, fp32 gates,
fp32 initial state, 64-token chunks.  The decode workload (N=256 sequences,
H=32, one token per step through kda_recurrent_step, fresh inputs per step) is
timed in the same run and reported under "decode"; the backward of the
prefill_8k workload (kda_chunk_backward) under "backward_8k"; the same prefill on raw
inputs through the fused prologue under "prefill_prologue_8k"; the 128k-token prefill
(T=131072) under "prefill_128k"; the 1,048,576-token packed prefill under
"prefill_varlen_1m" and the 256 decode steps of its 22 sequences under
"decode_varlen_22".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line.  For N > 1 it runs under torch.distributed (one process
per GPU); every rank processes its own full workload (weak scaling, no
collective on the data path) and the step time is the max over ranks.
--impl reference times the fp64 CPU oracle (the reference arm) on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PREFILL = dict(B=1, T=8192, H=32, dk=128, dv=128)
PREFILL_LONG = dict(B=1, T=131072, H=32, dk=128, dv=128)
DECODE = dict(N=256, H=32, dk=128, dv=128, steps=1024)
DECODE_VARLEN = dict(N=22, H=32, dk=128, dv=128, steps=256)
CHUNK = 64
# Algorithmic bytes per token-head: q, k, v (bf16) + log_alpha (fp32) + beta + o (bf16).
PREFILL_BYTES_PER_TOKEN_HEAD = 3 * 2 * 128 + 4 * 128 + 4 + 2 * 128          # 1540
STATE_BYTES = 4 * 128 * 128                                                   # one fp32 state
# Algorithmic flops per token-head of the chunked form (C x C products at full size
# plus the three C x d^2 state products): 10 C d + 6 d^2.
PREFILL_FLOPS_PER_TOKEN_HEAD = 10 * CHUNK * 128 + 6 * 128 * 128               # 180224
DECODE_BYTES_PER_PAIR = 2 * STATE_BYTES + PREFILL_BYTES_PER_TOKEN_HEAD        # 132612
# Backward, per token-head: q, k, v, d_o (bf16) + log_alpha + beta read, dq, dk, dv
# (bf16) + dlog_alpha + dbeta written; per (sequence, head) init_state and
# dfinal_state read, dinit_state written.  Flops: the gradient of every forward
# product is two products of the same size (recomputation is not credited).
BACKWARD_BYTES_PER_TOKEN_HEAD = 4 * 2 * 128 + 4 * 128 + 4 + 3 * 2 * 128 + 4 * 128 + 4   # 2824
BACKWARD_FLOPS_PER_TOKEN_HEAD = 2 * PREFILL_FLOPS_PER_TOKEN_HEAD                      # 360448
# The tensor-core backward of bf16 inputs with dk = dv = 128: three launches per call.
BACKWARD_KERNELS = "chunk_intra_kernel (with the backward extras) + bwd_sweeps_kernel + bwd_grad_kernel"
BACKWARD_LAUNCHES = 3
BACKWARD_REPS = 100   # ~0.1 s of backward_8k calls in the timed region
# Fused prologue, per token-head: raw q, k, v and the gate pre-activation (bf16), beta, o.
PROLOGUE_BYTES_PER_TOKEN_HEAD = 3 * 2 * 128 + 2 * 128 + 4 + 2 * 128                    # 1284
# DRAM bytes (read + write) per launch, taken from ncu captures (dram__bytes_read.sum +
# dram__bytes_write.sum) of the current kernels on these workloads; keyed by the kernels
# one step runs.  A kernel set without a capture on its workload reports null.
NCU_TRAFFIC = {
    ("prefill_8k", "chunk_intra_kernel + chunk_inter_kernel"): 272.3e6 + 185.0e6 + 308.4e6 + 50.4e6,
    # chunk_tc_kernel (--algo fused): captured before its timeout-path change, so reported null
    ("decode_b256", "decode_step_kernel"): 547.4e6 + 481.2e6,
    # backward: the three kernels of one call (read + write of each)
    ("backward_T8192", "bwd"): 274.2e6 + 287.8e6 + 492.7e6 + 232.3e6 + 912.7e6 + 311.0e6,
}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


_SAMPLER_CHILD = r"""
import select, sys, time
import pynvml
pynvml.nvmlInit()
uuid, index, period = sys.argv[1], int(sys.argv[2]), float(sys.argv[3])
h = None
if uuid:
    try:
        h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
    except Exception:
        h = None
if h is None:
    h = pynvml.nvmlDeviceGetHandleByIndex(index)
print("ready", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM), flush=True)
out = []
while not select.select([sys.stdin], [], [], period)[0]:
    t = time.monotonic()
    try:
        out.append((t, pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                    int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))))
    except Exception:
        pass
sys.stdout.write("".join(f"{t!r} {c} {r}\n" for t, c, r in out))
"""


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while a timed region runs.

    The reads happen in a child process (an NVML read can take ~0.2 ms, and a
    sampler thread in this process would compete with the launch loop for the
    interpreter); samples whose CLOCK_MONOTONIC time falls between entering and
    leaving the `with` block are kept."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.0005):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self.error = None
        self._index = device_index
        self._period = period_s
        self._proc = None
        self._t0 = self._t1 = None

    def _uuid(self) -> str:
        try:
            import torch

            u = str(torch.cuda.get_device_properties(self._index).uuid)
            return u if u.startswith("GPU-") else "GPU-" + u
        except Exception:  # noqa: BLE001
            return ""

    def poll(self, event):
        """Kept for the call sites: the child process samples on its own."""

    def __enter__(self):
        import subprocess

        try:
            self._proc = subprocess.Popen(
                [sys.executable, "-c", _SAMPLER_CHILD, self._uuid(), str(self._index), str(self._period)],
                stdin=subprocess.PIPE, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            line = self._proc.stdout.readline().split()
            if not line or line[0] != "ready":
                raise RuntimeError("NVML sampler did not start")
            self.max_mhz = int(line[1])
        except Exception as e:  # noqa: BLE001
            self.error = str(e)
            self._stop_child()
        self._t0 = time.monotonic()
        return self

    def _stop_child(self):
        if self._proc is None:
            return ""
        try:
            out, _ = self._proc.communicate(input="stop\n", timeout=30)
        except Exception:  # noqa: BLE001
            self._proc.kill()
            out = ""
        self._proc = None
        return out

    def __exit__(self, *exc):
        self._t1 = time.monotonic()
        for row in self._stop_child().splitlines():
            t, c, r = row.split()
            if self._t0 <= float(t) <= self._t1:
                self.samples.append(int(c))
                self.reasons |= int(r)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def _time_reps(dev, stream, reps, step):
    """CUDA-event time (ms) of `reps` calls of step() on `stream`, and the NVML clocks
    sampled while they run (from this thread too once the launches are queued)."""
    import torch

    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        e0.record(stream)
        for _ in range(reps):
            step()
        e1.record(stream)
        clk.poll(e1)
        torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1), clk.summary()


def _job_tokens_per_s(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput under weak scaling: every rank processes its own full
    workload in the step time (already the max over ranks)."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


def run_prefill(args, world, rank, dev):
    import torch

    import gated_delta_rule_85_b200 as kda
    from gated_delta_rule_85_b200.workloads import PrefillShape, prefill_inputs

    shape = PrefillShape(**PREFILL, dtype=torch.bfloat16)
    d = prefill_inputs(shape, seed=rank, device=dev)
    o = torch.empty((1, PREFILL["T"], PREFILL["H"], PREFILL["dv"]), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((1, PREFILL["H"], 128, 128), dtype=torch.float32, device=dev)
    ws_n = kda.workspace_size(1, PREFILL["T"], PREFILL["H"], 128, 128, 1, algo=args.algo)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=dev) if ws_n else None
    # the two-pass schedule (two kernels per call) is exactly the one that needs a workspace
    kernels = ["chunk_intra_kernel", "chunk_inter_kernel"] if ws_n else ["chunk_tc_kernel"]
    stream = torch.cuda.current_stream(dev)

    def step():
        kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"], None,
                          o=o, final_state=fs, workspace=ws, algo=args.algo)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if kda.device_status() != 0:
        raise RuntimeError("device status flags set after warm-up")
    if not (torch.isfinite(o.float()).all() and torch.isfinite(fs).all()):
        raise RuntimeError("non-finite prefill output")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    _barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clk:
        t_all0 = torch.cuda.Event(enable_timing=True)
        t_all1 = torch.cuda.Event(enable_timing=True)
        t_all0.record(stream)
        h0 = time.perf_counter()
        for i in range(args.steps):
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        t_all1.record(stream)
        host_ms = (time.perf_counter() - h0) * 1e3 / args.steps   # host time to enqueue one step
        clk.poll(t_all1)
        torch.cuda.synchronize(dev)
    _barrier(world)
    total_ms = t_all0.elapsed_time(t_all1)
    per_launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = _max_over_ranks(total_ms, world, dev)

    if args.no_e2e:
        return dict(total_ms=total_ms, per_launch_ms=per_launch_ms, clocks=clk.summary(), e2e_ms=float("nan"),
                    h2d=0, d2h=0, e2e_steps=0, kernels=kernels, host_ms=host_ms)
    # End to end through the public API with host buffers: H2D of every input,
    # the kernel, D2H of o and the final state, every step.
    host = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in d.items()}
    h2d = sum(v.numel() * v.element_size() for k, v in host.items() if v is not None)
    d2h = o.numel() * o.element_size() + fs.numel() * fs.element_size()
    o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    fs_h = torch.empty(fs.shape, dtype=fs.dtype, pin_memory=True)
    e2e_steps = max(2, min(args.steps, 10))
    kda.chunk_forward(host["q"], host["k"], host["v"], host["log_alpha"], host["beta"], host["init_state"],
                      None, o=o_h, final_state=fs_h, algo=args.algo)
    _barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        kda.chunk_forward(host["q"], host["k"], host["v"], host["log_alpha"], host["beta"], host["init_state"],
                          None, o=o_h, final_state=fs_h, algo=args.algo)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = _max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)
    del d
    return dict(total_ms=total_ms, per_launch_ms=per_launch_ms, clocks=clk.summary(), e2e_ms=e2e_ms,
                h2d=h2d, d2h=d2h, e2e_steps=e2e_steps, kernels=kernels, host_ms=host_ms)


def run_prefill_gdn(args, world, rank, dev):
    """prefill_8k with a Gated DeltaNet scalar gate (kda_gdn_chunk_forward), CUDA events per call."""
    import torch

    import gated_delta_rule_85_b200 as kda
    from gated_delta_rule_85_b200.workloads import PrefillShape, prefill_inputs

    shape = PrefillShape(**PREFILL, dtype=torch.bfloat16, gate="scalar")
    d = prefill_inputs(shape, seed=rank, device=dev)
    o = torch.empty((1, PREFILL["T"], PREFILL["H"], PREFILL["dv"]), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((1, PREFILL["H"], 128, 128), dtype=torch.float32, device=dev)
    ws_n = kda.workspace_size(1, PREFILL["T"], PREFILL["H"], 128, 128, 1)
    ws = torch.empty(ws_n, dtype=torch.uint8, device=dev) if ws_n else None

    def step():
        kda.gdn_chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"], o=o,
                              final_state=fs, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    reps = 300
    _barrier(world)
    total, clocks = _time_reps(dev, stream, reps, step)
    ms = _max_over_ranks(total / reps, world, dev)
    del d
    return dict(ms=ms, launches=reps * (2 if ws_n else 1), clocks=clocks)


def run_prefill_prologue(args, world, rank, dev):
    """prefill_8k on raw inputs through the fused prologue (kda_chunk_forward_prologue), CUDA events per call."""
    import torch

    import gated_delta_rule_85_b200 as kda
    from gated_delta_rule_85_b200.workloads import PrefillShape, prefill_inputs

    shape = PrefillShape(**PREFILL, dtype=torch.bfloat16, inputs="raw")
    d = prefill_inputs(shape, seed=rank, device=dev)
    o = torch.empty((1, PREFILL["T"], PREFILL["H"], PREFILL["dv"]), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((1, PREFILL["H"], 128, 128), dtype=torch.float32, device=dev)
    ws = torch.empty(kda.workspace_size(1, PREFILL["T"], PREFILL["H"], 128, 128, 1, algo="two_pass"),
                     dtype=torch.uint8, device=dev)

    def step():
        kda.chunk_forward_prologue(d["q"], d["k"], d["v"], d["gate_x"], d["beta"], d["init_state"], o=o,
                                   final_state=fs, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    reps = 300
    _barrier(world)
    total, clocks = _time_reps(dev, stream, reps, step)
    ms = _max_over_ranks(total / reps, world, dev)
    del d
    return dict(ms=ms, launches=reps * 2, clocks=clocks)


def run_backward(args, world, rank, dev):
    """Backward of the prefill_8k workload (kda_chunk_backward), CUDA events per call."""
    import torch

    import gated_delta_rule_85_b200 as kda
    from gated_delta_rule_85_b200.workloads import PrefillShape, backward_cotangents, prefill_inputs

    cfg = dict(PREFILL, T=args.backward_T)
    shape = PrefillShape(**cfg, dtype=torch.bfloat16)
    d = prefill_inputs(shape, seed=rank, device=dev)
    c = backward_cotangents(shape, seed=rank, device=dev)
    ws = torch.empty(kda.backward_workspace_size(1, cfg["T"], cfg["H"], 128, 128, 1, torch.bfloat16), dtype=torch.uint8,
                     device=dev)
    out = {}

    def step():
        out.update(kda.chunk_backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], c["d_o"],
                                      d["init_state"], c["dfinal_state"], workspace=ws, out=out))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    reps = BACKWARD_REPS
    _barrier(world)
    total, clocks = _time_reps(dev, stream, reps, step)
    ms = _max_over_ranks(total / reps, world, dev)
    del d, c, ws, out
    return dict(ms=ms, launches=reps * BACKWARD_LAUNCHES, clocks=clocks, reps=reps)


def run_prefill_varlen(args, world, rank, dev):
    """The 1,048,576-token packed (varlen) prefill: 22 sequences x 32 heads."""
    import torch

    import gated_delta_rule_85_b200 as kda
    from gated_delta_rule_85_b200.workloads import prefill_inputs, varlen_1m_shape

    shape = varlen_1m_shape()
    d = prefill_inputs(shape, seed=rank, device=dev)
    o = torch.empty((1, shape.T, shape.H, shape.dv), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((shape.num_seqs, shape.H, shape.dk, shape.dv), dtype=torch.float32, device=dev)
    ws_n = kda.workspace_size(1, shape.T, shape.H, shape.dk, shape.dv, shape.num_seqs)
    ws = torch.empty(ws_n, dtype=torch.uint8, device=dev) if ws_n else None
    kernels = ["chunk_intra_kernel", "chunk_inter_kernel"] if ws_n else ["chunk_tc_kernel"]

    def step():
        kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"], d["cu_seqlens"],
                          o=o, final_state=fs, workspace=ws)

    for _ in range(2):
        step()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    reps = 4
    _barrier(world)
    total, clocks = _time_reps(dev, stream, reps, step)
    ms = _max_over_ranks(total / reps, world, dev)
    token_heads = shape.T * shape.H
    alg_bytes = token_heads * PREFILL_BYTES_PER_TOKEN_HEAD + 2 * shape.num_seqs * shape.H * STATE_BYTES
    del d, o, fs
    return dict(ms=ms, tokens=shape.T, alg_bytes=alg_bytes, alg_flops=token_heads * PREFILL_FLOPS_PER_TOKEN_HEAD,
                seqs=shape.num_seqs, launches=reps * len(kernels), kernels=kernels, clocks=clocks)


def run_prefill_long(args, world, rank, dev):
    """The 128k-token prefill (B=1, T=131072, H=32, d=128), kda_chunk_forward (AUTO)."""
    import torch

    import gated_delta_rule_85_b200 as kda
    from gated_delta_rule_85_b200.workloads import PrefillShape, prefill_inputs

    shape = PrefillShape(**PREFILL_LONG, dtype=torch.bfloat16)
    d = prefill_inputs(shape, seed=rank, device=dev)
    o = torch.empty((1, shape.T, shape.H, shape.dv), dtype=torch.bfloat16, device=dev)
    fs = torch.empty((1, shape.H, shape.dk, shape.dv), dtype=torch.float32, device=dev)
    ws_n = kda.workspace_size(1, shape.T, shape.H, shape.dk, shape.dv, 1)
    ws = torch.empty(ws_n, dtype=torch.uint8, device=dev) if ws_n else None
    kernels = ["chunk_intra_kernel", "chunk_inter_kernel"] if ws_n else ["chunk_tc_kernel"]
    # AUTO runs one sequence beyond its workspace budget in windows of launch pairs
    windows = 1
    full = kda.workspace_size(1, shape.T, shape.H, shape.dk, shape.dv, 1, algo="two_pass")
    if ws_n and ws_n < full:
        per_chunk = full // (-(-shape.T // 64) + 1)
        carry = -(-2 * shape.H * shape.dk * shape.dv * 4 // 1024) * 1024
        window = ((ws_n - carry) // per_chunk - 1) * 64
        windows = -(-shape.T // window)

    def step():
        kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"], o=o, final_state=fs,
                          workspace=ws)

    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    reps = 16
    _barrier(world)
    with ClockSampler(dev.index) as clk:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    ms = _max_over_ranks(e0.elapsed_time(e1) / reps, world, dev)
    token_heads = shape.T * shape.H
    alg_bytes = token_heads * PREFILL_BYTES_PER_TOKEN_HEAD + 2 * shape.H * STATE_BYTES
    del d, o, fs, ws
    return dict(ms=ms, tokens=shape.T, alg_bytes=alg_bytes, alg_flops=token_heads * PREFILL_FLOPS_PER_TOKEN_HEAD,
                launches=reps * len(kernels) * windows, kernels=kernels, clocks=clk.summary(), reps=reps,
                workspace_bytes=ws_n, windows=windows)


def run_decode_varlen(args, world, rank, dev):
    """256 decode steps of the 22 packed sequences of the 1M-token workload, one CUDA
    graph per 256 steps (states ~93 MB: L2-resident, launch-bound)."""
    import torch

    import gated_delta_rule_85_b200 as kda
    from gated_delta_rule_85_b200.workloads import DecodeShape, decode_all_steps

    shape = DecodeShape(**DECODE_VARLEN, dtype=torch.bfloat16)
    d = decode_all_steps(shape, seed=rank, device=dev)
    state = d["state"]
    o = torch.empty((shape.N, shape.H, shape.dv), dtype=torch.bfloat16, device=dev)

    def run_all():
        for s in range(shape.steps):
            kda.recurrent_step(d["q"][s], d["k"][s], d["v"][s], d["log_alpha"][s], d["beta"][s], state, o=o)

    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        run_all()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run_all()
    torch.cuda.synchronize(dev)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize(dev)
    reps = 40
    stream = torch.cuda.current_stream(dev)
    _barrier(world)
    with ClockSampler(dev.index) as clk:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    ms = _max_over_ranks(e0.elapsed_time(e1), world, dev)
    if not torch.isfinite(state).all():
        raise RuntimeError("non-finite decode state")
    del g, d, state
    return dict(ms=ms, launches=reps * shape.steps, clocks=clk.summary())


def run_decode(args, world, rank, dev, pool_slots=0):
    """1024 consecutive decode steps of 256 sequences, captured in one CUDA graph.
    With pool_slots > 0 the states live in a pool of that many slots and the
    sequences use a seeded random choice of them (kda_recurrent_step_slots)."""
    import torch

    import gated_delta_rule_85_b200 as kda
    from gated_delta_rule_85_b200.workloads import DecodeShape, decode_all_steps

    shape = DecodeShape(**DECODE, dtype=torch.bfloat16)
    d = decode_all_steps(shape, seed=rank, device=dev)
    state = d["state"]
    o = torch.empty((DECODE["N"], DECODE["H"], 128), dtype=torch.bfloat16, device=dev)
    S = DECODE["steps"]
    if pool_slots:
        g = torch.Generator().manual_seed(1000 + rank)
        slots = torch.randperm(pool_slots, generator=g)[:DECODE["N"]].to(torch.int32).to(dev)
        pool = torch.zeros((pool_slots, DECODE["H"], 128, 128), dtype=torch.float32, device=dev)
        pool[slots.long()] = state
        del state
        state = pool

    def run_all():
        for s in range(S):
            if pool_slots:
                kda.recurrent_step_slots(d["q"][s], d["k"][s], d["v"][s], d["log_alpha"][s], d["beta"][s], state,
                                         slots, o=o)
            else:
                kda.recurrent_step(d["q"][s], d["k"][s], d["v"][s], d["log_alpha"][s], d["beta"][s], state, o=o)

    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        run_all()                       # warm-up (also loads the module)
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run_all()
    torch.cuda.synchronize(dev)
    for _ in range(max(1, args.warmup // 4)):
        g.replay()
    torch.cuda.synchronize(dev)
    reps = max(2, min(args.steps // 10, 10))
    stream = torch.cuda.current_stream(dev)
    _barrier(world)
    with ClockSampler(dev.index) as clk:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    ms = _max_over_ranks(e0.elapsed_time(e1), world, dev)
    if not torch.isfinite(state).all():
        raise RuntimeError("non-finite decode state")
    del g, d, state
    return dict(ms=ms, launches=reps * S, clocks=clk.summary())


def cpu_baseline(heads=32, threads=0):
    """fp64 oracle on the prefill_8k workload (a bounded sample of heads), host cores."""
    import numpy as np
    import torch

    import oracle
    from gated_delta_rule_85_b200.workloads import PrefillShape, prefill_inputs, to_f64

    shape = PrefillShape(**PREFILL, dtype=torch.bfloat16)
    d = prefill_inputs(shape, seed=0, device="cpu")
    arrs = [np.ascontiguousarray(to_f64(d[x])[:, :, :heads]) for x in ("q", "k", "v", "log_alpha", "beta")]
    s0 = np.ascontiguousarray(to_f64(d["init_state"])[:, :heads])
    cores = threads or oracle.max_threads()
    t0 = time.perf_counter()
    oracle.forward(*arrs, init_state=s0, nthreads=cores)
    dt = time.perf_counter() - t0
    token_heads = PREFILL["T"] * heads
    return {"value": token_heads / dt / PREFILL["H"], "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "seconds": dt,
            "sample": f"fp64 token recurrence on {heads} of {PREFILL['H']} heads x {PREFILL['T']} tokens of "
                      f"prefill_8k (rate scaled to all {PREFILL['H']} heads)"}


def config_block(algo="auto"):
    return {"workload": "prefill_8k", "B": PREFILL["B"], "T": PREFILL["T"], "H": PREFILL["H"],
            "dk": PREFILL["dk"], "dv": PREFILL["dv"], "chunk": CHUNK, "global_batch": PREFILL["B"],
            "seq_len": PREFILL["T"], "parallelism": "replicas", "schedule": algo,
            "l2": "inputs larger than L2 (408 MB per step vs 126 MB)"}


def main_reference(args):
    world, rank, _ = _dist()
    if rank != 0:
        return 0
    samples = []
    heads = 16
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(heads=heads)
        if i >= args.warmup:
            samples.append(r)
    secs = [s["seconds"] for s in samples]
    value = statistics.median([s["value"] for s in samples])
    line = {
        "impl": "reference", "metric": "KDA chunked prefill tokens/s (B=1, T=8192, H=32, d=128)",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.median(secs) * PREFILL["H"] / heads, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config_block(),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": samples[0]["cores"], "kind": "oracle",
                         "sample": samples[0]["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def backward_block(args, world, bw, hbm_gbs, bf16_tflops):
    T, H = args.backward_T, PREFILL["H"]
    bbytes = T * H * BACKWARD_BYTES_PER_TOKEN_HEAD + 3 * H * STATE_BYTES
    bflops = T * H * BACKWARD_FLOPS_PER_TOKEN_HEAD
    bgbs = bbytes / (bw["ms"] * 1e-3) / 1e9
    btf = bflops / (bw["ms"] * 1e-3) / 1e12
    return {
        "metric": f"KDA chunked backward tokens/s (gradients of the prefill: B=1, T={T}, H={H}, d=128)",
        "value": world * T / (bw["ms"] * 1e-3), "unit": "tokens/s", "ms_per_step": bw["ms"],
        "roofline": {"kernel": BACKWARD_KERNELS,
                     "bound": "hbm", "achieved": bgbs, "peak": hbm_gbs, "unit": "GB/s", "frac": bgbs / hbm_gbs,
                     "traffic": NCU_TRAFFIC.get((f"backward_T{T}", "bwd")), "algorithmic_bytes": bbytes,
                     "tensor": {"achieved_tflops": btf, "peak_tflops": bf16_tflops, "frac": btf / bf16_tflops,
                                "algorithmic_flops": bflops}},
        "calls": bw["reps"], "clocks": bw["clocks"],
    }


def main_backward_only(args, world, rank, dev):
    bw = run_backward(args, world, rank, dev)
    hbm_gbs, bf16_tflops, _ = _peaks()
    line = backward_block(args, world, bw, hbm_gbs, bf16_tflops)
    line.update({"n_gpus": world, "steps": bw["reps"], "warmup": args.warmup,
                 "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                 "data": "synthetic", "config": {"workload": f"backward T={args.backward_T} H=32 d=128 bf16"},
                 "gpu_launches": bw["launches"]})
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="kda", choices=["kda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end timing")
    ap.add_argument("--no-varlen", action="store_true", help="skip the 1M-token packed prefill line")
    ap.add_argument("--no-slots", action="store_true", help="skip the state-pool decode line")
    ap.add_argument("--no-gdn", action="store_true", help="skip the Gated DeltaNet (scalar gate) prefill line")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward (gradients) line")
    ap.add_argument("--no-prologue", action="store_true", help="skip the fused-prologue (raw inputs) prefill line")
    ap.add_argument("--no-long", action="store_true", help="skip the 128k-token prefill line")
    ap.add_argument("--no-varlen-decode", action="store_true", help="skip the 22-sequence decode line")
    ap.add_argument("--only-backward", action="store_true",
                    help="time only the backward and print its line (profiling a smaller --backward-T)")
    ap.add_argument("--backward-T", type=int, default=PREFILL["T"], help="tokens of the backward workload")
    ap.add_argument("--algo", default="auto", choices=["auto", "fused", "two_pass"],
                    help="tensor-core prefill schedule of the headline line (kda_chunk_forward_ex)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        return main_reference(args)

    import torch

    world, rank, local = _dist()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    import gated_delta_rule_85_b200 as kda

    kda.load_library()

    if args.only_backward:
        rc = main_backward_only(args, world, rank, dev)
        if world > 1:
            import torch.distributed as dist

            dist.barrier()
            dist.destroy_process_group()
        return rc
    pre = run_prefill(args, world, rank, dev)
    dec = None if args.no_decode else run_decode(args, world, rank, dev)
    dsl = None if (args.no_decode or args.no_slots) else run_decode(args, world, rank, dev, pool_slots=512)
    vl = None if args.no_varlen else run_prefill_varlen(args, world, rank, dev)
    gd = None if args.no_gdn else run_prefill_gdn(args, world, rank, dev)
    bw = None if args.no_backward else run_backward(args, world, rank, dev)
    pr = None if args.no_prologue else run_prefill_prologue(args, world, rank, dev)
    lg = None if args.no_long else run_prefill_long(args, world, rank, dev)
    dv22 = None if args.no_varlen_decode else run_decode_varlen(args, world, rank, dev)

    hbm_gbs, bf16_tflops, peak_src = _peaks()
    ms_step = pre["total_ms"] / args.steps
    tokens = PREFILL["B"] * PREFILL["T"]
    value = _job_tokens_per_s(world, tokens, ms_step)
    token_heads = tokens * PREFILL["H"]
    alg_bytes = token_heads * PREFILL_BYTES_PER_TOKEN_HEAD + 2 * PREFILL["H"] * STATE_BYTES
    alg_flops = token_heads * PREFILL_FLOPS_PER_TOKEN_HEAD
    launch_ms = statistics.mean(pre["per_launch_ms"])
    gbs = alg_bytes / (launch_ms * 1e-3) / 1e9
    tflops = alg_flops / (launch_ms * 1e-3) / 1e12
    line = {
        "metric": "KDA chunked prefill tokens/s (B=1, T=8192, H=32, d=128)",
        "value": value, "unit": "tokens/s",
        # the decode half of the metric up front (its full block is "decode" below)
        "decode_tokens_per_s": None, "decode_ms_per_step": None, "decode_hbm_frac": None,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic", "config": config_block(args.algo),
        "roofline": {"kernel": " + ".join(pre["kernels"]), "bound": "hbm", "achieved": gbs, "peak": hbm_gbs,
                     "unit": "GB/s", "frac": gbs / hbm_gbs,
                     "traffic": NCU_TRAFFIC.get(("prefill_8k", " + ".join(pre["kernels"]))),
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else peak_src,
                     "algorithmic_bytes": alg_bytes, "launch_ms": launch_ms,
                     "tensor": {"achieved_tflops": tflops, "peak_tflops": bf16_tflops,
                                "frac": tflops / bf16_tflops, "algorithmic_flops": alg_flops}},
        "e2e": {"value": world * tokens / (pre["e2e_ms"] * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": pre["h2d"], "d2h_bytes_per_step": pre["d2h"],
                "api": "gated_delta_rule_85_b200.chunk_forward with pinned host tensors"},
        "gpu_launches": args.steps * len(pre["kernels"]),
        "clocks": pre["clocks"],
        # host time to enqueue one step (events + the API call); below ms_per_step the GPU never waits
        "host_enqueue_ms_per_step": pre["host_ms"],
    }
    if dec is not None:
        step_ms = dec["ms"] / dec["launches"]
        dbytes = DECODE["N"] * DECODE["H"] * DECODE_BYTES_PER_PAIR
        dgbs = dbytes / (step_ms * 1e-3) / 1e9
        line["decode"] = {
            "metric": "KDA decode tokens/s (N=256 sequences, H=32, d=128, 1 token per step)",
            "value": world * DECODE["N"] / (step_ms * 1e-3), "unit": "tokens/s", "ms_per_step": step_ms,
            "steps": dec["launches"], "graph": "1024 steps per CUDA graph replay",
            "roofline": {"kernel": "decode_step_kernel", "bound": "hbm", "achieved": dgbs, "peak": hbm_gbs,
                         "unit": "GB/s", "frac": dgbs / hbm_gbs,
                         "traffic": NCU_TRAFFIC.get(("decode_b256", "decode_step_kernel")),
                         "algorithmic_bytes": dbytes},
            "clocks": dec["clocks"],
        }
        line["gpu_launches"] += dec["launches"]
        line["decode_tokens_per_s"] = line["decode"]["value"]
        line["decode_ms_per_step"] = step_ms
        line["decode_hbm_frac"] = dgbs / hbm_gbs
    if gd is not None:
        gbytes = token_heads * (PREFILL_BYTES_PER_TOKEN_HEAD - 4 * 128 + 4) + 2 * PREFILL["H"] * STATE_BYTES
        ggbs = gbytes / (gd["ms"] * 1e-3) / 1e9
        gtf = alg_flops / (gd["ms"] * 1e-3) / 1e12
        line["prefill_gdn_8k"] = {
            "metric": "Gated DeltaNet (scalar gate) chunked prefill tokens/s (B=1, T=8192, H=32, d=128)",
            "value": world * tokens / (gd["ms"] * 1e-3), "unit": "tokens/s", "ms_per_step": gd["ms"],
            "roofline": {"kernel": "chunk_intra_kernel + chunk_inter_kernel (scalar gate)", "bound": "hbm",
                         "achieved": ggbs, "peak": hbm_gbs, "unit": "GB/s", "frac": ggbs / hbm_gbs, "traffic": None,
                         "algorithmic_bytes": gbytes,
                         "tensor": {"achieved_tflops": gtf, "peak_tflops": bf16_tflops, "frac": gtf / bf16_tflops}},
            "clocks": gd["clocks"],
        }
        line["gpu_launches"] += gd["launches"]
    if pr is not None:
        pbytes = token_heads * PROLOGUE_BYTES_PER_TOKEN_HEAD + 2 * PREFILL["H"] * STATE_BYTES
        pgbs = pbytes / (pr["ms"] * 1e-3) / 1e9
        ptf = alg_flops / (pr["ms"] * 1e-3) / 1e12
        line["prefill_prologue_8k"] = {
            "metric": "KDA chunked prefill tokens/s on raw inputs, q/k normalisation and gate in the kernel "
                      "(B=1, T=8192, H=32, d=128)",
            "value": world * tokens / (pr["ms"] * 1e-3), "unit": "tokens/s", "ms_per_step": pr["ms"],
            "roofline": {"kernel": "chunk_intra_kernel (prologue) + chunk_inter_kernel", "bound": "hbm",
                         "achieved": pgbs, "peak": hbm_gbs, "unit": "GB/s", "frac": pgbs / hbm_gbs, "traffic": None,
                         "algorithmic_bytes": pbytes,
                         "tensor": {"achieved_tflops": ptf, "peak_tflops": bf16_tflops, "frac": ptf / bf16_tflops}},
            "clocks": pr["clocks"],
        }
        line["gpu_launches"] += pr["launches"]
    if bw is not None:
        line["backward_8k"] = backward_block(args, world, bw, hbm_gbs, bf16_tflops)
        line["gpu_launches"] += bw["launches"]
    if dsl is not None:
        step_ms = dsl["ms"] / dsl["launches"]
        dbytes = DECODE["N"] * DECODE["H"] * DECODE_BYTES_PER_PAIR + DECODE["N"] * 4   # + the slot table
        dgbs = dbytes / (step_ms * 1e-3) / 1e9
        line["decode_slots"] = {
            "metric": "KDA decode tokens/s on a state pool (N=256 sequences in 512 slots, H=32, d=128)",
            "value": world * DECODE["N"] / (step_ms * 1e-3), "unit": "tokens/s", "ms_per_step": step_ms,
            "steps": dsl["launches"], "graph": "1024 steps per CUDA graph replay",
            "roofline": {"kernel": "decode_step_kernel (slot table)", "bound": "hbm", "achieved": dgbs,
                         "peak": hbm_gbs, "unit": "GB/s", "frac": dgbs / hbm_gbs, "traffic": None,
                         "algorithmic_bytes": dbytes},
            "clocks": dsl["clocks"],
        }
        line["gpu_launches"] += dsl["launches"]
    if vl is not None:
        vgbs = vl["alg_bytes"] / (vl["ms"] * 1e-3) / 1e9
        vtf = vl["alg_flops"] / (vl["ms"] * 1e-3) / 1e12
        line["prefill_varlen_1m"] = {
            "metric": "KDA packed (varlen) prefill tokens/s (1,048,576 tokens in 22 sequences, H=32, d=128)",
            "value": world * vl["tokens"] / (vl["ms"] * 1e-3), "unit": "tokens/s", "ms_per_step": vl["ms"],
            "roofline": {"kernel": " + ".join(vl["kernels"]), "bound": "hbm", "achieved": vgbs, "peak": hbm_gbs,
                         "unit": "GB/s", "frac": vgbs / hbm_gbs, "traffic": None,
                         "algorithmic_bytes": vl["alg_bytes"],
                         "tensor": {"achieved_tflops": vtf, "peak_tflops": bf16_tflops, "frac": vtf / bf16_tflops}},
            "clocks": vl["clocks"],
        }
        line["gpu_launches"] += vl["launches"]
    if lg is not None:
        lgbs = lg["alg_bytes"] / (lg["ms"] * 1e-3) / 1e9
        ltf = lg["alg_flops"] / (lg["ms"] * 1e-3) / 1e12
        line["prefill_128k"] = {
            "metric": "KDA chunked prefill tokens/s (B=1, T=131072, H=32, d=128)",
            "value": world * lg["tokens"] / (lg["ms"] * 1e-3), "unit": "tokens/s", "ms_per_step": lg["ms"],
            "steps": lg["reps"], "gpu_launches": lg["launches"], "workspace_bytes": lg["workspace_bytes"],
            "windows": lg["windows"],
            "roofline": {"kernel": " + ".join(lg["kernels"]), "bound": "hbm", "achieved": lgbs, "peak": hbm_gbs,
                         "unit": "GB/s", "frac": lgbs / hbm_gbs, "traffic": None, "algorithmic_bytes": lg["alg_bytes"],
                         "tensor": {"achieved_tflops": ltf, "peak_tflops": bf16_tflops, "frac": ltf / bf16_tflops}},
            "clocks": lg["clocks"],
        }
        line["gpu_launches"] += lg["launches"]
    if dv22 is not None:
        step_ms = dv22["ms"] / dv22["launches"]
        n22 = DECODE_VARLEN["N"] * DECODE_VARLEN["H"]
        vbytes = n22 * DECODE_BYTES_PER_PAIR
        line["decode_varlen_22"] = {
            "metric": "KDA decode tokens/s after the 1M-token packed prefill (22 sequences, H=32, d=128, "
                      "256 steps per CUDA graph)",
            "value": world * DECODE_VARLEN["N"] / (step_ms * 1e-3), "unit": "tokens/s", "ms_per_step": step_ms,
            "steps": dv22["launches"], "graph": "256 steps per CUDA graph replay",
            "roofline": None,
            "note": f"launch-bound: {vbytes / 1e6:.0f} MB of state per step stays in the 126 MB L2; "
                    f"{vbytes / (step_ms * 1e-3) / 1e9:.0f} GB/s of state traffic, no roofline claim",
            "clocks": dv22["clocks"],
        }
        line["gpu_launches"] += dv22["launches"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(heads=32)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
