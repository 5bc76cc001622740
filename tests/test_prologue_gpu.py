"""Fused input prologue (kda_chunk_forward_prologue, kda_recurrent_step_prologue)
against the fp64 oracle run on oracle.prologue of the same raw inputs: q and k
scaled to unit norm over dk, log_alpha = -softplus(gate_x)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_85_b200 as kda
import oracle
from gated_delta_rule_85_b200.workloads import DecodeShape, PrefillShape, decode_step_inputs, prefill_inputs, to_f64
from kda_testutil import assert_close

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16
DEV = torch.device("cuda")


def _oracle(d, heads=None):
    pick = (lambda x: x) if heads is None else (lambda x: x.index_select(2, torch.as_tensor(heads, device=x.device)))
    q, k, g = oracle.prologue(to_f64(pick(d["q"])), to_f64(pick(d["k"])), to_f64(pick(d["gate_x"])))
    s0 = d.get("init_state")
    if s0 is not None and heads is not None:
        s0 = s0.index_select(1, torch.as_tensor(heads, device=s0.device))
    cu = None if d.get("cu_seqlens") is None else d["cu_seqlens"].cpu().numpy()
    return oracle.forward(q, k, to_f64(pick(d["v"])), g, to_f64(pick(d["beta"])),
                          init_state=None if s0 is None else to_f64(s0), cu_seqlens=cu)


@pytest.mark.parametrize("dtype", [BF16, torch.float32])
@pytest.mark.parametrize("B,T,H,dk,dv", [(2, 200, 2, 128, 128), (1, 130, 3, 64, 64), (1, 64, 2, 128, 64),
                                         (3, 1, 2, 64, 128)])
def test_prologue_prefill_matches_oracle(dtype, B, T, H, dk, dv):
    shape = PrefillShape(B=B, T=T, H=H, dk=dk, dv=dv, dtype=dtype, inputs="raw")
    d = prefill_inputs(shape, 300 + T + dk, DEV)
    assert "log_alpha" not in d and d["gate_x"].dtype == dtype
    o, S = kda.chunk_forward_prologue(d["q"], d["k"], d["v"], d["gate_x"], d["beta"], d["init_state"])
    torch.cuda.synchronize()
    o_ref, S_ref = _oracle(d)
    assert_close(to_f64(o), o_ref, dtype, "o")
    assert_close(to_f64(S), S_ref, dtype, "final state")
    assert kda.device_status() == 0


@pytest.mark.parametrize("dtype", [BF16, torch.float32])
def test_prologue_packed_and_decode(dtype):
    """Packed sequences (empty, single-token, ragged), then one decode step from
    the final states on raw inputs; against one oracle recurrence."""
    lens = [70, 0, 129, 1, 64]
    cu = tuple(np.cumsum([0] + lens).tolist())
    shape = PrefillShape(B=1, T=sum(lens), H=3, dk=128, dv=128, dtype=dtype, inputs="raw", cu_seqlens=cu)
    d = prefill_inputs(shape, 41, DEV)
    o, S = kda.chunk_forward_prologue(d["q"], d["k"], d["v"], d["gate_x"], d["beta"], d["init_state"],
                                      d["cu_seqlens"])
    st = decode_step_inputs(DecodeShape(N=len(lens), H=3, dk=128, dv=128, steps=1, dtype=dtype, inputs="raw"), 0,
                            seed=42, device=DEV)
    o_dec = kda.recurrent_step_prologue(st["q"], st["k"], st["v"], st["gate_x"], st["beta"], S)
    torch.cuda.synchronize()
    o_ref, S_ref = _oracle(d)
    assert_close(to_f64(o), o_ref, dtype, "packed o")
    q, k, g = oracle.prologue(to_f64(st["q"]), to_f64(st["k"]), to_f64(st["gate_x"]))
    od_ref, Sd_ref = oracle.step(q, k, to_f64(st["v"]), g, to_f64(st["beta"]), S_ref)
    assert_close(to_f64(o_dec), od_ref, dtype, "decode o")
    assert_close(to_f64(S), Sd_ref, dtype, "decoded state")


def test_prologue_scale_invariance():
    """Scaling q or k rows by any positive factor changes nothing (they are
    normalised inside); the fp32 path shows it to rounding."""
    shape = PrefillShape(B=1, T=150, H=2, dk=64, dv=64, dtype=torch.float32, inputs="raw")
    d = prefill_inputs(shape, 5, DEV)
    o1, S1 = kda.chunk_forward_prologue(d["q"], d["k"], d["v"], d["gate_x"], d["beta"], d["init_state"])
    o2, S2 = kda.chunk_forward_prologue(d["q"] * 8.0, d["k"] * 0.25, d["v"], d["gate_x"], d["beta"], d["init_state"])
    torch.cuda.synchronize()
    torch.testing.assert_close(o1, o2, rtol=1e-5, atol=1e-6)
    torch.testing.assert_close(S1, S2, rtol=1e-5, atol=1e-6)


def test_prologue_rejects_fused_schedule():
    shape = PrefillShape(B=1, T=64, H=1, dk=128, dv=128, dtype=BF16, inputs="raw")
    d = prefill_inputs(shape, 6, DEV)
    with pytest.raises(kda.KDAError):
        kda.chunk_forward_prologue(d["q"], d["k"], d["v"], d["gate_x"], d["beta"], d["init_state"], algo="fused")


@pytest.mark.slow
def test_prologue_prefill_8k_sampled_heads():
    shape = PrefillShape(B=1, T=8192, H=32, dk=128, dv=128, dtype=BF16, inputs="raw")
    d = prefill_inputs(shape, 0, DEV)
    o, S = kda.chunk_forward_prologue(d["q"], d["k"], d["v"], d["gate_x"], d["beta"], d["init_state"])
    torch.cuda.synchronize()
    heads = [0, 13, 31]
    o_ref, S_ref = _oracle(d, heads)
    idx = torch.as_tensor(heads, device=DEV)
    assert_close(to_f64(o.index_select(2, idx)), o_ref, BF16, "o")
    assert_close(to_f64(S.index_select(1, idx)), S_ref, BF16, "final state")
