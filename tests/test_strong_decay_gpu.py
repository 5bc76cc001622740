"""Strong decay: the tensor-core prefill against the fp64 oracle when channels
forget fast -- single-token hard resets (log_alpha = -100), whole chunks at
log_alpha = -2 (a chunk's summed decay -128), channels at -10, and mixtures of
strong and weak channels in one head.

Each channel keeps or discards its memory on its own ("Kimi Delta Attention 徹底
解説" (tech-tide.dev), § "Kimi Delta Attention の仕組み"); a transient cue is meant
to go stale fast while other channels hold on ("Kimi Linear、独自の土俵でFull
Attentionを上回る" (remio.ai), § "Kimi Linearがより賢いRecurrent Memoryを使う方法").
So arbitrarily strong decay is legal input, and every schedule (fused, two-pass,
Gated DeltaNet, fused prologue) must match the oracle on it, with no device flag.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_85_b200 as kda
import oracle
from gated_delta_rule_85_b200.workloads import (DecodeShape, PrefillShape, STRONG_KINDS, decode_step_inputs,
                                                prefill_inputs, strong_decay, to_f64)
from kda_testutil import assert_close, oracle_prefill

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16
DEV = torch.device("cuda")
LENS = [70, 0, 129, 1, 256, 300]


def _shape(dk, dv, T, packed, **kw):
    if packed:
        cu = tuple(np.cumsum([0] + LENS).tolist())
        return PrefillShape(B=1, T=cu[-1], H=2, dk=dk, dv=dv, dtype=BF16, cu_seqlens=cu, **kw)
    return PrefillShape(B=2, T=T, H=2, dk=dk, dv=dv, dtype=BF16, **kw)


def _no_flags():
    torch.cuda.synchronize()
    assert kda.device_status(clear=True) == 0


@pytest.mark.parametrize("kind", STRONG_KINDS)
@pytest.mark.parametrize("algo", ["fused", "two_pass"])
@pytest.mark.parametrize("dk,dv,T,packed", [(128, 128, 300, False), (64, 128, 200, False), (128, 64, 0, True)])
def test_kda_strong_decay_matches_oracle(kind, algo, dk, dv, T, packed):
    d = prefill_inputs(_shape(dk, dv, T, packed), 900 + dk + T, DEV)
    strong_decay(d["log_alpha"], kind, 17)
    kda.device_status(clear=True)
    o, S = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"], d["cu_seqlens"],
                             algo=algo)
    _no_flags()
    o_ref, S_ref = oracle_prefill(d)
    assert_close(to_f64(o), o_ref, BF16, f"{kind} {algo} o")
    assert_close(to_f64(S), S_ref, BF16, f"{kind} {algo} final state")


@pytest.mark.parametrize("kind", STRONG_KINDS)
@pytest.mark.parametrize("algo", ["fused", "two_pass"])
def test_gdn_strong_decay_matches_oracle(kind, algo):
    d = prefill_inputs(_shape(128, 128, 0, True, gate="scalar"), 950, DEV)
    strong_decay(d["log_alpha"], kind, 18)
    kda.device_status(clear=True)
    o, S = kda.gdn_chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"],
                                 d["cu_seqlens"], algo=algo)
    _no_flags()
    g = np.repeat(to_f64(d["log_alpha"])[..., None], 128, axis=-1)
    o_ref, S_ref = oracle.forward(to_f64(d["q"]), to_f64(d["k"]), to_f64(d["v"]), g, to_f64(d["beta"]),
                                  init_state=to_f64(d["init_state"]), cu_seqlens=d["cu_seqlens"].cpu().numpy())
    assert_close(to_f64(o), o_ref, BF16, f"gdn {kind} {algo} o")
    assert_close(to_f64(S), S_ref, BF16, f"gdn {kind} {algo} final state")


@pytest.mark.parametrize("kind", STRONG_KINDS)
@pytest.mark.parametrize("dk,dv,T,packed", [(128, 128, 300, False), (64, 64, 0, True)])
def test_prologue_strong_decay_matches_oracle(kind, dk, dv, T, packed):
    """Gate pre-activations up to +100 (log_alpha = -softplus(x) down to -100)."""
    d = prefill_inputs(_shape(dk, dv, T, packed, inputs="raw"), 970 + dk, DEV)
    strong_decay(d["gate_x"], kind, 19, raw=True)
    kda.device_status(clear=True)
    o, S = kda.chunk_forward_prologue(d["q"], d["k"], d["v"], d["gate_x"], d["beta"], d["init_state"],
                                      d["cu_seqlens"])
    _no_flags()
    q, k, g = oracle.prologue(to_f64(d["q"]), to_f64(d["k"]), to_f64(d["gate_x"]))
    # some 64-token chunk of some channel decays past e^-80 (the tensor cores' strong-decay path)
    n64 = g.shape[1] // 64 * 64
    assert g[:, :n64].reshape(g.shape[0], -1, 64, *g.shape[2:]).sum(axis=2).min() < -80.0
    cu = None if d["cu_seqlens"] is None else d["cu_seqlens"].cpu().numpy()
    o_ref, S_ref = oracle.forward(q, k, to_f64(d["v"]), g, to_f64(d["beta"]), init_state=to_f64(d["init_state"]),
                                  cu_seqlens=cu)
    assert_close(to_f64(o), o_ref, BF16, f"prologue {kind} o")
    assert_close(to_f64(S), S_ref, BF16, f"prologue {kind} final state")


@pytest.mark.parametrize("algo", ["fused", "two_pass"])
def test_strong_decay_prefill_then_decode(algo):
    """Prefill with hard resets, then decode steps from its final state: one recurrence."""
    T0, steps = 250, 8
    d = prefill_inputs(PrefillShape(B=2, T=T0, H=2, dk=128, dv=128, dtype=BF16), 990, DEV)
    strong_decay(d["log_alpha"], "mixed", 20)
    o, S = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"], algo=algo)
    dshape = DecodeShape(N=2, H=2, dk=128, dv=128, steps=steps, dtype=BF16)
    dec = [decode_step_inputs(dshape, t, 991, DEV) for t in range(steps)]
    for x in dec[::2]:
        x["log_alpha"][..., :16] = -100.0
    o_dec = [kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S) for x in dec]
    _no_flags()
    cat = {key: np.concatenate([to_f64(d[key]), np.stack([to_f64(x[key]) for x in dec], axis=1)], axis=1)
           for key in ("q", "k", "v", "log_alpha", "beta")}
    o_ref, S_ref = oracle.forward(cat["q"], cat["k"], cat["v"], cat["log_alpha"], cat["beta"],
                                  init_state=to_f64(d["init_state"]))
    assert_close(to_f64(o), o_ref[:, :T0], BF16, "prefill o")
    assert_close(np.stack([to_f64(x) for x in o_dec], axis=1), o_ref[:, T0:], BF16, "decode o")
    assert_close(to_f64(S), S_ref, BF16, "final state")


def test_strong_decay_fullsize_sampled_heads():
    """prefill_8k (B=1, T=8192, H=32, d=128) with hard resets, the AUTO schedule,
    checked on three sampled heads."""
    d = prefill_inputs(PrefillShape(B=1, T=8192, H=32, dk=128, dv=128, dtype=BF16), 995, DEV)
    strong_decay(d["log_alpha"], "mixed", 21)
    o, S = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"])
    _no_flags()
    heads = [0, 13, 31]
    o_ref, S_ref = oracle_prefill(d, heads)
    idx = torch.as_tensor(heads, device=DEV)
    assert_close(to_f64(o.index_select(2, idx)), o_ref, BF16, "o (sampled heads)")
    assert_close(to_f64(S.index_select(1, idx)), S_ref, BF16, "final state (sampled heads)")
