"""Gated DeltaNet mode (one decay rate per token-head; kda_gdn_chunk_forward,
kda_gdn_recurrent_step) against the fp64 oracle run on the same gate broadcast
over the key channels -- the oracle's own "scalar gate" pin checks that reading.
Every prefill schedule, both dtypes, ragged and packed inputs, decode, and
prefill followed by decode."""
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


def _oracle(d, dk):
    g = np.repeat(to_f64(d["log_alpha"])[..., None], dk, axis=-1)
    cu = None if d.get("cu_seqlens") is None else d["cu_seqlens"].cpu().numpy()
    s0 = None if d.get("init_state") is None else to_f64(d["init_state"])
    return oracle.forward(to_f64(d["q"]), to_f64(d["k"]), to_f64(d["v"]), g, to_f64(d["beta"]), init_state=s0,
                          cu_seqlens=cu)


@pytest.mark.parametrize("algo,dtype", [("fused", BF16), ("two_pass", BF16), ("auto", torch.float32)])
@pytest.mark.parametrize("dk,dv,T,packed", [(128, 128, 517, False), (64, 128, 200, False), (128, 64, 0, True)])
def test_gdn_prefill(algo, dtype, dk, dv, T, packed):
    if packed:
        lens = [70, 0, 129, 1, 200]
        shape = PrefillShape(B=1, T=sum(lens), H=3, dk=dk, dv=dv, dtype=dtype, gate="scalar",
                             cu_seqlens=tuple(np.cumsum([0] + lens).tolist()))
    else:
        shape = PrefillShape(B=2, T=T, H=3, dk=dk, dv=dv, dtype=dtype, gate="scalar")
    d = prefill_inputs(shape, 61 + dk + dv, DEV)
    assert d["log_alpha"].shape == d["beta"].shape
    o, S = kda.gdn_chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"],
                                 d["cu_seqlens"], algo=algo)
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    o_ref, S_ref = _oracle(d, dk)
    assert_close(to_f64(o), o_ref, dtype, "o")
    assert_close(to_f64(S), S_ref, dtype, "final state")


@pytest.mark.parametrize("dtype", [BF16, torch.float32])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64)])
def test_gdn_prefill_then_decode(dtype, dk, dv):
    H, T0, steps = 2, 150, 12
    shape = PrefillShape(B=2, T=T0, H=H, dk=dk, dv=dv, dtype=dtype, gate="scalar")
    d = prefill_inputs(shape, 71, DEV)
    o, S = kda.gdn_chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"])
    dshape = DecodeShape(N=2, H=H, dk=dk, dv=dv, steps=steps, dtype=dtype, gate="scalar")
    dec = [decode_step_inputs(dshape, t, 72, DEV) for t in range(steps)]
    o_dec = [kda.gdn_recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S) for x in dec]
    torch.cuda.synchronize()
    cat = {key: np.concatenate([to_f64(d[key]), np.stack([to_f64(x[key]) for x in dec], axis=1)], axis=1)
           for key in ("q", "k", "v", "log_alpha", "beta")}
    cat["log_alpha"] = np.repeat(cat["log_alpha"][..., None], dk, axis=-1)
    o_ref, S_ref = oracle.forward(cat["q"], cat["k"], cat["v"], cat["log_alpha"], cat["beta"],
                                  init_state=to_f64(d["init_state"]))
    assert_close(to_f64(o), o_ref[:, :T0], dtype, "prefill o")
    assert_close(np.stack([to_f64(x) for x in o_dec], axis=1), o_ref[:, T0:], dtype, "decode o")
    assert_close(to_f64(S), S_ref, dtype, "state")


def test_gdn_equals_kda_with_a_broadcast_gate():
    """The scalar-gate path and the per-channel path given the broadcast gate take
    the same arithmetic: identical results."""
    shape = PrefillShape(B=1, T=300, H=2, dk=128, dv=128, dtype=BF16, gate="scalar")
    d = prefill_inputs(shape, 81, DEV)
    g_full = d["log_alpha"].unsqueeze(-1).expand(*d["log_alpha"].shape, 128).contiguous()
    for algo in ("fused", "two_pass"):
        o1, S1 = kda.gdn_chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"], algo=algo)
        o2, S2 = kda.chunk_forward(d["q"], d["k"], d["v"], g_full, d["beta"], d["init_state"], algo=algo)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(S1, S2), algo
    x = decode_step_inputs(DecodeShape(N=3, H=2, dk=128, dv=128, steps=1, dtype=BF16, gate="scalar"), 0, 82, DEV)
    S_a = d["init_state"].new_zeros((3, 2, 128, 128)).normal_(0, 0.01)
    S_b = S_a.clone()
    oa = kda.gdn_recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S_a)
    ob = kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"].unsqueeze(-1).expand(3, 2, 128).contiguous(),
                            x["beta"], S_b)
    torch.cuda.synchronize()
    assert torch.equal(oa, ob) and torch.equal(S_a, S_b)
