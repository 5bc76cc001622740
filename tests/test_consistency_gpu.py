"""Invariants of the CUDA path (GPU vs GPU and vs the oracle).

The remio.ai page ("Kimi Linear、独自の土俵でFull Attentionを上回る", § "オープンコー
ドにより主張は検証可能になる一方、ソフトウェアスタックはリスクを加える") reports a
recurrent-state layout error in chunked prefill that broke long-context retrieval
while short prompts looked fine, and asks for tests of long prefill, batched
decode and state across chunk boundaries.  These tests check exactly those
hand-offs: prefill split at arbitrary points, prefill followed by decode from its
final state, packed sequences against separate runs, and column equivariance.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_85_b200 as kda
import oracle
from gated_delta_rule_85_b200.workloads import (DecodeShape, PrefillShape, decode_step_inputs, prefill_inputs,
                                                to_f64)
from kda_testutil import assert_close, oracle_prefill, rel_l2

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16


def _fwd(d, sl=slice(None), s0="init", simt=False, algo="auto"):
    init = d["init_state"] if isinstance(s0, str) else s0
    return kda.chunk_forward(d["q"][:, sl].contiguous(), d["k"][:, sl].contiguous(), d["v"][:, sl].contiguous(),
                             d["log_alpha"][:, sl].contiguous(), d["beta"][:, sl].contiguous(), init, simt=simt,
                             algo=algo)


# the tensor-core path under each schedule, and the fp32 CUDA-core path
PATHS = [("fused", False), ("two_pass", False), ("auto", True)]


@pytest.mark.parametrize("split", [64, 100, 320])
@pytest.mark.parametrize("algo,simt", PATHS)
def test_split_prefill_resumes_exactly(split, algo, simt):
    dtype = torch.float32 if simt else BF16
    shape = PrefillShape(B=1, T=500, H=3, dk=128, dv=128, dtype=dtype)
    d = prefill_inputs(shape, 31, torch.device("cuda"))
    o1, S1 = _fwd(d, slice(0, split), simt=simt, algo=algo)
    o2, S2 = _fwd(d, slice(split, None), s0=S1, simt=simt, algo=algo)
    o, S = _fwd(d, simt=simt, algo=algo)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_prefill(d)
    o_cat = np.concatenate([to_f64(o1), to_f64(o2)], axis=1)
    assert_close(o_cat, o_ref, dtype, "split o")
    assert_close(to_f64(S2), S_ref, dtype, "split final state")
    if split % 64 == 0:
        # a split on a chunk boundary performs the same chunk sequence: bit-identical
        assert torch.equal(torch.cat([o1, o2], dim=1), o) and torch.equal(S2, S)


@pytest.mark.parametrize("algo", ["fused", "two_pass"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128)])
def test_prefill_then_decode_matches_one_recurrence(dk, dv, algo):
    """The prefill's final_state is directly the decode state (one layout for both)."""
    T0, steps = 333, 24
    shape = PrefillShape(B=2, T=T0, H=4, dk=dk, dv=dv, dtype=BF16)
    dev = torch.device("cuda")
    d = prefill_inputs(shape, 40, dev)
    o, S = _fwd(d, algo=algo)
    dshape = DecodeShape(N=2, H=4, dk=dk, dv=dv, steps=steps, dtype=BF16)
    dec = [decode_step_inputs(dshape, t, 41, dev) for t in range(steps)]
    o_dec = [kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S) for x in dec]
    torch.cuda.synchronize()
    # one long recurrence over T0 + steps tokens
    cat = {key: np.concatenate([to_f64(d[key]), np.stack([to_f64(x[key]) for x in dec], axis=1)], axis=1)
           for key in ("q", "k", "v", "log_alpha", "beta")}
    o_ref, S_ref = oracle.forward(cat["q"], cat["k"], cat["v"], cat["log_alpha"], cat["beta"],
                                  init_state=to_f64(d["init_state"]))
    assert_close(to_f64(o), o_ref[:, :T0], BF16, "prefill o")
    assert_close(np.stack([to_f64(x) for x in o_dec], axis=1), o_ref[:, T0:], BF16, "decode o")
    assert_close(to_f64(S), S_ref, BF16, "final state")


@pytest.mark.parametrize("algo,simt", PATHS)
def test_packed_equals_separate_runs(algo, simt):
    dtype = torch.float32 if simt else BF16
    lens = [70, 0, 129, 1, 256, 33]
    cu = tuple(np.cumsum([0] + lens).tolist())
    shape = PrefillShape(B=1, T=cu[-1], H=2, dk=128, dv=128, dtype=dtype, cu_seqlens=cu)
    d = prefill_inputs(shape, 50, torch.device("cuda"))
    o, S = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"], d["cu_seqlens"],
                             simt=simt, algo=algo)
    for n, L in enumerate(lens):
        sl = slice(cu[n], cu[n + 1])
        on, Sn = _fwd(d, sl, s0=d["init_state"][n:n + 1].contiguous(), simt=simt, algo=algo)
        torch.cuda.synchronize()
        if L:
            assert rel_l2(to_f64(o[:, sl]), to_f64(on)) < (1e-6 if simt else 5e-3)
        assert rel_l2(to_f64(S[n]), to_f64(Sn[0])) < (1e-6 if simt else 5e-3)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_prefill(d)
    assert_close(to_f64(o), o_ref, dtype, "packed o")
    assert_close(to_f64(S), S_ref, dtype, "packed final state")
    assert torch.equal(S[1], d["init_state"][1])   # empty sequence keeps its state


@pytest.mark.parametrize("algo", ["fused", "two_pass"])
def test_value_column_permutation_is_equivariant(algo):
    shape = PrefillShape(B=1, T=200, H=2, dk=128, dv=128, dtype=BF16)
    d = prefill_inputs(shape, 60, torch.device("cuda"))
    perm = torch.randperm(128, generator=torch.Generator().manual_seed(0)).cuda()
    o, S = _fwd(d, algo=algo)
    d2 = dict(d)
    d2["v"] = d["v"][..., perm].contiguous()
    d2["init_state"] = d["init_state"][..., perm].contiguous()
    o2, S2 = _fwd(d2, algo=algo)
    torch.cuda.synchronize()
    assert rel_l2(to_f64(o2), to_f64(o[..., perm])) < 5e-3
    assert rel_l2(to_f64(S2), to_f64(S[..., perm])) < 5e-3


@pytest.mark.parametrize("algo", ["fused", "two_pass"])
def test_empty_and_zero_length_inputs(algo):
    dev = torch.device("cuda")
    shape = PrefillShape(B=2, T=0, H=2, dk=128, dv=128, dtype=BF16)
    d = prefill_inputs(shape, 70, dev)
    o, S = _fwd(d, algo=algo)
    torch.cuda.synchronize()
    assert o.numel() == 0 and torch.equal(S, d["init_state"])
    o, S = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, algo=algo)
    torch.cuda.synchronize()
    assert torch.count_nonzero(S) == 0
