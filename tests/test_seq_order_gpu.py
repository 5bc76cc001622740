"""Packed (varlen) prefill with many sequences of mixed lengths, which the kernels
take longest first (up to 256 sequences) or in index order (more): every schedule
must give each sequence exactly its own recurrence, whatever order its CTAs ran in.
Covers equal lengths (ties broken by index), empty sequences, exactly 256
sequences (the largest ranked case) and 300 (the index-order case)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_85_b200 as kda
from gated_delta_rule_85_b200.workloads import PrefillShape, prefill_inputs, to_f64
from kda_testutil import assert_close, oracle_prefill

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16


def _lengths(kind, n):
    rng = np.random.default_rng(n)
    if kind == "equal":
        return [96] * n
    L = rng.integers(0, 150, size=n)
    L[::7] = 0                       # some empty sequences
    return L.tolist()


@pytest.mark.parametrize("kind,n", [("equal", 5), ("mixed", 17), ("mixed", 256), ("mixed", 300)])
@pytest.mark.parametrize("algo,simt", [("fused", False), ("two_pass", False), ("auto", True)])
def test_many_packed_sequences(kind, n, algo, simt):
    lens = _lengths(kind, n)
    cu = tuple(np.cumsum([0] + lens).tolist())
    dtype = torch.float32 if simt else BF16
    shape = PrefillShape(B=1, T=cu[-1], H=2, dk=128, dv=128, dtype=dtype, cu_seqlens=cu)
    d = prefill_inputs(shape, 7 + n, torch.device("cuda"))
    o, S = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"], d["cu_seqlens"],
                             simt=simt, algo=algo)
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    o_ref, S_ref = oracle_prefill(d)
    assert_close(to_f64(o), o_ref, dtype, "o")
    assert_close(to_f64(S), S_ref, dtype, "final state")
    for i, L in enumerate(lens):
        if L == 0:   # an empty sequence keeps its initial state exactly
            assert torch.equal(S[i], d["init_state"][i])
