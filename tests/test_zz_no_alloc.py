"""kda_chunk_forward_static_ws (two-pass prefill on the library's built-in scratch)
against kda_chunk_forward_ex with a caller-allocated workspace, on two consecutive
calls with different inputs (GPU).

Both run the same kernels on the same inputs, so the results must be bit-identical;
the second call checks that nothing of the first call's scratch content leaks into
it.  The file is named to be collected last, and the test passes on its own as well
as after the rest of the suite (it assumes nothing about earlier use of the
scratch)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_85_b200 as kda
from gated_delta_rule_85_b200.workloads import PrefillShape, prefill_inputs

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16


def _pair(d):
    o1, S1 = kda.chunk_forward_static_ws(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"],
                                         d["cu_seqlens"])
    o2, S2 = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"],
                               d["cu_seqlens"], algo="two_pass")
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    return (o1, S1), (o2, S2)


@pytest.mark.parametrize("shape", [
    PrefillShape(B=1, T=1000, H=8, dk=128, dv=128, dtype=BF16),
    PrefillShape(B=2, T=333, H=4, dk=64, dv=128, dtype=BF16),
    PrefillShape(B=1, T=700, H=3, dk=128, dv=64, dtype=BF16, cu_seqlens=(0, 5, 5, 300, 700)),
], ids=["dense_d128", "dense_dk64", "packed_dv64"])
def test_static_scratch_matches_caller_workspace_on_consecutive_calls(shape):
    need = kda.workspace_size(shape.B, shape.T, shape.H, shape.dk, shape.dv,
                              shape.B if shape.cu_seqlens is None else len(shape.cu_seqlens) - 1, algo="two_pass")
    assert 0 < need <= kda.STATIC_WS_BYTES
    dev = torch.device("cuda")
    for seed in (101, 202):   # two consecutive calls, different inputs
        d = prefill_inputs(shape, seed, dev)
        (o1, S1), (o2, S2) = _pair(d)
        assert torch.equal(o1, o2), f"o differs (seed {seed})"
        assert torch.equal(S1, S2), f"final state differs (seed {seed})"
        assert np.isfinite(o1.float().cpu().numpy()).all()


def test_static_scratch_oversize_takes_the_fused_schedule():
    """Sizes whose two-pass scratch would not fit the built-in array run the fused
    schedule, which needs no scratch: bit-identical to kda_chunk_forward_ex with
    algo=fused, on two consecutive calls."""
    shape = PrefillShape(B=1, T=8192, H=32, dk=128, dv=128, dtype=BF16)
    need = kda.workspace_size(1, 8192, 32, 128, 128, 1, algo="two_pass")
    assert need > kda.STATIC_WS_BYTES
    dev = torch.device("cuda")
    for seed in (7, 8):
        d = prefill_inputs(shape, seed, dev)
        o1, S1 = kda.chunk_forward_static_ws(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"])
        o2, S2 = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"],
                                   algo="fused")
        torch.cuda.synchronize()
        assert kda.device_status() == 0
        assert torch.equal(o1, o2) and torch.equal(S1, S2), f"differs from the fused schedule (seed {seed})"
