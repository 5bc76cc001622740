"""kda_chunk_forward_simt (fp32 CUDA-core prefill) vs the fp64 oracle (GPU)."""
import pytest
import torch

import gated_delta_rule_85_b200 as kda
from gated_delta_rule_85_b200.workloads import CONFIGS, PrefillShape, prefill_inputs, to_f64
from kda_testutil import assert_close, oracle_prefill

pytestmark = pytest.mark.gpu


def _check(shape, seed=0, simt=True, heads=None):
    d = prefill_inputs(shape, seed, torch.device("cuda"))
    o, S = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"],
                             d["cu_seqlens"], simt=simt)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_prefill(d, heads)
    o_got, S_got = to_f64(o), to_f64(S)
    if heads is not None:
        o_got, S_got = o_got[:, :, heads], S_got[:, heads]
    assert_close(o_got, o_ref, shape.dtype, "o")
    assert_close(S_got, S_ref, shape.dtype, "final state")


def test_tiny_f32_config():
    """B=1, H=2, T=256, dk=dv=64, fp32, zero initial state (rel-L2 <= 1e-4)."""
    _check(CONFIGS["tiny_f32"], seed=0)


@pytest.mark.parametrize("T", [1, 37, 64, 65, 200])
@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64), (128, 128)])
def test_ragged_lengths_f32(T, dk, dv):
    _check(PrefillShape(B=2, T=T, H=2, dk=dk, dv=dv, dtype=torch.float32), seed=T)


def test_bf16_inputs():
    _check(PrefillShape(B=1, T=300, H=4, dk=128, dv=128, dtype=torch.bfloat16), seed=5)


def test_varlen_f32():
    cu = (0, 5, 5, 133, 200, 264)
    _check(PrefillShape(B=1, T=264, H=2, dk=128, dv=128, dtype=torch.float32, cu_seqlens=cu), seed=7)


def test_no_initial_state():
    _check(PrefillShape(B=1, T=130, H=2, dk=64, dv=64, dtype=torch.float32, init_state="none"), seed=8)
