"""kda_recurrent_step vs the fp64 oracle (GPU)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_85_b200 as kda
import oracle
from gated_delta_rule_85_b200.workloads import DecodeShape, decode_step_inputs, draw_state, to_f64
from kda_testutil import assert_close

pytestmark = pytest.mark.gpu


def _run_steps(shape, steps, seed=0, state_kind="normal"):
    dev = torch.device("cuda")
    S = draw_state((shape.N, shape.H, shape.dk, shape.dv), dev, seed, 6, state_kind)
    S_ref = to_f64(S)
    for t in range(steps):
        d = decode_step_inputs(shape, t, seed, dev)
        o = kda.recurrent_step(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S)
        o_ref, S_ref = oracle.step(*(to_f64(d[x]) for x in ("q", "k", "v", "log_alpha", "beta")), S_ref)
        assert_close(to_f64(o), o_ref, shape.dtype, f"o step {t}")
    torch.cuda.synchronize()
    return to_f64(S), S_ref


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_matches_oracle(dk, dv, dtype):
    shape = DecodeShape(N=5, H=3, dk=dk, dv=dv, steps=0, dtype=dtype)
    S, S_ref = _run_steps(shape, steps=12, seed=dk + dv)
    assert_close(S, S_ref, dtype, "final state")


def test_decode_many_steps_bf16():
    """64 consecutive steps: errors must not accumulate beyond the bf16 bound."""
    shape = DecodeShape(N=16, H=4, dk=128, dv=128, steps=0, dtype=torch.bfloat16)
    S, S_ref = _run_steps(shape, steps=64, seed=3)
    assert_close(S, S_ref, torch.bfloat16, "final state")


def test_decode_full_replacement():
    """beta = 1 and unit keys: reading with the key just written returns v (fp32)."""
    dev = torch.device("cuda")
    shape = DecodeShape(N=3, H=2, dk=128, dv=128, steps=0, dtype=torch.float32)
    S = draw_state((3, 2, 128, 128), dev, 1, 6)
    for t in range(4):
        d = decode_step_inputs(shape, t, 1, dev)
        d["beta"].fill_(1.0)
        o = kda.recurrent_step(d["k"], d["k"], d["v"], d["log_alpha"], d["beta"], S)
        np.testing.assert_allclose(o.cpu().numpy(), d["v"].cpu().numpy(), rtol=0, atol=2e-5)
