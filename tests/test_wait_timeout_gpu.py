"""Failure detection on the GPU without a fault: a bounded wait on an mbarrier that
nothing completes runs out, the CTA flags KDA_DEV_WAIT_TIMEOUT and returns; the host
reads the flag, clears it, and the context keeps working."""
import pytest
import torch

import gated_delta_rule_85_b200 as kda
from gated_delta_rule_85_b200.workloads import PrefillShape, prefill_inputs, to_f64
from kda_testutil import assert_close, oracle_prefill

pytestmark = pytest.mark.gpu


def test_timed_out_wait_is_reported_and_context_survives():
    torch.cuda.init()
    assert kda.device_status() == 0
    kda.debug_wait_timeout(2_000_000)   # about a millisecond of SM cycles
    assert kda.device_status(clear=True) & kda.DEV_WAIT_TIMEOUT
    assert kda.device_status() == 0     # cleared
    d = prefill_inputs(PrefillShape(B=1, T=130, H=2, dk=128, dv=128, dtype=torch.bfloat16), 3, torch.device("cuda"))
    o, S = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"], d["cu_seqlens"])
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    o_ref, S_ref = oracle_prefill(d)
    assert_close(to_f64(o), o_ref, torch.bfloat16, "o")
    assert_close(to_f64(S), S_ref, torch.bfloat16, "final state")
