"""kda_chunk_forward (tcgen05 tensor-core prefill, bf16) vs the fp64 oracle (GPU),
under both schedules (fused; two-pass with workspace).

Bound for bf16 inputs: rel-L2 <= 1e-2 and max-abs <= 5e-2 on o and the final state."""
import pytest
import torch

import gated_delta_rule_85_b200 as kda
from gated_delta_rule_85_b200.workloads import PrefillShape, prefill_inputs, to_f64
from kda_testutil import assert_close, oracle_prefill, rel_l2

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16
ALGOS = ["fused", "two_pass"]
algo_param = pytest.mark.parametrize("algo", ALGOS)


def _run(shape, seed=0, final_state=True, algo="auto"):
    d = prefill_inputs(shape, seed, torch.device("cuda"))
    o, S = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"],
                             d["cu_seqlens"], final_state=final_state, algo=algo)
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    return d, o, S


def _check(shape, seed=0, algo="auto"):
    d, o, S = _run(shape, seed, algo=algo)
    o_ref, S_ref = oracle_prefill(d)
    assert_close(to_f64(o), o_ref, BF16, "o")
    assert_close(to_f64(S), S_ref, BF16, "final state")


@algo_param
@pytest.mark.parametrize("T", [1, 63, 64, 65, 130, 517])
def test_lengths_d128(T, algo):
    _check(PrefillShape(B=1, T=T, H=2, dk=128, dv=128, dtype=BF16), seed=T, algo=algo)


@algo_param
@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
def test_head_dims(dk, dv, algo):
    _check(PrefillShape(B=2, T=200, H=2, dk=dk, dv=dv, dtype=BF16), seed=dk * 3 + dv, algo=algo)


@algo_param
@pytest.mark.parametrize("B,H,dk,dv", [
    (2, 40, 128, 128),    # 80 chains: fused 32-column tiles, two-pass 64
    (4, 40, 128, 128),    # 160 chains: fused 64, two-pass 128
    (4, 80, 128, 128),    # 320 chains: 128-column tiles
    (4, 80, 64, 128),
    (4, 80, 64, 64),      # dv = 64 -> one 64-column tile
])
def test_value_tile_widths(B, H, dk, dv, algo):
    """The launchers pick the value-tile width from the number of chains; cover each."""
    _check(PrefillShape(B=B, T=150, H=H, dk=dk, dv=dv, dtype=BF16), seed=11 + H + dk, algo=algo)


@algo_param
def test_zero_initial_state_and_no_final_state(algo):
    shape = PrefillShape(B=1, T=150, H=2, dk=128, dv=128, dtype=BF16, init_state="none")
    d, o, S = _run(shape, seed=4, final_state=False, algo=algo)
    assert S is None
    o_ref, _ = oracle_prefill(d)
    assert_close(to_f64(o), o_ref, BF16, "o")


@algo_param
def test_varlen_with_empty_and_short_sequences(algo):
    cu = (0, 0, 1, 64, 64, 200, 391)
    _check(PrefillShape(B=1, T=391, H=3, dk=128, dv=128, dtype=BF16, cu_seqlens=cu), seed=9, algo=algo)


@algo_param
def test_two_schedules_agree(algo):
    """Both schedules compute the same bf16 operands and products; their results
    differ only in accumulation details of the tensor cores."""
    shape = PrefillShape(B=1, T=700, H=3, dk=128, dv=128, dtype=BF16)
    d, o, S = _run(shape, seed=22, algo=algo)
    o2, S2 = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"],
                               algo="two_pass" if algo == "fused" else "fused")
    torch.cuda.synchronize()
    assert rel_l2(to_f64(o), to_f64(o2)) < 1e-3
    assert rel_l2(to_f64(S), to_f64(S2)) < 1e-3


@algo_param
def test_matches_fp32_path_closely(algo):
    """Tensor-core and fp32 CUDA-core paths on the same bf16 inputs."""
    shape = PrefillShape(B=1, T=1024, H=4, dk=128, dv=128, dtype=BF16)
    d, o, S = _run(shape, seed=21, algo=algo)
    o2, S2 = kda.chunk_forward_simt(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"])
    torch.cuda.synchronize()
    assert rel_l2(to_f64(o), to_f64(o2)) < 1e-2
    assert rel_l2(to_f64(S), to_f64(S2)) < 1e-2


@algo_param
def test_full_replacement_regime(algo):
    """beta = 1: the delta rule overwrites the value stored under each key; the
    chunked tensor-core form must still agree with the recurrence."""
    shape = PrefillShape(B=1, T=256, H=2, dk=128, dv=128, dtype=BF16)
    d = prefill_inputs(shape, 5, torch.device("cuda"))
    d["beta"].fill_(1.0)
    o, S = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"], algo=algo)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_prefill(d)
    assert_close(to_f64(o), o_ref, BF16, "o")
    assert_close(to_f64(S), S_ref, BF16, "final state")


@algo_param
def test_scalar_gate_gated_deltanet_regime(algo):
    """log_alpha equal across channels (the Gated DeltaNet special case)."""
    shape = PrefillShape(B=1, T=256, H=2, dk=128, dv=128, dtype=BF16)
    d = prefill_inputs(shape, 6, torch.device("cuda"))
    d["log_alpha"].copy_(d["log_alpha"][..., :1].expand_as(d["log_alpha"]))
    o, S = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"], algo=algo)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_prefill(d)
    assert_close(to_f64(o), o_ref, BF16, "o")
    assert_close(to_f64(S), S_ref, BF16, "final state")


@pytest.fixture
def small_auto_budget():
    """AUTO's workspace budget at 2 MiB: one sequence at H=4 runs the two-pass
    schedule in windows of 320 tokens (dk=dv=128) or 832 tokens (dk=dv=64)."""
    prev = kda.set_auto_workspace_limit(2 << 20)
    yield
    kda.set_auto_workspace_limit(prev)


@pytest.mark.parametrize("T,dk,dv", [(1000, 128, 128), (640, 128, 128), (1000, 64, 64), (2000, 64, 128)])
def test_auto_windows_match_oracle_and_one_launch_pair(T, dk, dv, small_auto_budget):
    """Windows of the two-pass schedule (ragged last window, exact multiple, two
    head sizes): the state handed on in fp32 between windows gives the oracle's
    result and the one-pair result."""
    H = 4
    assert kda.workspace_size(1, T, H, dk, dv, 1, algo="auto") < kda.workspace_size(1, T, H, dk, dv, 1,
                                                                                      algo="two_pass")
    shape = PrefillShape(B=1, T=T, H=H, dk=dk, dv=dv, dtype=BF16)
    d, o, S = _run(shape, seed=31 + T + dk, algo="auto")
    o_ref, S_ref = oracle_prefill(d)
    assert_close(to_f64(o), o_ref, BF16, "o")
    assert_close(to_f64(S), S_ref, BF16, "final state")
    o2, S2 = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"],
                               algo="two_pass")
    torch.cuda.synchronize()
    assert rel_l2(to_f64(o), to_f64(o2)) < 1e-3
    assert rel_l2(to_f64(S), to_f64(S2)) < 1e-3


def test_auto_windows_zero_start_no_final_state(small_auto_budget):
    shape = PrefillShape(B=1, T=777, H=4, dk=128, dv=128, dtype=BF16, init_state="none")
    d, o, S = _run(shape, seed=41, final_state=False)
    assert S is None
    o_ref, _ = oracle_prefill(d)
    assert_close(to_f64(o), o_ref, BF16, "o")


def test_auto_windows_scalar_gate(small_auto_budget):
    """kda_gdn_chunk_forward through the windows: the [T, H] gate is sliced per window."""
    shape = PrefillShape(B=1, T=900, H=4, dk=128, dv=128, dtype=BF16, gate="scalar")
    d = prefill_inputs(shape, 43, torch.device("cuda"))
    o, S = kda.gdn_chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"])
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    full = dict(d, log_alpha=d["log_alpha"].unsqueeze(-1).expand(*d["q"].shape).contiguous())
    o_ref, S_ref = oracle_prefill(full)
    assert_close(to_f64(o), o_ref, BF16, "o")
    assert_close(to_f64(S), S_ref, BF16, "final state")


def test_auto_windowed_plan_with_cu_seqlens_runs_fused(small_auto_budget):
    """A single packed sequence (cu_seqlens) cannot be sliced on the host: the
    windowed plan runs the fused schedule, with no workspace."""
    shape = PrefillShape(B=1, T=1000, H=4, dk=128, dv=128, dtype=BF16, cu_seqlens=(0, 1000))
    d = prefill_inputs(shape, 44, torch.device("cuda"))
    o, S = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["init_state"], d["cu_seqlens"])
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_prefill(d)
    assert_close(to_f64(o), o_ref, BF16, "o")
    assert_close(to_f64(S), S_ref, BF16, "final state")
