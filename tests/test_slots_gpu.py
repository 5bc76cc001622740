"""State-slot prefill and decode (kda_chunk_forward_slots, kda_recurrent_step_slots)
against the fp64 oracle: states live in a pool, each sequence names its slot
(-1: no state).  Covers the serving hand-offs the remio.ai page asks to test
(batched decode, prefix caching, state across chunk boundaries): resuming a
prefill from a cached prefix state, prefill into slots followed by decode from
them, padding rows, untouched slots, and out-of-range slot entries."""
import numpy as np
import pytest
import torch

import gated_delta_rule_85_b200 as kda
import oracle
from gated_delta_rule_85_b200.workloads import (DecodeShape, PrefillShape, decode_step_inputs, draw_state,
                                                prefill_inputs, to_f64)
from kda_testutil import assert_close

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16
DEV = torch.device("cuda")


def _pool(P, H, dk, dv, seed):
    return draw_state((P, H, dk, dv), DEV, seed, 9)


def _oracle_from_slots(d, pool0, slots):
    """Oracle prefill with init = pool0[slot] (zeros for -1); returns o, per-sequence final states."""
    init = np.stack([to_f64(pool0[s]) if s >= 0 else np.zeros(pool0.shape[1:]) for s in slots])
    cu = None if d.get("cu_seqlens") is None else d["cu_seqlens"].cpu().numpy()
    return oracle.forward(*(to_f64(d[x]) for x in ("q", "k", "v", "log_alpha", "beta")), init_state=init,
                          cu_seqlens=cu)


def _expected_pool(pool0, slots, finals):
    out = to_f64(pool0).copy()
    for n, s in enumerate(slots):
        if s >= 0:
            out[s] = finals[n]
    return out


@pytest.mark.parametrize("algo,simt", [("fused", False), ("two_pass", False), ("auto", True)])
@pytest.mark.parametrize("packed", [False, True])
def test_prefill_into_and_out_of_slots(algo, simt, packed):
    dtype = torch.float32 if simt else BF16
    H, dk, dv, P = 3, 128, 128, 8
    slots = [6, -1, 2] if not packed else [5, 0, -1, 7]
    if packed:
        lens = [70, 130, 1, 64]
        shape = PrefillShape(B=1, T=sum(lens), H=H, dk=dk, dv=dv, dtype=dtype,
                             cu_seqlens=tuple(np.cumsum([0] + lens).tolist()))
    else:
        shape = PrefillShape(B=3, T=150, H=H, dk=dk, dv=dv, dtype=dtype)
    d = prefill_inputs(shape, 11, DEV)
    pool = _pool(P, H, dk, dv, 12)
    pool0 = pool.clone()
    st = torch.tensor(slots, dtype=torch.int32, device=DEV)
    if simt:
        o = kda.chunk_forward_slots(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], pool, st, d["cu_seqlens"])
    else:
        o = kda.chunk_forward_slots(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], pool, st, d["cu_seqlens"],
                                    algo=algo)
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    o_ref, S_ref = _oracle_from_slots(d, pool0, slots)
    assert_close(to_f64(o), o_ref, dtype, "o")
    want = _expected_pool(pool0, slots, S_ref)
    touched = [s for s in slots if s >= 0]
    assert_close(to_f64(pool[touched]), want[touched], dtype, "slot states")
    untouched = [s for s in range(P) if s not in touched]
    assert torch.equal(pool[untouched], pool0[untouched])   # other slots are not written


@pytest.mark.parametrize("algo", ["fused", "two_pass"])
def test_prefix_cache_resume_equals_one_prefill(algo):
    """Prefill a prefix into slots, then prefill the continuation resuming from the
    cached slots: the result equals one recurrence over prefix + continuation."""
    H, dk, dv, P, T0, T1 = 2, 128, 128, 4, 192, 133      # prefix ends on a chunk boundary
    shape = PrefillShape(B=2, T=T0 + T1, H=H, dk=dk, dv=dv, dtype=BF16, init_state="none")
    d = prefill_inputs(shape, 21, DEV)
    pool = torch.zeros((P, H, dk, dv), dtype=torch.float32, device=DEV)
    st = torch.tensor([3, 1], dtype=torch.int32, device=DEV)
    part = lambda sl: [d[x][:, sl].contiguous() for x in ("q", "k", "v", "log_alpha", "beta")]
    o0 = kda.chunk_forward_slots(*part(slice(0, T0)), pool, st, algo=algo)
    o1 = kda.chunk_forward_slots(*part(slice(T0, None)), pool, st, algo=algo)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.forward(*(to_f64(d[x]) for x in ("q", "k", "v", "log_alpha", "beta")))
    assert_close(np.concatenate([to_f64(o0), to_f64(o1)], axis=1), o_ref, BF16, "o")
    assert_close(to_f64(pool[[3, 1]]), S_ref, BF16, "cached states")
    o_one, S_one = kda.chunk_forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, algo=algo)
    torch.cuda.synchronize()
    # a prefix ending on a chunk boundary resumes into exactly the same chunk sequence
    assert torch.equal(torch.cat([o0, o1], dim=1), o_one) and torch.equal(pool[[3, 1]], S_one)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128)])
def test_decode_on_state_pool(dk, dv):
    H, P, N, steps = 4, 10, 6, 5
    slots = [3, -1, 7, 0, 9, 5]
    pool = _pool(P, H, dk, dv, 31)
    pool0 = pool.clone()
    st = torch.tensor(slots, dtype=torch.int32, device=DEV)
    dshape = DecodeShape(N=N, H=H, dk=dk, dv=dv, steps=steps, dtype=BF16)
    live = [n for n, s in enumerate(slots) if s >= 0]
    S_ref = np.stack([to_f64(pool0[slots[n]]) for n in live])
    for t in range(steps):
        x = decode_step_inputs(dshape, t, 32, DEV)
        o = kda.recurrent_step_slots(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, st)
        torch.cuda.synchronize()
        sel = [to_f64(x[key][live]) for key in ("q", "k", "v", "log_alpha", "beta")]
        o_t, S_ref = oracle.step(*sel, S_ref)
        assert_close(to_f64(o[live]), o_t, BF16, f"o step {t}")
        assert torch.count_nonzero(o[1]) == 0          # padding row
    assert kda.device_status() == 0
    assert_close(to_f64(pool[[slots[n] for n in live]]), S_ref, BF16, "pool states")
    untouched = [s for s in range(P) if s not in slots]
    assert torch.equal(pool[untouched], pool0[untouched])


def test_prefill_into_slots_then_decode_matches_one_recurrence():
    H, dk, dv, P, T0, steps = 2, 128, 128, 5, 200, 16
    slots = [4, 2]
    shape = PrefillShape(B=2, T=T0, H=H, dk=dk, dv=dv, dtype=BF16, init_state="none")
    d = prefill_inputs(shape, 41, DEV)
    pool = torch.zeros((P, H, dk, dv), dtype=torch.float32, device=DEV)
    st = torch.tensor(slots, dtype=torch.int32, device=DEV)
    o = kda.chunk_forward_slots(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], pool, st)
    dshape = DecodeShape(N=2, H=H, dk=dk, dv=dv, steps=steps, dtype=BF16)
    dec = [decode_step_inputs(dshape, t, 42, DEV) for t in range(steps)]
    o_dec = [kda.recurrent_step_slots(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, st) for x in dec]
    torch.cuda.synchronize()
    cat = {key: np.concatenate([to_f64(d[key]), np.stack([to_f64(x[key]) for x in dec], axis=1)], axis=1)
           for key in ("q", "k", "v", "log_alpha", "beta")}
    o_ref, S_ref = oracle.forward(cat["q"], cat["k"], cat["v"], cat["log_alpha"], cat["beta"])
    assert_close(to_f64(o), o_ref[:, :T0], BF16, "prefill o")
    assert_close(np.stack([to_f64(x) for x in o_dec], axis=1), o_ref[:, T0:], BF16, "decode o")
    assert_close(to_f64(pool[slots]), S_ref, BF16, "final states")


def test_out_of_range_slot_is_flagged_and_skipped():
    H, dk, dv, P = 2, 128, 128, 4
    shape = PrefillShape(B=2, T=100, H=H, dk=dk, dv=dv, dtype=BF16)
    d = prefill_inputs(shape, 51, DEV)
    pool = _pool(P, H, dk, dv, 52)
    pool0 = pool.clone()
    st = torch.tensor([1, 99], dtype=torch.int32, device=DEV)
    kda.device_status(clear=True)
    o = kda.chunk_forward_slots(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], pool, st)
    torch.cuda.synchronize()
    assert kda.device_status(clear=True) & kda.DEV_BAD_SLOT
    o_ref, S_ref = _oracle_from_slots(d, pool0, [1, -1])   # the bad entry counts as "no state"
    assert_close(to_f64(o), o_ref, BF16, "o")
    assert_close(to_f64(pool[1]), S_ref[0], BF16, "slot 1")
    assert torch.equal(pool[[0, 2, 3]], pool0[[0, 2, 3]])
    x = decode_step_inputs(DecodeShape(N=2, H=H, dk=dk, dv=dv, steps=1, dtype=BF16), 0, 53, DEV)
    od = kda.recurrent_step_slots(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool,
                                  torch.tensor([-5, 0], dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert kda.device_status(clear=True) & kda.DEV_BAD_SLOT
    assert torch.count_nonzero(od[0]) == 0
