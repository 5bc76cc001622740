"""Backward of the chunked prefill (kda_chunk_backward) against the fp64 oracle's
reverse-mode gradients of the token recurrence, on the same inputs.

The loss is L = sum <d_o, o> + <dfinal_state, final_state> with seeded
cotangents; every gradient (dq, dk, dv, dlog_alpha, dbeta, dinit_state) is
compared element by element.  The backward accumulates in fp32 with the
forward's operand precision (split tf32 for fp32 inputs, bf16/tf32 operands for
bf16 inputs), so the operator's bounds apply: rel-L2 <= 1e-4 for fp32 inputs;
for bf16 inputs rel-L2 <= 1e-2 and max-abs <= 5e-2 relative to the largest
reference magnitude (gradients are not O(1) quantities like o and S).
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_85_b200 as kda
import oracle
from gated_delta_rule_85_b200.workloads import (PrefillShape, STRONG_KINDS, backward_cotangents, prefill_inputs,
                                                strong_decay, to_f64)
from kda_testutil import max_abs, rel_l2

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
BF16 = torch.bfloat16
GRADS = ["dq", "dk", "dv", "dlog_alpha", "dbeta", "dinit_state"]


def _pick(x, heads, axis):
    if x is None:
        return None
    if heads is not None:
        x = x.index_select(axis, torch.as_tensor(heads, device=x.device))
    return to_f64(x)


def oracle_grads(d, c, heads=None):
    cu = None if d.get("cu_seqlens") is None else d["cu_seqlens"].cpu().numpy()
    return oracle.backward(*(_pick(d[n], heads, 2) for n in ("q", "k", "v", "log_alpha", "beta")),
                           _pick(c["d_o"], heads, 2), init_state=_pick(d.get("init_state"), heads, 1),
                           dfinal=_pick(c.get("dfinal_state"), heads, 1), cu_seqlens=cu)


def check(got, want, dtype, heads=None, what=""):
    for name in GRADS:
        if got.get(name) is None:
            continue
        axis = 1 if name == "dinit_state" else 2
        g = _pick(got[name], heads, axis)
        w = want[name]
        assert np.all(np.isfinite(g)), f"{what} {name}: non-finite"
        r = rel_l2(g, w)
        if dtype == torch.float32:
            assert r <= 1e-4, f"{what} {name}: rel-L2 {r:.2e}"
        else:
            assert r <= 1e-2, f"{what} {name}: rel-L2 {r:.2e}"
            scale = max(1.0, float(np.max(np.abs(w)))) if w.size else 1.0
            m = max_abs(g, w)
            # the unscaled max-abs is reported beside the scaled bound (pytest -rA shows it)
            print(f"{what} {name}: rel-L2 {r:.2e}, max-abs {m:.2e} unscaled, largest |ref| {scale:.2e}, "
                  f"bound {5e-2 * scale:.2e}")
            assert m <= 5e-2 * scale, f"{what} {name}: max-abs {m:.2e} unscaled (bound 5e-2 x scale {scale:.2e})"


def run(d, c, **kw):
    return kda.chunk_backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], c["d_o"], d.get("init_state"),
                              c.get("dfinal_state"), d.get("cu_seqlens"), **kw)


# (dtype, schedule): the tensor-core schedule covers bf16 with dk = dv = 128;
# the SIMT schedule takes everything (AUTO picks it for the other sizes).
SCHEDULES = [(torch.float32, "auto"), (BF16, "simt"), (BF16, "auto")]


@pytest.mark.parametrize("dtype,algo", SCHEDULES)
@pytest.mark.parametrize("B,T,H,dk,dv", [(2, 200, 2, 128, 128), (2, 130, 3, 64, 64), (1, 64, 2, 128, 64),
                                         (3, 1, 2, 64, 128), (1, 333, 1, 128, 128), (2, 64, 2, 128, 128),
                                         (1, 129, 2, 128, 128)])
def test_backward_matches_oracle(dtype, algo, B, T, H, dk, dv):
    shape = PrefillShape(B=B, T=T, H=H, dk=dk, dv=dv, dtype=dtype)
    d = prefill_inputs(shape, 100 + T + dk, DEV)
    c = backward_cotangents(shape, 200 + T, DEV)
    got = run(d, c, algo=algo)
    torch.cuda.synchronize()
    check(got, oracle_grads(d, c), dtype, what=f"{algo} B{B} T{T} dk{dk} dv{dv}")
    assert kda.device_status() == 0


def test_backward_tensor_schedule_refuses_other_sizes():
    shape = PrefillShape(B=1, T=64, H=1, dk=64, dv=64, dtype=BF16)
    d = prefill_inputs(shape, 3, DEV)
    c = backward_cotangents(shape, 4, DEV)
    with pytest.raises(kda.KDAError):
        run(d, c, algo="tensor")


@pytest.mark.parametrize("dtype,algo", SCHEDULES)
def test_backward_packed_sequences(dtype, algo):
    """Packed input with empty, single-token, exact-chunk and ragged sequences;
    equal bit for bit to running each sequence alone."""
    lens = [0, 1, 63, 64, 65, 130, 7, 0]
    cu = tuple(np.cumsum([0] + lens).tolist())
    shape = PrefillShape(B=1, T=sum(lens), H=3, dk=128, dv=128, dtype=dtype, cu_seqlens=cu)
    d = prefill_inputs(shape, 7, DEV)
    c = backward_cotangents(shape, 8, DEV)
    got = run(d, c, algo=algo)
    torch.cuda.synchronize()
    check(got, oracle_grads(d, c), dtype, what=f"packed {algo}")
    for n, L in enumerate(lens):
        a = cu[n]
        one = {x: d[x][:, a:a + L] for x in ("q", "k", "v", "log_alpha", "beta")}
        one["init_state"] = d["init_state"][n:n + 1]
        co = {"d_o": c["d_o"][:, a:a + L], "dfinal_state": c["dfinal_state"][n:n + 1]}
        g1 = run(one, co, algo=algo)
        for name in GRADS:
            whole = got[name][n:n + 1] if name == "dinit_state" else got[name][:, a:a + L]
            assert torch.equal(whole, g1[name]), (n, name)


@pytest.mark.parametrize("dtype,algo", SCHEDULES)
def test_backward_strong_decay_blocks(dtype, algo):
    """Sequence 0 decays by ~3.5 per token (more than the in-block range the
    diagonal blocks may take through a block boundary, and far past the chunk
    range of the tensor-core chain rule), sequence 1 as usual: both the exact
    path and the tensor-core one run, and both match."""
    shape = PrefillShape(B=2, T=160, H=2, dk=128, dv=128, dtype=dtype)
    d = prefill_inputs(shape, 77, DEV)
    gen = torch.Generator(device=DEV).manual_seed(79)
    d["log_alpha"][0] = -3.5 + 0.2 * torch.rand(d["log_alpha"][0].shape, generator=gen, device=DEV)
    c = backward_cotangents(shape, 78, DEV)
    got = run(d, c, algo=algo)
    torch.cuda.synchronize()
    check(got, oracle_grads(d, c), dtype, what=f"strong decay {algo}")


@pytest.mark.parametrize("dtype,dk,algo", [(torch.float32, 64, "auto"), (BF16, 128, "tensor")])
def test_backward_without_states(dtype, dk, algo):
    """init_state NULL (zeros) and dfinal_state NULL (zero cotangent): dinit_state is
    the gradient at the zero state."""
    shape = PrefillShape(B=2, T=150, H=2, dk=dk, dv=128, dtype=dtype, init_state="none")
    d = prefill_inputs(shape, 31, DEV)
    assert d["init_state"] is None
    c = backward_cotangents(shape, 32, DEV, dfinal=False)
    got = run(d, c, algo=algo)
    torch.cuda.synchronize()
    check(got, oracle_grads(d, c), dtype, what=f"no states {algo}")
    assert got["dinit_state"].abs().max().item() > 0


@pytest.mark.parametrize("kind", STRONG_KINDS)
@pytest.mark.parametrize("algo", ["simt", "tensor"])
@pytest.mark.parametrize("packed", [False, True])
def test_backward_strong_decay_kinds(kind, algo, packed):
    """The forward's strong-decay patterns -- single-token hard resets (-100), whole
    chunks at -2, strong and weak channels mixed in one head -- through both bf16
    schedules; the tensor-core one takes its exact tier for these chunks, dense and
    packed (empty and one-token sequences included)."""
    if packed:
        lens = [70, 0, 129, 1, 256]
        cu = tuple(np.cumsum([0] + lens).tolist())
        shape = PrefillShape(B=1, T=cu[-1], H=2, dk=128, dv=128, dtype=BF16, cu_seqlens=cu)
    else:
        shape = PrefillShape(B=2, T=300, H=2, dk=128, dv=128, dtype=BF16)
    d = prefill_inputs(shape, 600 + len(kind), DEV)
    strong_decay(d["log_alpha"], kind, 21)
    c = backward_cotangents(shape, 601, DEV)
    kda.device_status(clear=True)
    got = run(d, c, algo=algo)
    torch.cuda.synchronize()
    assert kda.device_status(clear=True) == 0
    check(got, oracle_grads(d, c), BF16, what=f"{kind} {algo}")


@pytest.mark.parametrize("dv", [64, 128])
def test_backward_no_tokens(dv):
    """T = 0: nothing to differentiate through; dinit_state = dfinal_state exactly."""
    shape = PrefillShape(B=3, T=0, H=2, dk=128, dv=dv, dtype=BF16)
    d = prefill_inputs(shape, 5, DEV)
    c = backward_cotangents(shape, 6, DEV)
    got = run(d, c)
    torch.cuda.synchronize()
    assert torch.equal(got["dinit_state"], c["dfinal_state"])
    c["dfinal_state"] = None
    got = run(d, c)
    torch.cuda.synchronize()
    assert torch.count_nonzero(got["dinit_state"]).item() == 0


@pytest.mark.parametrize("algo", ["simt", "tensor"])
def test_backward_is_deterministic(algo):
    shape = PrefillShape(B=1, T=300, H=4, dk=128, dv=128, dtype=BF16)
    d = prefill_inputs(shape, 9, DEV)
    c = backward_cotangents(shape, 10, DEV)
    a = run(d, c, algo=algo)
    b = run(d, c, algo=algo)
    for name in GRADS:
        assert torch.equal(a[name], b[name]), name


@pytest.mark.parametrize("dk,dv,algo", [(64, 64, "auto"), (128, 128, "tensor")])
def test_backward_skips_dinit_state(dk, dv, algo):
    shape = PrefillShape(B=1, T=100, H=2, dk=dk, dv=dv, dtype=BF16)
    d = prefill_inputs(shape, 11, DEV)
    c = backward_cotangents(shape, 12, DEV)
    full = run(d, c, algo=algo)
    part = run(d, c, dinit_state=False, algo=algo)
    assert part["dinit_state"] is None
    for name in GRADS[:-1]:
        assert torch.equal(full[name], part[name]), name


@pytest.mark.slow
@pytest.mark.parametrize("algo", ["simt", "tensor"])
def test_backward_prefill_8k_sampled_heads(algo):
    """Full-size prefill_8k (B=1, T=8192, H=32, d=128, bf16) in one call; the oracle
    runs on three of the 32 heads (heads are independent)."""
    shape = PrefillShape(B=1, T=8192, H=32, dk=128, dv=128, dtype=BF16)
    d = prefill_inputs(shape, 0, DEV)
    c = backward_cotangents(shape, 0, DEV)
    got = run(d, c, algo=algo)
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    heads = [0, 17, 31]
    check(got, oracle_grads(d, c, heads), BF16, heads=heads, what="prefill_8k")


@pytest.mark.parametrize("dtype,algo", SCHEDULES)
@pytest.mark.parametrize("packed", [False, True])
@pytest.mark.parametrize("d128", [False, True])
def test_gdn_backward_matches_oracle(dtype, algo, packed, d128):
    """Gated DeltaNet (one decay rate per token-head): the oracle's gradients with
    the rate broadcast over the key channels, dlog_alpha summed over them (the
    gradient of a broadcast value).  d128: dk = dv = 128, which the tensor-core
    schedule takes."""
    if packed:
        lens = [70, 0, 129, 1]
        shape = PrefillShape(B=1, T=sum(lens), H=2, dk=128, dv=128 if d128 else 64, dtype=dtype, gate="scalar",
                             cu_seqlens=tuple(np.cumsum([0] + lens).tolist()))
    else:
        shape = PrefillShape(B=2, T=150, H=2, dk=128 if d128 else 64, dv=128, dtype=dtype, gate="scalar")
    d = prefill_inputs(shape, 91, DEV)
    assert d["log_alpha"].shape == d["beta"].shape
    c = backward_cotangents(shape, 92, DEV)
    got = kda.gdn_chunk_backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], c["d_o"], d["init_state"],
                                 c["dfinal_state"], d["cu_seqlens"], algo=algo)
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    dk = shape.dk
    d_b = dict(d, log_alpha=d["log_alpha"][..., None].expand(*d["log_alpha"].shape, dk).contiguous())
    want = oracle_grads(d_b, c)
    want["dlog_alpha"] = want["dlog_alpha"].sum(axis=-1)
    check(got, want, dtype, what=f"gdn {algo}")
    # the same schedule with the rate broadcast and the channel gradients summed
    full = run(d_b, c, algo=algo)
    torch.testing.assert_close(got["dlog_alpha"], full["dlog_alpha"].sum(-1), rtol=1e-4, atol=1e-4)
    for name in ("dq", "dk", "dv", "dbeta", "dinit_state"):
        assert torch.equal(got[name], full[name]), name


@pytest.mark.parametrize("split", [128, 100])
def test_backward_split_resume_chain_rule(split):
    """Split a sequence at token `split`: the second part starts from the state the
    forward reaches there, and its dL/dinit_state is the first part's dfinal.  The
    gradients of the two parts together equal one call (the state hand-off of the
    chain rule), fp32."""
    shape = PrefillShape(B=1, T=300, H=2, dk=64, dv=64, dtype=torch.float32)
    d = prefill_inputs(shape, 55, DEV)
    c = backward_cotangents(shape, 56, DEV)
    whole = run(d, c)
    cut = lambda x, a, b: x[:, a:b].contiguous()
    first = {x: cut(d[x], 0, split) for x in ("q", "k", "v", "log_alpha", "beta")}
    first["init_state"] = d["init_state"]
    second = {x: cut(d[x], split, 300) for x in ("q", "k", "v", "log_alpha", "beta")}
    _, S_mid = kda.chunk_forward(*(first[x] for x in ("q", "k", "v", "log_alpha", "beta")), first["init_state"],
                                 simt=True)
    second["init_state"] = S_mid
    g2 = run(second, {"d_o": cut(c["d_o"], split, 300), "dfinal_state": c["dfinal_state"]})
    g1 = run(first, {"d_o": cut(c["d_o"], 0, split), "dfinal_state": g2["dinit_state"]})
    torch.cuda.synchronize()
    for name in ("dq", "dk", "dv", "dlog_alpha", "dbeta"):
        both = torch.cat([g1[name], g2[name]], dim=1)
        torch.testing.assert_close(both, whole[name], rtol=1e-4, atol=1e-5, msg=name)
    torch.testing.assert_close(g1["dinit_state"], whole["dinit_state"], rtol=1e-4, atol=1e-5)


def test_backward_split_resume_tensor_schedule():
    """The split/resume chain rule on the tensor-core schedule (bf16, dk = dv = 128),
    split at a chunk boundary: the two parts joined by the state and its adjoint
    match one call to bf16 accuracy, and each part matches the oracle."""
    shape = PrefillShape(B=1, T=300, H=2, dk=128, dv=128, dtype=BF16)
    d = prefill_inputs(shape, 57, DEV)
    c = backward_cotangents(shape, 58, DEV)
    whole = run(d, c, algo="tensor")
    split = 128
    cut = lambda x, a, b: x[:, a:b].contiguous()
    first = {x: cut(d[x], 0, split) for x in ("q", "k", "v", "log_alpha", "beta")}
    first["init_state"] = d["init_state"]
    second = {x: cut(d[x], split, 300) for x in ("q", "k", "v", "log_alpha", "beta")}
    _, S_mid = kda.chunk_forward(*(first[x] for x in ("q", "k", "v", "log_alpha", "beta")), first["init_state"],
                                 simt=True)
    second["init_state"] = S_mid
    c2 = {"d_o": cut(c["d_o"], split, 300), "dfinal_state": c["dfinal_state"]}
    g2 = run(second, c2, algo="tensor")
    c1 = {"d_o": cut(c["d_o"], 0, split), "dfinal_state": g2["dinit_state"]}
    g1 = run(first, c1, algo="tensor")
    torch.cuda.synchronize()
    check(g2, oracle_grads(second, c2), BF16, what="second part")
    check(g1, oracle_grads(first, c1), BF16, what="first part")
    for name in ("dq", "dk", "dv", "dlog_alpha", "dbeta"):
        both = to_f64(torch.cat([g1[name], g2[name]], dim=1))
        assert rel_l2(both, to_f64(whole[name])) <= 1e-2, name
    assert rel_l2(to_f64(g1["dinit_state"]), to_f64(whole["dinit_state"])) <= 1e-2

