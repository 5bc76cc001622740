"""Pins for the fp64 oracle (CPU only).

The oracle is checked against things other than itself: special cases that
reduce to DeltaNet and Gated DeltaNet ("Kimi Delta Attention 徹底解説"
(tech-tide.dev), § "Kimi Delta Attention の仕組み"), the closed forms of a
full replacement (beta = 1) and of an orthonormal key memory, a scalar
(dk = dv = 1) recurrence, brute-force transition products on tiny inputs, the
chunked regrouping, and invariants (linearity, column independence, varlen
packing).  Each independent reference is written here from the page's
statement, not from the oracle's code.
"""
import json
import math
import os

import numpy as np
import pytest

import chunk_model
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(rng, B=1, T=7, H=2, dk=4, dv=3, unit_k=False, scalar_gate=False, s0=True):
    q = rng.normal(size=(B, T, H, dk))
    k = rng.normal(size=(B, T, H, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(B, T, H, dv))
    x = rng.normal(-2.0, 1.0, size=(B, T, H, 1 if scalar_gate else dk))
    g = -np.log1p(np.exp(x))
    if scalar_gate:
        g = np.repeat(g, dk, axis=-1)
    b = 1.0 / (1.0 + np.exp(-rng.normal(size=(B, T, H))))
    S0 = rng.normal(size=(B, H, dk, dv)) if s0 else None
    return q, k, v, g, b, S0


# ---------------------------------------------------------------- special cases

def test_identity_gate_zero_beta_keeps_state():
    """alpha = 1, beta = 0: nothing is forgotten or written; o_t = S0^T q_t."""
    rng = np.random.default_rng(1)
    q, k, v, g, b, S0 = _rand_case(rng, T=9, dk=5, dv=4)
    g[:] = 0.0
    b[:] = 0.0
    o, S = oracle.forward(q, k, v, g, b, S0)
    assert np.array_equal(S, S0)
    want = np.einsum("bhcj,bthc->bthj", S0, q)
    np.testing.assert_allclose(o, want, rtol=0, atol=1e-13)


def test_full_replacement_beta_one():
    """beta = 1 and |k_t| = 1 replace the value stored under k_t: S_t^T k_t = v_t,
    whatever the gate and the prior state (the page: beta = 1 is a full replacement)."""
    rng = np.random.default_rng(2)
    q, k, v, g, b, S0 = _rand_case(rng, B=2, T=12, H=3, dk=6, dv=5, unit_k=True)
    b[:] = 1.0
    o, _ = oracle.forward(k, k, v, g, b, S0)  # query with the key just written
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)


def test_orthonormal_keys_store_and_recall():
    """alpha = 1, S0 = 0, beta = 1, orthonormal keys: after writing (k_i, v_i) for
    i = 1..m, a read with k_i (tokens with beta = 0 do not write) returns v_i."""
    rng = np.random.default_rng(3)
    dk, dv, m = 8, 5, 8
    Qm, _ = np.linalg.qr(rng.normal(size=(dk, dk)))
    keys = Qm.T[:m]                       # orthonormal rows
    vals = rng.normal(size=(m, dv))
    T = 2 * m
    k = np.zeros((1, T, 1, dk))
    q = np.zeros((1, T, 1, dk))
    v = np.zeros((1, T, 1, dv))
    b = np.zeros((1, T, 1))
    k[0, :m, 0] = keys
    v[0, :m, 0] = vals
    b[0, :m, 0] = 1.0
    q[0, m:, 0] = keys                    # read phase: beta = 0, k = 0
    g = np.zeros((1, T, 1, dk))
    o, S = oracle.forward(q, k, v, g, b, None)
    np.testing.assert_allclose(o[0, m:, 0], vals, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], keys.T @ vals, rtol=0, atol=1e-12)


def _gdn_reference(q, k, v, a_scalar, b, S0):
    """Gated DeltaNet in transition form: S_t = a_t (I - b_t k_t k_t^T) S_{t-1} + b_t k_t v_t^T."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    S_out = np.zeros((B, H, dk, dv))
    for bb in range(B):
        for h in range(H):
            S = S0[bb, h].copy()
            for t in range(T):
                kt = k[bb, t, h]
                P = np.eye(dk) - b[bb, t, h] * np.outer(kt, kt)
                S = a_scalar[bb, t, h] * (P @ S) + b[bb, t, h] * np.outer(kt, v[bb, t, h])
                o[bb, t, h] = S.T @ q[bb, t, h]
            S_out[bb, h] = S
    return o, S_out


def test_scalar_gate_is_gated_deltanet():
    """log_alpha broadcast over dk reduces KDA to Gated DeltaNet."""
    rng = np.random.default_rng(4)
    q, k, v, g, b, S0 = _rand_case(rng, B=2, T=20, H=2, dk=6, dv=4, scalar_gate=True)
    o, S = oracle.forward(q, k, v, g, b, S0)
    o_ref, S_ref = _gdn_reference(q, k, v, np.exp(g[..., 0]), b, S0)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=0, atol=1e-12)


def test_unit_gate_is_deltanet():
    """alpha = 1 reduces KDA to DeltaNet: S_t = S_{t-1} + b k (v - S_{t-1}^T k)^T."""
    rng = np.random.default_rng(5)
    q, k, v, g, b, S0 = _rand_case(rng, B=1, T=25, H=3, dk=5, dv=6, unit_k=True)
    g[:] = 0.0
    o, S = oracle.forward(q, k, v, g, b, S0)
    B, T, H, dk = q.shape
    for h in range(H):
        St = S0[0, h].copy()
        for t in range(T):
            kt = k[0, t, h]
            err = v[0, t, h] - St.T @ kt
            St = St + b[0, t, h] * np.outer(kt, err)
            np.testing.assert_allclose(o[0, t, h], St.T @ q[0, t, h], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(S[0, h], St, rtol=1e-12, atol=1e-12)


def test_scalar_recurrence_dk_dv_one():
    """dk = dv = 1: s_t = alpha s (1 - beta k^2) + beta k v, o_t = q s_t."""
    rng = np.random.default_rng(6)
    T = 30
    q, k, v = (rng.normal(size=(1, T, 1, 1)) for _ in range(3))
    g = -np.abs(rng.normal(size=(1, T, 1, 1)))
    b = rng.uniform(size=(1, T, 1))
    s0 = np.array([[[[0.7]]]])
    o, S = oracle.forward(q, k, v, g, b, s0)
    s = 0.7
    for t in range(T):
        a = math.exp(g[0, t, 0, 0])
        kk, bb = k[0, t, 0, 0], b[0, t, 0]
        s = a * s * (1.0 - bb * kk * kk) + bb * kk * v[0, t, 0, 0]
        assert abs(o[0, t, 0, 0] - q[0, t, 0, 0] * s) <= 1e-13 * max(1.0, abs(s))
    assert abs(S[0, 0, 0, 0] - s) <= 1e-13


def test_gate_acts_on_key_axis():
    """Diag(alpha) scales rows (key channels) of the dk x dv state: with beta = 0,
    a channel whose alpha is ~0 is erased and the others are kept."""
    dk, dv = 3, 4
    S0 = np.arange(1, dk * dv + 1, dtype=np.float64).reshape(1, 1, dk, dv)
    q = np.zeros((1, 1, 1, dk))
    k = np.zeros((1, 1, 1, dk))
    v = np.zeros((1, 1, 1, dv))
    b = np.zeros((1, 1, 1))
    g = np.array([0.0, -800.0, math.log(0.5)]).reshape(1, 1, 1, dk)
    _, S = oracle.forward(q, k, v, g, b, S0)
    np.testing.assert_array_equal(S[0, 0, 0], S0[0, 0, 0])
    np.testing.assert_array_equal(S[0, 0, 1], np.zeros(dv))
    np.testing.assert_allclose(S[0, 0, 2], 0.5 * S0[0, 0, 2], rtol=1e-15)


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("seed", range(6))
def test_unrolled_product_matches_recurrence(seed):
    rng = np.random.default_rng(100 + seed)
    dk = int(rng.integers(1, 5))
    dv = int(rng.integers(1, 4))
    T = int(rng.integers(1, 9))
    q, k, v, g, b, S0 = _rand_case(rng, B=2, T=T, H=2, dk=dk, dv=dv, s0=bool(seed % 2))
    o1, S1 = oracle.forward(q, k, v, g, b, S0)
    o2, S2 = oracle.unrolled(q, k, v, g, b, S0)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S1, S2, rtol=0, atol=1e-12)


@pytest.mark.parametrize("pairwise", [False, True])
def test_chunked_regrouping_matches(pairwise):
    """The chunked regrouping (exact in real arithmetic) agrees to rounding."""
    rng = np.random.default_rng(7)
    q, k, v, g, b, S0 = _rand_case(rng, B=2, T=150, H=2, dk=16, dv=8, unit_k=True)
    o1, S1 = oracle.forward(q, k, v, g, b, S0)
    o2, S2 = chunk_model.chunked_forward(q, k, v, g, b, S0, pairwise=pairwise)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-11 * np.abs(o1).max())
    np.testing.assert_allclose(S1, S2, rtol=0, atol=1e-11 * np.abs(S1).max())


# ---------------------------------------------------------------- invariants

def test_linear_in_values_and_state():
    rng = np.random.default_rng(8)
    q, k, v, g, b, S0 = _rand_case(rng, T=10, dk=4, dv=3)
    _, _, v2, _, _, S02 = _rand_case(rng, T=10, dk=4, dv=3)
    oa, Sa = oracle.forward(q, k, v, g, b, S0)
    ob, Sb = oracle.forward(q, k, v2, g, b, S02)
    oc, Sc = oracle.forward(q, k, 2.0 * v - 3.0 * v2, g, b, 2.0 * S0 - 3.0 * S02)
    np.testing.assert_allclose(oc, 2.0 * oa - 3.0 * ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Sc, 2.0 * Sa - 3.0 * Sb, rtol=0, atol=1e-12)


def test_value_columns_are_independent():
    """Permuting dv columns of v and S0 permutes o and S the same way."""
    rng = np.random.default_rng(9)
    q, k, v, g, b, S0 = _rand_case(rng, T=11, dk=4, dv=6)
    perm = rng.permutation(6)
    o, S = oracle.forward(q, k, v, g, b, S0)
    op, Sp = oracle.forward(q, k, v[..., perm], g, b, S0[..., perm])
    np.testing.assert_allclose(op, o[..., perm], rtol=0, atol=1e-13)
    np.testing.assert_allclose(Sp, S[..., perm], rtol=0, atol=1e-13)


def test_varlen_equals_separate_runs():
    rng = np.random.default_rng(10)
    lens = [5, 0, 17, 1, 9]
    cu = np.cumsum([0] + lens)
    Tt = int(cu[-1])
    q, k, v, g, b, _ = _rand_case(rng, B=1, T=Tt, H=2, dk=4, dv=3)
    S0 = rng.normal(size=(len(lens), 2, 4, 3))
    o, S = oracle.forward(q, k, v, g, b, S0, cu_seqlens=cu)
    for n, L in enumerate(lens):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        on, Sn = oracle.forward(q[:, t0:t1], k[:, t0:t1], v[:, t0:t1], g[:, t0:t1], b[:, t0:t1], S0[n:n + 1])
        np.testing.assert_array_equal(o[:, t0:t1], on)
        np.testing.assert_array_equal(S[n], Sn[0])
    np.testing.assert_array_equal(S[1], S0[1])        # empty sequence keeps its state


def test_split_and_resume():
    rng = np.random.default_rng(11)
    q, k, v, g, b, S0 = _rand_case(rng, T=40, dk=4, dv=3)
    o, S = oracle.forward(q, k, v, g, b, S0)
    o1, S1 = oracle.forward(q[:, :13], k[:, :13], v[:, :13], g[:, :13], b[:, :13], S0)
    o2, S2 = oracle.forward(q[:, 13:], k[:, 13:], v[:, 13:], g[:, 13:], b[:, 13:], S1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, rtol=0, atol=1e-14)
    np.testing.assert_allclose(S2, S, rtol=0, atol=1e-14)


def test_step_equals_forward():
    rng = np.random.default_rng(12)
    N, H, dk, dv, steps = 3, 2, 4, 5, 6
    state = rng.normal(size=(N, H, dk, dv))
    q, k, v, g, b, _ = _rand_case(rng, B=N, T=steps, H=H, dk=dk, dv=dv)
    o_ref, S_ref = oracle.forward(q, k, v, g, b, state)
    s = state.copy()
    for t in range(steps):
        o_t, s = oracle.step(q[:, t], k[:, t], v[:, t], g[:, t], b[:, t], s)
        np.testing.assert_allclose(o_t, o_ref[:, t], rtol=0, atol=1e-14)
    np.testing.assert_allclose(s, S_ref, rtol=0, atol=1e-14)


def test_golden_regression():
    """Stored oracle output (written by tests/golden/make_golden.py, which calls only
    oracle/) guards the oracle's arithmetic against silent change."""
    with open(os.path.join(GOLDEN, "oracle_small.json")) as f:
        gold = json.load(f)
    inp = {k: np.array(v, dtype=np.float64) for k, v in gold["inputs"].items()}
    o, S = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["init_state"])
    np.testing.assert_allclose(o, np.array(gold["o"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(S, np.array(gold["final_state"]), rtol=0, atol=1e-13)


def test_rejects_bad_arguments():
    rng = np.random.default_rng(13)
    q, k, v, g, b, S0 = _rand_case(rng, T=4)
    with pytest.raises(ValueError):
        oracle.forward(q, k[:, :3], v, g, b, S0)
    with pytest.raises(ValueError):
        oracle.forward(q, k, v, g, b, None, cu_seqlens=[0, 2, 1, 4])
