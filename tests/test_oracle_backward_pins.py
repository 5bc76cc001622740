"""Pins for the oracle's gradients (CPU only).

``oracle.backward`` is reverse-mode differentiation of the token recurrence
("Kimi Delta Attention 徹底解説" (tech-tide.dev), § "Kimi Delta Attention の仕組み";
the gradients are what the chunkwise training algorithm of "Kimi Linear、独自の
土俵でFull Attentionを上回る" (remio.ai), § "Kimi Linearがより賢いRecurrent
Memoryを使う方法" computes).  It is checked against things other than itself:
central finite differences of the loss through the forward recurrence and
through the independent transition-product form, a scalar (dk = dv = 1)
derivative worked by hand, the closed form with alpha = 1 and beta = 0, and
invariants (varlen packing, linearity in the cotangents).
"""
import numpy as np
import pytest

import oracle

FIELDS = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("log_alpha", "dlog_alpha"),
          ("beta", "dbeta"), ("init_state", "dinit_state")]


def _case(rng, B=2, T=7, H=2, dk=4, dv=3, kscale=0.6):
    q = rng.normal(size=(B, T, H, dk))
    k = rng.normal(size=(B, T, H, dk)) * kscale
    v = rng.normal(size=(B, T, H, dv))
    g = -np.log1p(np.exp(rng.normal(-2.0, 1.0, size=(B, T, H, dk))))
    b = 1.0 / (1.0 + np.exp(-rng.normal(size=(B, T, H))))
    S0 = rng.normal(size=(B, H, dk, dv))
    do = rng.normal(size=(B, T, H, dv))
    dF = rng.normal(size=(B, H, dk, dv))
    return dict(q=q, k=k, v=v, log_alpha=g, beta=b, init_state=S0), do, dF


def _loss(fwd, x, do, dF, cu=None):
    if cu is None:
        o, S = fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["init_state"])
    else:
        o, S = fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["init_state"], cu_seqlens=cu)
    return float((o * do).sum() + (S * dF).sum())


def _fd(fwd, x, do, dF, name, idx, eps=1e-6, cu=None):
    """Central difference of the loss in one input entry."""
    xp = dict(x)
    xm = dict(x)
    xp[name] = x[name].copy()
    xm[name] = x[name].copy()
    xp[name][idx] += eps
    xm[name][idx] -= eps
    return (_loss(fwd, xp, do, dF, cu) - _loss(fwd, xm, do, dF, cu)) / (2 * eps)


def _check_fd(fwd, x, do, dF, grads, samples=None, rng=None, cu=None, tol=1e-7):
    for name, gname in FIELDS:
        arr = x[name]
        if samples is None:
            idxs = list(np.ndindex(arr.shape))
        else:
            idxs = [tuple(int(rng.integers(0, s)) for s in arr.shape) for _ in range(samples)]
        for idx in idxs:
            want = _fd(fwd, x, do, dF, name, idx, cu=cu)
            got = grads[gname][idx]
            assert abs(got - want) <= tol * (1.0 + abs(want)), (name, idx, got, want)


def test_gradients_match_central_differences():
    """Every entry of every gradient, against the forward recurrence."""
    rng = np.random.default_rng(11)
    x, do, dF = _case(rng)
    gr = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], do,
                         init_state=x["init_state"], dfinal=dF)
    _check_fd(oracle.forward, x, do, dF, gr)


def test_gradients_match_differences_of_transition_products():
    """The same check through the brute-force transition-product form, which
    shares no loop with either the recurrence or its reverse sweep."""
    rng = np.random.default_rng(12)
    x, do, dF = _case(rng, B=1, T=5, H=1, dk=3, dv=2)
    gr = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], do,
                         init_state=x["init_state"], dfinal=dF)
    _check_fd(oracle.unrolled, x, do, dF, gr)


def test_gradients_across_checkpoint_segments():
    """T = 150 spans three recomputation segments of the reverse sweep."""
    rng = np.random.default_rng(13)
    x, do, dF = _case(rng, B=1, T=150, H=1, dk=4, dv=3, kscale=0.4)
    gr = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], do,
                         init_state=x["init_state"], dfinal=dF)
    _check_fd(oracle.forward, x, do, dF, gr, samples=40, rng=rng, tol=1e-6)


def test_varlen_gradients():
    """Packed sequences: equal to the per-sequence gradients, and to differences."""
    rng = np.random.default_rng(14)
    lens = [5, 0, 9, 1, 70]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    N, T, H, dk, dv = len(lens), int(cu[-1]), 2, 4, 3
    x, do, _ = _case(rng, B=1, T=T, H=H, dk=dk, dv=dv, kscale=0.5)
    x["init_state"] = rng.normal(size=(N, H, dk, dv))
    dF = rng.normal(size=(N, H, dk, dv))
    gr = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], do,
                         init_state=x["init_state"], dfinal=dF, cu_seqlens=cu)
    for n in range(N):
        a, b = int(cu[n]), int(cu[n + 1])
        sl = lambda t: t[:, a:b]
        one = oracle.backward(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["log_alpha"]), sl(x["beta"]),
                              sl(do), init_state=x["init_state"][n:n + 1], dfinal=dF[n:n + 1])
        for _, gname in FIELDS:
            got = gr[gname][n:n + 1] if gname == "dinit_state" else sl(gr[gname])
            assert np.array_equal(got, one[gname]), (n, gname)
    _check_fd(oracle.forward, x, do, dF, gr, samples=15, rng=rng, cu=cu, tol=1e-6)


def test_scalar_recurrence_derivative_by_hand():
    """dk = dv = 1: s_t = a_t s_{t-1} (1 - b_t k_t^2) + b_t k_t v_t, o_t = q_t s_t.
    Differentiating by hand, with w_t = dL/ds_t (the total derivative through
    every later token): w_T = do_T q_T + dF, w_{t-1} = do_{t-1} q_{t-1}
    + w_t a_t (1 - b_t k_t^2), and
      dq_t = do_t s_t
      dv_t = w_t b_t k_t
      db_t = w_t (k_t v_t - a_t s_{t-1} k_t^2)
      dk_t = w_t (b_t v_t - 2 a_t s_{t-1} b_t k_t)
      dg_t = w_t a_t s_{t-1} (1 - b_t k_t^2)      (a_t = exp(g_t))
      ds_0 = w_1 a_1 (1 - b_1 k_1^2)."""
    q = np.array([0.7, -1.3, 0.4])
    k = np.array([0.9, 0.5, -1.1])
    v = np.array([1.5, -0.2, 0.8])
    g = np.array([-0.1, -0.7, -0.3])
    b = np.array([0.6, 0.3, 0.9])
    s0, dF = 0.25, -0.6
    do = np.array([0.3, 1.1, -0.5])
    T = 3
    a = np.exp(g)
    s = [s0]
    for t in range(T):
        s.append(a[t] * s[-1] * (1 - b[t] * k[t] ** 2) + b[t] * k[t] * v[t])
    w = [0.0] * (T + 1)
    w[T] = do[T - 1] * q[T - 1] + dF
    for t in range(T, 1, -1):
        w[t - 1] = do[t - 2] * q[t - 2] + w[t] * a[t - 1] * (1 - b[t - 1] * k[t - 1] ** 2)
    want = dict(
        dq=[do[t] * s[t + 1] for t in range(T)],
        dv=[w[t + 1] * b[t] * k[t] for t in range(T)],
        dbeta=[w[t + 1] * (k[t] * v[t] - a[t] * s[t] * k[t] ** 2) for t in range(T)],
        dk=[w[t + 1] * (b[t] * v[t] - 2 * a[t] * s[t] * b[t] * k[t]) for t in range(T)],
        dlog_alpha=[w[t + 1] * a[t] * s[t] * (1 - b[t] * k[t] ** 2) for t in range(T)],
    )
    sh = lambda x: np.asarray(x, dtype=float).reshape(1, T, 1, 1)
    gr = oracle.backward(sh(q), sh(k), sh(v), sh(g), b.reshape(1, T, 1), sh(do),
                         init_state=np.full((1, 1, 1, 1), s0), dfinal=np.full((1, 1, 1, 1), dF))
    for key, val in want.items():
        got = gr[key].reshape(T)
        np.testing.assert_allclose(got, val, rtol=1e-13, atol=1e-14, err_msg=key)
    np.testing.assert_allclose(gr["dinit_state"].item(), w[1] * a[0] * (1 - b[0] * k[0] ** 2),
                               rtol=1e-13)


def test_identity_gate_zero_beta_closed_form():
    """alpha = 1, beta = 0: the state stays S0, so with R_t = dF + sum_{s>=t} q_s do_s^T
      dq_t = S0 do_t,  dk_t = 0,  dv_t = 0,  dS0 = R_1,
      dbeta_t = k_t^T R_t (v_t - S0^T k_t),   dg_t[c] = sum_j R_t[c][j] S0[c][j]
    (a first-order change of beta_t adds k_t (v_t - S0^T k_t)^T to every later
    state; one of g_t[c] scales row c of every later state)."""
    rng = np.random.default_rng(15)
    x, do, dF = _case(rng, B=1, T=6, H=1, dk=4, dv=3)
    x["log_alpha"][:] = 0.0
    x["beta"][:] = 0.0
    gr = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], do,
                         init_state=x["init_state"], dfinal=dF)
    S0 = x["init_state"][0, 0]
    q, k, v, d = x["q"][0, :, 0], x["k"][0, :, 0], x["v"][0, :, 0], do[0, :, 0]
    T = q.shape[0]
    R = [None] * (T + 1)
    R[T] = dF[0, 0].copy()
    for t in range(T - 1, -1, -1):
        R[t] = R[t + 1] + np.outer(q[t], d[t])
    np.testing.assert_allclose(gr["dq"][0, :, 0], d @ S0.T, rtol=1e-13, atol=1e-13)
    assert np.all(gr["dk"] == 0) and np.all(gr["dv"] == 0)
    np.testing.assert_allclose(gr["dinit_state"][0, 0], R[0], rtol=1e-13, atol=1e-13)
    for t in range(T):
        np.testing.assert_allclose(gr["dbeta"][0, t, 0], k[t] @ R[t] @ (v[t] - S0.T @ k[t]),
                                   rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(gr["dlog_alpha"][0, t, 0], (R[t] * S0).sum(axis=1),
                                   rtol=1e-12, atol=1e-13)


def test_gradients_linear_in_cotangents():
    rng = np.random.default_rng(16)
    x, do, dF = _case(rng, B=1, T=9, H=2)
    do2 = rng.normal(size=do.shape)
    dF2 = rng.normal(size=dF.shape)
    args = (x["q"], x["k"], x["v"], x["log_alpha"], x["beta"])
    g1 = oracle.backward(*args, do, init_state=x["init_state"], dfinal=dF)
    g2 = oracle.backward(*args, do2, init_state=x["init_state"], dfinal=dF2)
    g3 = oracle.backward(*args, 2.0 * do - do2, init_state=x["init_state"], dfinal=2.0 * dF - dF2)
    for _, gname in FIELDS:
        np.testing.assert_allclose(g3[gname], 2.0 * g1[gname] - g2[gname], rtol=1e-10, atol=1e-11)


def test_no_init_state_means_zero_state():
    rng = np.random.default_rng(17)
    x, do, dF = _case(rng, B=1, T=8, H=1)
    args = (x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], do)
    a = oracle.backward(*args, init_state=None, dfinal=dF)
    b = oracle.backward(*args, init_state=np.zeros_like(x["init_state"]), dfinal=dF)
    for _, gname in FIELDS:
        assert np.array_equal(a[gname], b[gname])
    with pytest.raises(ValueError):
        oracle.backward(*args[:5], do[:, :3])


def test_scalar_gate_gradient_is_the_channel_sum():
    """Gated DeltaNet reading: one decay rate per token-head, applied to every key
    channel.  The gradient of such a rate is the sum over the channels of the
    per-channel gradients; checked against central differences that move all
    channels of one (token, head) together."""
    rng = np.random.default_rng(17)
    x, do, dF = _case(rng, B=1, T=9, H=2, dk=4, dv=3)
    g = -np.log1p(np.exp(rng.normal(-2.0, 1.0, size=(1, 9, 2))))
    x["log_alpha"] = np.repeat(g[..., None], 4, axis=-1)
    gr = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], do,
                         init_state=x["init_state"], dfinal=dF)
    d_scalar = gr["dlog_alpha"].sum(axis=-1)
    eps = 1e-6
    for t in range(9):
        for h in range(2):
            xp, xm = dict(x), dict(x)
            xp["log_alpha"] = x["log_alpha"].copy()
            xm["log_alpha"] = x["log_alpha"].copy()
            xp["log_alpha"][0, t, h, :] += eps
            xm["log_alpha"][0, t, h, :] -= eps
            want = (_loss(oracle.forward, xp, do, dF) - _loss(oracle.forward, xm, do, dF)) / (2 * eps)
            assert abs(d_scalar[0, t, h] - want) <= 1e-7 * (1.0 + abs(want)), (t, h, d_scalar[0, t, h], want)
