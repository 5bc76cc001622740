"""The tensor-core kernels' two tiers for the Gram's pairwise decay (numpy model in
chunk_model.py, operands rounded to bf16 as the kernels round them) against the
exact pairwise Gram, on strong decay: hard resets, whole chunks at log_alpha = -2,
mixed channels, and log_alpha = -10 on every token (every block decays past e^80).

A development check of the factorisation the kernels implement, not of the oracle:
in exact arithmetic both tiers equal the pairwise Gram, so only bf16 rounding
separates them."""
import numpy as np
import pytest

from chunk_model import bf16_round, exact_gram, tiered_gram


def _inputs(kind, seed=0, C=64, D=128):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((C, D))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((C, D))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    q, k = bf16_round(q), bf16_round(k)
    g = -np.log1p(np.exp(rng.normal(-2.0, 1.0, (C, D))))
    if kind == "reset":
        for c in rng.choice(D, 20, replace=False):
            g[rng.integers(0, C), c] = -100.0
    elif kind == "minus2":
        g[:] = -2.0
    elif kind == "mixed":
        g[:, :64] = -2.0
        g[:, 64:72] = -10.0
        g[5, 100] = -100.0
    elif kind == "minus10":
        g[:] = -10.0
    return q, k, g


@pytest.mark.parametrize("kind,tier", [("plain", "A"), ("reset", "B"), ("minus2", "B"), ("mixed", "B"),
                                       ("minus10", "B")])
def test_tiers_match_pairwise_gram(kind, tier):
    q, k, g = _inputs(kind)
    want = exact_gram(q, k, g)
    got, t = tiered_gram(q, k, g)
    assert t == tier
    C = k.shape[0]
    mask = np.concatenate([np.tril(np.ones((C, C)), -1), np.tril(np.ones((C, C)))], 0) > 0
    got, want = np.where(mask, got, 0.0), np.where(mask, want, 0.0)
    assert np.all(np.isfinite(got))
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert rel < 5e-3, f"{kind}: rel-L2 {rel:.2e}"
    assert np.max(np.abs(got - want)) < 2e-2


def test_leaving_a_bad_channel_out_is_needed():
    """Planted mistake: without the fp32 diagonal terms a channel reset inside a
    block loses its in-block pairs, and the Gram is visibly wrong."""
    q, k, g = _inputs("minus10")
    want = exact_gram(q, k, g)
    C, D = k.shape
    G = np.cumsum(g, 0)
    # tier B's block products alone (no fp32 diagonal terms)
    x = np.concatenate([k, q], 0)
    blk = (np.arange(2 * C) % C) // 16
    Gs = np.zeros((4, D))
    for b in range(1, 4):
        Gs[b] = G[16 * b - 1]
    A = np.exp(np.concatenate([G, G], 0) - Gs[blk]) * x
    gram = np.zeros((2 * C, C))
    for b in range(4):
        n = 16 * b   # block b's own columns left out entirely
        if n:
            gram[blk == b, :n] = (A @ (np.exp(Gs[b][None, :] - G[:n]) * k[:n]).T)[blk == b]
    mask = np.concatenate([np.tril(np.ones((C, C)), -1), np.tril(np.ones((C, C)))], 0) > 0
    rel = np.linalg.norm(np.where(mask, gram - want, 0)) / np.linalg.norm(np.where(mask, want, 0))
    assert rel > 0.1
