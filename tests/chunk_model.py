"""fp64 numpy model of the chunked KDA algorithm the CUDA kernels implement.

Development aid and derivation check, not the oracle: it regroups the
token recurrence into 64-token chunks ("Kimi Linear、独自の土俵でFull Attentionを
上回る" (remio.ai), § "Kimi Linearがより賢いRecurrent Memoryを使う方法": chunkwise
processing through a diagonal-plus-low-rank transition; "Kimi Delta Attention
徹底解説" (tech-tide.dev), § "Kimi Delta Attention の仕組み": prefill turns the
same computation into large matrix products).  In exact arithmetic it equals
the recurrence, so tests compare it with the oracle to ~1e-12.

Within one chunk of C tokens starting from state S (dk x dv), with
G_i = sum_{s<=i} g_s (per channel, g = log alpha):

  u_i = beta_i (v_i - S^T (e^{G_i} k_i) - sum_{j<i} (k_i . e^{G_i-G_j} k_j) u_j)
  o_i = S^T (e^{G_i} q_i) + sum_{j<=i} (q_i . e^{G_i-G_j} k_j) u_j
  S'  = Diag(e^{G_C}) S + sum_j (e^{G_C-G_j} k_j) u_j^T

In matrix form, with Khat = e^G * K, Qhat = e^G * Q, Kbar = e^{G_C - G} * K,
Akk[i,j] = k_i . e^{G_i-G_j} k_j (j<i), Aqk[i,j] = q_i . e^{G_i-G_j} k_j (j<=i):
  (I + Diag(beta) Akk) U = Diag(beta) (V - Khat S)
so with Tb = (I + Diag(beta) Akk)^{-1} Diag(beta) and Z = V - Khat S:
  U = Tb Z,   O = Qhat S + (Aqk Tb) Z,   S' = Diag(e^{G_C}) S + (Kbar^T Tb) Z.
Pt = Aqk Tb and Kt = Kbar^T Tb do not depend on S.
"""
from __future__ import annotations

import numpy as np


def _chunk(q, k, v, g, b, S, *, pairwise):
    C = q.shape[0]
    G = np.cumsum(g, axis=0)                       # [C, dk]
    if pairwise:
        # exact pairwise decay e^{G_i - G_j} per channel
        D = np.exp(G[:, None, :] - G[None, :, :])  # [i, j, c]
        Akk = np.einsum("ic,jc,ijc->ij", k, k, D)
        Aqk = np.einsum("ic,jc,ijc->ij", q, k, D)
    else:
        # factorised through the chunk start, as the tensor-core kernel does
        Akk = (k * np.exp(G)) @ (k * np.exp(-G)).T
        Aqk = (q * np.exp(G)) @ (k * np.exp(-G)).T
    Akk = np.tril(Akk, -1)
    Aqk = np.tril(Aqk, 0)
    Tb = np.linalg.solve(np.eye(C) + b[:, None] * Akk, np.diag(b))
    Khat = k * np.exp(G)
    Qhat = q * np.exp(G)
    Kbar = k * np.exp(G[-1][None, :] - G)
    Z = v - Khat @ S
    O = Qhat @ S + (Aqk @ Tb) @ Z
    S_new = np.exp(G[-1])[:, None] * S + (Kbar.T @ Tb) @ Z
    return O, S_new


def chunked_forward(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, chunk=64,
                    pairwise=False):
    """Same contract as oracle.forward, computed chunk by chunk in fp64."""
    q, k, v, g, b = (np.asarray(x, dtype=np.float64) for x in (q, k, v, log_alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        spans = [(n, n * T, (n + 1) * T) for n in range(B)]
        N = B
    else:
        cu = list(int(x) for x in cu_seqlens)
        N = len(cu) - 1
        spans = [(n, cu[n], cu[n + 1]) for n in range(N)]
    qf, kf, vf, gf = (x.reshape(B * T, H, -1) for x in (q, k, v, g))
    bf = b.reshape(B * T, H)
    o = np.zeros((B * T, H, dv))
    fs = np.zeros((N, H, dk, dv))
    for n, t0, t1 in spans:
        for h in range(H):
            S = np.zeros((dk, dv)) if init_state is None else np.array(init_state[n, h], dtype=np.float64)
            for c0 in range(t0, t1, chunk):
                c1 = min(t1, c0 + chunk)
                O, S = _chunk(qf[c0:c1, h], kf[c0:c1, h], vf[c0:c1, h], gf[c0:c1, h], bf[c0:c1, h], S,
                              pairwise=pairwise)
                o[c0:c1, h] = O
            fs[n, h] = S
    return o.reshape(B, T, H, dv), fs


# ---------------------------------------------------------------------------
# The tensor-core kernels' split of the Gram's pairwise decay into two operand
# factors (bf16 operands, fp32 exponents), in the two tiers they choose per chunk.

DECAY_LIM = 80.0


def bf16_round(x):
    """Round to bfloat16 (nearest even) and widen back to float64."""
    x = np.asarray(x, np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def exact_gram(q, k, g):
    """[Akk; Aqk] rows (k rows then q rows) x 64 columns: sum_c x_ic k_jc e^{G_ic - G_jc} for j <= i."""
    C = k.shape[0]
    G = np.cumsum(np.asarray(g, np.float64), 0)
    out = np.zeros((2 * C, C))
    x = np.concatenate([k, q], 0)
    for r in range(2 * C):
        i = r % C
        for j in range(i + 1):
            out[r, j] = np.sum(x[r] * k[j] * np.exp(G[i] - G[j]))
    return out


def tiered_gram(q, k, g):
    """The same Gram as the kernels compute it.  Tier A (every channel's chunk
    decay >= -DECAY_LIM): e^{G_i} x_i against e^{-G_j} k_j.  Tier B: per 16-token
    block b, rows scaled from the block start against e^{G_s(b) - G_j} k_j for
    j < 16 (b + 1); channels whose in-block decay passes -DECAY_LIM are left out of
    the block's own columns and their diagonal terms added in fp32 from running
    products of alpha.  Returns (gram, tier)."""
    C, D = k.shape
    g = np.asarray(g, np.float32)
    G = np.cumsum(g, 0, dtype=np.float32)
    x = np.concatenate([k, q], 0)
    Gx = np.concatenate([G, G], 0)
    if np.all(G[-1] >= -DECAY_LIM):
        A = bf16_round(np.exp(Gx) * x)
        B = bf16_round(np.exp(-G) * k)
        return A @ B.T, "A"
    Gs = np.zeros((5, D), np.float32)
    for b in range(1, 5):
        Gs[b] = G[16 * b - 1]
    Gs[4] = G[-1]
    bad = (Gs[1:] - Gs[:4]) < -DECAY_LIM                     # [block, channel]
    blk = (np.arange(2 * C) % C) // 16
    A = bf16_round(np.exp(Gx - Gs[blk]) * x)
    gram = np.zeros((2 * C, C))
    for b in range(4):
        n = 16 * (b + 1)
        Bb = np.exp(np.minimum(Gs[b][None, :] - G[:n], DECAY_LIM)) * k[:n]
        Bb[16 * b:n][:, bad[b]] = 0.0
        Db = A @ bf16_round(Bb).T
        gram[blk == b, :n] = Db[blk == b]
    alpha = np.exp(g).astype(np.float32)
    for r in range(2 * C):
        i = r % C
        b = i // 16
        for c in np.nonzero(bad[b])[0]:
            P = np.float32(1.0)
            for j in range(i, 16 * b - 1, -1):
                gram[r, j] += np.float32(x[r, c]) * np.float32(k[j, c]) * P
                P = np.float32(P * alpha[j, c])
    return gram, "B"
