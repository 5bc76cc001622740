/*
 * KDA oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU statement of what the Kimi Delta Attention (KDA)
 * operator computes.  Only the tests, the package smoke check and the
 * benchmark's CPU-baseline / reference leg may load this library.  The CUDA
 * product path never links, imports or calls it, and shares no code with it.
 *
 * Sources (web pages; the recurrence is stated in words there, the symbols
 * below are this file's own):
 *   [P5] "Kimi Delta Attention 徹底解説" (tech-tide.dev)
 *        § "なぜ今「線形アテンション」なのか": the past is folded into a fixed-size
 *          state through (|v><k|)|q> = <k|q>|v>; here the state S is dk x dv,
 *          so a write is S += k v^T and a read is S^T q.
 *        § "Kimi Delta Attention の仕組み": DeltaNet writes only the error
 *          beta (v - S k); Gated DeltaNet first decays the whole state by a
 *          scalar alpha ("forget first, then remember"); KDA turns alpha into
 *          Diag(alpha), one forget rate per state channel (the key axis dk).
 *          Decode is the token-by-token recurrence; prefill regroups the same
 *          computation into chunks (that form is NOT used here).
 *   [P1] "Kimi Linear、独自の土俵でFull Attentionを上回る" (remio.ai)
 *        § "Kimi Linearがより賢いRecurrent Memoryを使う方法": per-channel
 *          decay gate combined with a delta-rule update of a fixed-size state.
 *
 * For every sequence n and head h independently, with S = init_state[n,h]
 * (or zeros) and t running over the sequence's tokens in order:
 *
 *     S'  = Diag(exp(log_alpha_t)) S        (row c of S scaled by alpha_t[c])
 *     r   = S'^T k_t                        (dv)
 *     S   = S' + beta_t k_t (v_t - r)^T
 *     o_t = S^T q_t                         (read after the write)
 *
 * Layouts (row-major, last index contiguous), identical to the product:
 *   q, k, log_alpha : [B, T, H, dk]     v, o : [B, T, H, dv]
 *   beta            : [B, T, H]         states : [N, H, dk, dv]
 *   varlen          : B == 1, cu_seqlens[N+1] (host int32), sequence n is
 *                     tokens [cu_seqlens[n], cu_seqlens[n+1]); otherwise
 *                     N == B and every sequence has T tokens.
 *
 * Everything is double; inputs are the exact values the GPU receives,
 * widened to double by the caller.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define KDA_ORACLE_OK 0
#define KDA_ORACLE_EINVAL -1
#define KDA_ORACLE_ENOMEM -2

/* Token range [t0, t1) of sequence n in the flattened [B*T] token axis. */
static int seq_range(const int32_t *cu_seqlens, int B, int T, int n, long *t0, long *t1) {
    if (cu_seqlens) {
        *t0 = cu_seqlens[n];
        *t1 = cu_seqlens[n + 1];
        if (*t1 < *t0) return -1;
        (void)B;
    } else {
        *t0 = (long)n * T;
        *t1 = (long)(n + 1) * T;
    }
    return 0;
}

static int check_args(const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv, int num_seqs) {
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ORACLE_EINVAL;
    if (cu_seqlens) {
        if (B != 1 || num_seqs < 0) return KDA_ORACLE_EINVAL;
        if (cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != T) return KDA_ORACLE_EINVAL;
        for (int n = 0; n < num_seqs; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return KDA_ORACLE_EINVAL;
    } else if (num_seqs != B) {
        return KDA_ORACLE_EINVAL;
    }
    return KDA_ORACLE_OK;
}

/*
 * Token-by-token recurrence (the definition above).  init_state and
 * final_state may be NULL.  nthreads <= 0 lets OpenMP choose.
 */
int kda_oracle_forward(const double *q, const double *k, const double *v,
                       const double *log_alpha, const double *beta,
                       const double *init_state, double *o, double *final_state,
                       const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv,
                       int num_seqs, int nthreads) {
    int rc = check_args(cu_seqlens, B, T, H, dk, dv, num_seqs);
    if (rc) return rc;
    if (!q || !k || !v || !log_alpha || !beta || !o) return KDA_ORACLE_EINVAL;
    const long pairs = (long)num_seqs * H;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *r = (double *)malloc(sizeof(double) * (size_t)dv);
        double *alpha = (double *)malloc(sizeof(double) * (size_t)dk);
        if (!S || !r || !alpha) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            failed = 1;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (long p = 0; p < pairs; ++p) {
            if (!S || !r || !alpha) continue;
            const int n = (int)(p / H), h = (int)(p % H);
            long t0, t1;
            seq_range(cu_seqlens, B, T, n, &t0, &t1);
            if (init_state)
                memcpy(S, init_state + (size_t)p * dk * dv, sizeof(double) * (size_t)dk * dv);
            else
                memset(S, 0, sizeof(double) * (size_t)dk * dv);
            for (long t = t0; t < t1; ++t) {
                const size_t tk = ((size_t)t * H + h) * dk;   /* row of q, k, log_alpha */
                const size_t tv = ((size_t)t * H + h) * dv;   /* row of v, o */
                const double b = beta[(size_t)t * H + h];
                /* forget first: S' = Diag(alpha_t) S, alpha on the key axis */
                for (int c = 0; c < dk; ++c) alpha[c] = exp(log_alpha[tk + c]);
                for (int c = 0; c < dk; ++c)
                    for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= alpha[c];
                /* current prediction for key k_t: r = S'^T k_t */
                for (int j = 0; j < dv; ++j) r[j] = 0.0;
                for (int c = 0; c < dk; ++c) {
                    const double kc = k[tk + c];
                    for (int j = 0; j < dv; ++j) r[j] += S[(size_t)c * dv + j] * kc;
                }
                /* then remember: write only the error, scaled by beta_t */
                for (int j = 0; j < dv; ++j) r[j] = b * (v[tv + j] - r[j]);
                for (int c = 0; c < dk; ++c) {
                    const double kc = k[tk + c];
                    for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] += kc * r[j];
                }
                /* read the updated state: o_t = S^T q_t */
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * q[tk + c];
                    o[tv + j] = acc;
                }
            }
            if (final_state)
                memcpy(final_state + (size_t)p * dk * dv, S, sizeof(double) * (size_t)dk * dv);
        }
        free(S);
        free(r);
        free(alpha);
    }
    return failed ? KDA_ORACLE_ENOMEM : KDA_ORACLE_OK;
}

/*
 * Brute-force unrolled form, for tiny sizes only (cost ~ T^2 dk^2 (dk+dv)).
 *
 * The per-token update above is the linear map
 *     S_t = A_t S_{t-1} + beta_t k_t v_t^T,   A_t = (I - beta_t k_t k_t^T) Diag(alpha_t),
 * so
 *     S_t = Phi(t,0) S_0 + sum_{s<=t} Phi(t,s) beta_s k_s v_s^T,
 *     Phi(t,s) = A_t A_{t-1} ... A_{s+1},   Phi(t,t) = I,
 * and o_t = S_t^T q_t.  This routine forms every A_t as an explicit dk x dk
 * matrix and every Phi(t,s) by repeated matrix products; it never runs the
 * decay-then-correct recurrence, so it checks that recurrence independently.
 * Dense (non-varlen) layout only; final_state may be NULL.
 */
int kda_oracle_unrolled(const double *q, const double *k, const double *v,
                        const double *log_alpha, const double *beta,
                        const double *init_state, double *o, double *final_state,
                        int B, int T, int H, int dk, int dv) {
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ORACLE_EINVAL;
    if (!q || !k || !v || !log_alpha || !beta || !o) return KDA_ORACLE_EINVAL;
    const size_t kk = (size_t)dk * dk, kv = (size_t)dk * dv;
    double *A = (double *)malloc(sizeof(double) * kk * (size_t)(T > 0 ? T : 1));
    double *Phi = (double *)malloc(sizeof(double) * kk);
    double *tmp = (double *)malloc(sizeof(double) * kk);
    double *St = (double *)malloc(sizeof(double) * kv);
    if (!A || !Phi || !tmp || !St) {
        free(A); free(Phi); free(tmp); free(St);
        return KDA_ORACLE_ENOMEM;
    }
    int rc = KDA_ORACLE_OK;
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            const size_t pair = (size_t)b * H + h;
            /* A_t = (I - beta k k^T) Diag(alpha): entry (a,c) = (delta_ac - beta k_a k_c) alpha_c */
            for (int t = 0; t < T; ++t) {
                const size_t tk = (((size_t)b * T + t) * H + h) * dk;
                const double bt = beta[((size_t)b * T + t) * H + h];
                double *At = A + (size_t)t * kk;
                for (int a = 0; a < dk; ++a)
                    for (int c = 0; c < dk; ++c)
                        At[(size_t)a * dk + c] =
                            ((a == c ? 1.0 : 0.0) - bt * k[tk + a] * k[tk + c]) * exp(log_alpha[tk + c]);
            }
            for (int t = 0; t < T; ++t) {
                memset(St, 0, sizeof(double) * kv);
                /* Phi = I, then walk s = t, t-1, ..., 0 (0-based tokens; s = -1 means S_0) */
                for (size_t e = 0; e < kk; ++e) Phi[e] = 0.0;
                for (int a = 0; a < dk; ++a) Phi[(size_t)a * dk + a] = 1.0;
                for (int s = t; s >= 0; --s) {
                    const size_t sk = (((size_t)b * T + s) * H + h) * dk;
                    const size_t sv = (((size_t)b * T + s) * H + h) * dv;
                    const double bs = beta[((size_t)b * T + s) * H + h];
                    /* St += Phi * (beta_s k_s v_s^T) */
                    for (int a = 0; a < dk; ++a) {
                        double pk = 0.0;
                        for (int c = 0; c < dk; ++c) pk += Phi[(size_t)a * dk + c] * k[sk + c];
                        for (int j = 0; j < dv; ++j) St[(size_t)a * dv + j] += pk * bs * v[sv + j];
                    }
                    /* Phi = Phi * A_s */
                    const double *As = A + (size_t)s * kk;
                    for (int a = 0; a < dk; ++a)
                        for (int c = 0; c < dk; ++c) {
                            double acc = 0.0;
                            for (int m = 0; m < dk; ++m) acc += Phi[(size_t)a * dk + m] * As[(size_t)m * dk + c];
                            tmp[(size_t)a * dk + c] = acc;
                        }
                    memcpy(Phi, tmp, sizeof(double) * kk);
                }
                /* Phi is now Phi(t,-1) = A_t ... A_0: St += Phi S_0 */
                if (init_state) {
                    const double *S0 = init_state + pair * kv;
                    for (int a = 0; a < dk; ++a)
                        for (int j = 0; j < dv; ++j) {
                            double acc = 0.0;
                            for (int c = 0; c < dk; ++c) acc += Phi[(size_t)a * dk + c] * S0[(size_t)c * dv + j];
                            St[(size_t)a * dv + j] += acc;
                        }
                }
                const size_t tk = (((size_t)b * T + t) * H + h) * dk;
                const size_t tv = (((size_t)b * T + t) * H + h) * dv;
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int a = 0; a < dk; ++a) acc += St[(size_t)a * dv + j] * q[tk + a];
                    o[tv + j] = acc;
                }
                if (final_state && t == T - 1) memcpy(final_state + pair * kv, St, sizeof(double) * kv);
            }
            if (final_state && T == 0) {
                if (init_state)
                    memcpy(final_state + pair * kv, init_state + pair * kv, sizeof(double) * kv);
                else
                    memset(final_state + pair * kv, 0, sizeof(double) * kv);
            }
        }
    }
    free(A); free(Phi); free(tmp); free(St);
    return rc;
}

/*
 * Reverse-mode derivative of kda_oracle_forward (the "chunkwise training
 * algorithm" of "Kimi Linear、独自の土俵でFull Attentionを上回る" (remio.ai),
 * § "Kimi Linearがより賢いRecurrent Memoryを使う方法", needs these gradients;
 * here they are taken of the plain token recurrence, not of any chunk form).
 *
 * For the scalar loss  L = sum_t <do_t, o_t> + <dfinal, S_T>  (do and dfinal
 * are given; dfinal may be NULL = 0) it returns dL/dq, dL/dk, dL/dv,
 * dL/dlog_alpha, dL/dbeta and dL/dinit_state (every output is required;
 * dinit_state is dL/dS_0 whether or not init_state is NULL).
 *
 * One token, written with its intermediates:
 *     a  = exp(g_t)               Sp = Diag(a) S          r = Sp^T k_t
 *     u  = beta_t (v_t - r)       Sn = Sp + k_t u^T       o_t = Sn^T q_t
 * and its adjoint, with dS the adjoint of Sn on entry:
 *     dq_t  = Sn do_t                           dS  += q_t do_t^T
 *     dk_t  = dS u                              du   = dS^T k_t
 *     dbeta = <du, v_t - r>                     dv_t = beta_t du
 *     dr    = -beta_t du                        dSp  = dS + k_t dr^T
 *     dk_t += Sp dr                             dg_t[c] = sum_j dSp[c][j] Sp[c][j]
 *     dS    = Diag(a) dSp                       (adjoint of S before the token)
 * (dg_t uses d exp(g)/dg = exp(g): dL/dg_c = a_c sum_j dSp[c][j] S[c][j].)
 *
 * The reverse sweep needs the state before every token.  They are recomputed,
 * with the forward's own arithmetic, from states kept every KDA_ORACLE_CKPT
 * tokens, so memory is (T / KDA_ORACLE_CKPT + KDA_ORACLE_CKPT) dk dv doubles
 * per (sequence, head) in flight instead of T dk dv; the values are the same.
 */
#define KDA_ORACLE_CKPT 64

/* One forward token on S in place; keeps Sp (the decayed state) and r if asked. */
static void token_forward(double *S, double *Sp, double *r, double *alpha,
                          const double *qt, const double *kt, const double *vt,
                          const double *gt, double bt, int dk, int dv) {
    (void)qt;
    for (int c = 0; c < dk; ++c) alpha[c] = exp(gt[c]);
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= alpha[c];
    if (Sp) memcpy(Sp, S, sizeof(double) * (size_t)dk * dv);
    for (int j = 0; j < dv; ++j) r[j] = 0.0;
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j) r[j] += S[(size_t)c * dv + j] * kt[c];
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] += kt[c] * bt * (vt[j] - r[j]);
}

int kda_oracle_backward(const double *q, const double *k, const double *v,
                        const double *log_alpha, const double *beta,
                        const double *init_state, const double *d_o, const double *dfinal,
                        double *dq, double *dk_out, double *dv_out, double *dlog_alpha,
                        double *dbeta, double *dinit_state,
                        const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv,
                        int num_seqs, int nthreads) {
    int rc = check_args(cu_seqlens, B, T, H, dk, dv, num_seqs);
    if (rc) return rc;
    if (!q || !k || !v || !log_alpha || !beta || !d_o) return KDA_ORACLE_EINVAL;
    if (!dq || !dk_out || !dv_out || !dlog_alpha || !dbeta || !dinit_state) return KDA_ORACLE_EINVAL;
    const long pairs = (long)num_seqs * H;
    const size_t kv = (size_t)dk * dv;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double *S = (double *)malloc(sizeof(double) * kv);
        double *Sp = (double *)malloc(sizeof(double) * kv);
        double *dS = (double *)malloc(sizeof(double) * kv);
        double *seg = (double *)malloc(sizeof(double) * kv * KDA_ORACLE_CKPT);
        double *r = (double *)malloc(sizeof(double) * (size_t)dv);
        double *u = (double *)malloc(sizeof(double) * (size_t)dv);
        double *du = (double *)malloc(sizeof(double) * (size_t)dv);
        double *alpha = (double *)malloc(sizeof(double) * (size_t)dk);
        double *ckpt = NULL;
        size_t ckpt_cap = 0;
        int ok = S && Sp && dS && seg && r && u && du && alpha;
        if (!ok) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            failed = 1;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (long p = 0; p < pairs; ++p) {
            if (!ok) continue;
            const int n = (int)(p / H), h = (int)(p % H);
            long t0, t1;
            seq_range(cu_seqlens, B, T, n, &t0, &t1);
            const long L = t1 - t0;
            const long nck = (L + KDA_ORACLE_CKPT - 1) / KDA_ORACLE_CKPT;
            if ((size_t)(nck > 0 ? nck : 1) > ckpt_cap) {
                free(ckpt);
                ckpt_cap = (size_t)(nck > 0 ? nck : 1);
                ckpt = (double *)malloc(sizeof(double) * kv * ckpt_cap);
                if (!ckpt) {
                    ckpt_cap = 0;
#ifdef _OPENMP
#pragma omp atomic write
#endif
                    failed = 1;
                    continue;
                }
            }
            /* forward: keep the state before tokens t0, t0 + CKPT, t0 + 2 CKPT, ... */
            if (init_state)
                memcpy(S, init_state + (size_t)p * kv, sizeof(double) * kv);
            else
                memset(S, 0, sizeof(double) * kv);
            for (long t = t0; t < t1; ++t) {
                if ((t - t0) % KDA_ORACLE_CKPT == 0)
                    memcpy(ckpt + (size_t)((t - t0) / KDA_ORACLE_CKPT) * kv, S, sizeof(double) * kv);
                const size_t tk = ((size_t)t * H + h) * dk, tv = ((size_t)t * H + h) * dv;
                token_forward(S, NULL, r, alpha, q + tk, k + tk, v + tv, log_alpha + tk,
                              beta[(size_t)t * H + h], dk, dv);
            }
            /* reverse sweep */
            if (dfinal)
                memcpy(dS, dfinal + (size_t)p * kv, sizeof(double) * kv);
            else
                memset(dS, 0, sizeof(double) * kv);
            for (long sgi = nck - 1; sgi >= 0; --sgi) {
                const long s0 = t0 + sgi * KDA_ORACLE_CKPT;
                const long s1 = (s0 + KDA_ORACLE_CKPT < t1) ? s0 + KDA_ORACLE_CKPT : t1;
                /* states before each token of the segment */
                memcpy(S, ckpt + (size_t)sgi * kv, sizeof(double) * kv);
                for (long t = s0; t < s1; ++t) {
                    memcpy(seg + (size_t)(t - s0) * kv, S, sizeof(double) * kv);
                    const size_t tk = ((size_t)t * H + h) * dk, tv = ((size_t)t * H + h) * dv;
                    token_forward(S, NULL, r, alpha, q + tk, k + tk, v + tv, log_alpha + tk,
                                  beta[(size_t)t * H + h], dk, dv);
                }
                for (long t = s1 - 1; t >= s0; --t) {
                    const size_t tk = ((size_t)t * H + h) * dk, tv = ((size_t)t * H + h) * dv;
                    const double bt = beta[(size_t)t * H + h];
                    const double *qt = q + tk, *kt = k + tk, *vt = v + tv, *dot = d_o + tv;
                    /* recompute this token: S <- state after it, Sp, r, u */
                    memcpy(S, seg + (size_t)(t - s0) * kv, sizeof(double) * kv);
                    token_forward(S, Sp, r, alpha, qt, kt, vt, log_alpha + tk, bt, dk, dv);
                    for (int j = 0; j < dv; ++j) u[j] = bt * (vt[j] - r[j]);
                    /* o_t = Sn^T q_t */
                    for (int c = 0; c < dk; ++c) {
                        double acc = 0.0;
                        for (int j = 0; j < dv; ++j) acc += S[(size_t)c * dv + j] * dot[j];
                        dq[tk + c] = acc;
                    }
                    for (int c = 0; c < dk; ++c)
                        for (int j = 0; j < dv; ++j) dS[(size_t)c * dv + j] += qt[c] * dot[j];
                    /* Sn = Sp + k u^T */
                    for (int c = 0; c < dk; ++c) {
                        double acc = 0.0;
                        for (int j = 0; j < dv; ++j) acc += dS[(size_t)c * dv + j] * u[j];
                        dk_out[tk + c] = acc;
                    }
                    for (int j = 0; j < dv; ++j) {
                        double acc = 0.0;
                        for (int c = 0; c < dk; ++c) acc += dS[(size_t)c * dv + j] * kt[c];
                        du[j] = acc;
                    }
                    /* u = beta (v - r) */
                    double db = 0.0;
                    for (int j = 0; j < dv; ++j) db += du[j] * (vt[j] - r[j]);
                    dbeta[(size_t)t * H + h] = db;
                    for (int j = 0; j < dv; ++j) dv_out[tv + j] = bt * du[j];
                    /* r = Sp^T k: dr = -beta du; dSp = dS + k dr^T; dk += Sp dr */
                    for (int j = 0; j < dv; ++j) du[j] = -bt * du[j];
                    for (int c = 0; c < dk; ++c) {
                        double acc = 0.0;
                        for (int j = 0; j < dv; ++j) {
                            dS[(size_t)c * dv + j] += kt[c] * du[j];
                            acc += Sp[(size_t)c * dv + j] * du[j];
                        }
                        dk_out[tk + c] += acc;
                    }
                    /* Sp = Diag(exp(g)) S_prev */
                    for (int c = 0; c < dk; ++c) {
                        double acc = 0.0;
                        for (int j = 0; j < dv; ++j) acc += dS[(size_t)c * dv + j] * Sp[(size_t)c * dv + j];
                        dlog_alpha[tk + c] = acc;
                        for (int j = 0; j < dv; ++j) dS[(size_t)c * dv + j] *= alpha[c];
                    }
                }
            }
            memcpy(dinit_state + (size_t)p * kv, dS, sizeof(double) * kv);
        }
        free(S); free(Sp); free(dS); free(seg); free(r); free(u); free(du); free(alpha); free(ckpt);
    }
    return failed ? KDA_ORACLE_ENOMEM : KDA_ORACLE_OK;
}

/*
 * One decode step for N independent (sequence, head) states, in place:
 * the same recurrence as kda_oracle_forward with T = 1.  q, k, log_alpha
 * are [N, H, dk], v and o are [N, H, dv], beta is [N, H], state [N, H, dk, dv].
 */
int kda_oracle_step(const double *q, const double *k, const double *v,
                    const double *log_alpha, const double *beta,
                    double *state, double *o, int N, int H, int dk, int dv, int nthreads) {
    if (!state) return KDA_ORACLE_EINVAL;
    return kda_oracle_forward(q, k, v, log_alpha, beta, state, o, state, NULL,
                              N, 1, H, dk, dv, N, nthreads);
}

int kda_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
