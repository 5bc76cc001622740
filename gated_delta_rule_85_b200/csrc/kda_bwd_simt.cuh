// KDA chunked backward on CUDA cores, fp32 throughout.
//
// Gradients of L = sum_t <do_t, o_t> + <dS_T, S_T> for the recurrence of
// "Kimi Delta Attention 徹底解説" (tech-tide.dev), § "Kimi Delta Attention の仕組み",
// taken through its chunk form -- the chunkwise training algorithm of
// "Kimi Linear、独自の土俵でFull Attentionを上回る" (remio.ai),
// § "Kimi Linearがより賢いRecurrent Memoryを使う方法".
//
// Forward of one 64-token chunk from state S (G_i = sum_{s<=i} log_alpha_s per
// channel, G_C the last row's; every exponent below is <= 0):
//   Akk[i][j] = sum_c k_ic k_jc e^{G_ic - G_jc}  (j < i)
//   Aqk[i][j] = sum_c q_ic k_jc e^{G_ic - G_jc}  (j <= i)
//   Qh = e^G q, Kh = e^G k, Kb = e^{G_C - G} k, D = e^{G_C}
//   W = V - Kh S;  U_i = beta_i R_i,  R_i = W_i - sum_{j<i} Akk[i][j] U_j
//     (so U = Tb W with Tb = (I + Diag(beta) Akk)^{-1} Diag(beta))
//   O = Qh S + Aqk U;  S_next = Diag(D) S + Kb^T U = Diag(D) S + Kt W,  Kt = Kb^T Tb
// Backward of the chunk, given dO and dS (the adjoint of S_next):
//   dU = Aqk^T dO + Kb dS
//   lam: (I + Diag(beta) Akk)^T lam = dU   (back substitution)
//   mu = beta lam = Pt^T dO + Kt^T dS,  Pt = Aqk Tb
//   dV = mu;  dbeta_i = <lam_i, R_i>
//   dAkk[i][j] = -<mu_i, U_j> (j < i);  dAqk[i][j] = <dO_i, U_j> (j <= i)
//   dQh = dO S^T;  dKh = -mu S^T;  dKb = U dS^T
//   dS_prev = Diag(D) dS + Qh^T dO - Kh^T mu
// and through the decay factors, with a = e^G dKh, b = e^{G_C - G} dKb and
// E_ij = e^{G_i - G_j} per channel:
//   dq_i = e^{G_i} dQh_i + sum_{j<=i} dAqk[i][j] k_j E_ij
//   dk_i = a_i + b_i + sum_{j<i} dAkk[i][j] k_j E_ij
//          + sum_{m>=i} (dAqk[m][i] q_m + [m>i] dAkk[m][i] k_m) E_mi
//   dG_i = q_i (dq_i) + k_i (a_i - b_i + row Akk terms) - k_i (column terms of dk_i)
//   dG_C += D sum_j S[:, j] dS[:, j] + sum_i k_i b_i;   dlog_alpha_s = sum_{i>=s} dG_i
//
// Kernels, in launch order:
//   bwd_prep_kernel   one CTA per (chunk slot, head): G, Akk, Aqk, the decay
//                     factors, T, Tb, Kt and Pt, written as a record.
//   bwd_state_kernel  one CTA per (direction, 32-column value tile, head,
//                     sequence): the only serial work.  Forward it stores the
//                     state at every chunk start (S <- Diag(D) S + Kt (V - Kh S));
//                     backward the adjoint at every chunk end
//                     (dS <- Diag(D) dS + Qh^T dO - Kh^T (Pt^T dO + Kt^T dS)) and dS_0.
//   bwd_part_kernel   one CTA per (chunk slot, head): everything column-separable
//                     (U = Tb W, R = W - Akk U, lam = T^T dU, mu, dV, and the sums
//                     over the value columns of dQh, dKh, dKb, dAqk, dAkk, dbeta,
//                     S.dS), value tile by tile.
// The dense products run on the tensor cores as warp-level m16n8k8 tf32 MMAs
// with fp32 accumulation; for fp32 inputs each operand is split into a tf32
// high part and a tf32 remainder and three products are summed (hi.hi + hi.lo
// + lo.hi), which keeps fp32 accuracy.  Everything else is fp32 on CUDA cores.
//   bwd_chunk_kernel  one CTA per (chunk slot, head): the chain rule through the
//                     decay factors; writes dq, dk, dlog_alpha, dbeta.
// Chunk slots as in the two-pass forward: chunk c of sequence n (tokens
// [t0, t1)) is slot n + floor(t0 / 64) + c.
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace bwd {

constexpr int C = 64;      // chunk length
constexpr int DVT = 32;    // value columns per tile
constexpr int NT = 256;    // threads per CTA
// Padded row strides of shared-memory tiles: 4 mod 32 floats, so the tensor-core
// fragment loads (8 rows x 4 columns per warp) hit 32 distinct banks.
constexpr int TP = DVT + 4;   // [*][DVT]
constexpr int CP = C + 4;     // [*][C]
template <int DK>
struct Pad {
    static constexpr int K = DK + 4;   // [*][DK]
};

inline long long chunk_slots(long long tokens, int num_seqs) { return (tokens + C - 1) / C + num_seqs; }

// Per (chunk slot, head) record of bwd_prep_kernel, in floats.
template <int DK>
struct Rec {
    static constexpr int KH = 0;                 // [C][DK]  e^G k
    static constexpr int QH = KH + C * DK;       // [C][DK]  e^G q
    static constexpr int KB = QH + C * DK;       // [C][DK]  e^{G_C - G} k
    static constexpr int AKK = KB + C * DK;      // [C][C]   strictly lower (zero elsewhere)
    static constexpr int AQK = AKK + C * C;      // [C][C]   lower with the diagonal (zero above)
    static constexpr int TI = AQK + C * C;       // [C][C]   T = (I + Diag(beta) Akk)^{-1}, unit lower
    static constexpr int TB = TI + C * C;        // [C][C]   Tb = T Diag(beta)
    static constexpr int PT = TB + C * C;        // [C][C]   Aqk Tb
    static constexpr int KT = PT + C * C;        // [DK][C]  Kb^T Tb
    static constexpr int D = KT + DK * C;        // [DK]     e^{G_C}
    static constexpr int FLOATS = D + DK;
};

// Per (chunk slot, head) sums over the value columns, in floats.
template <int DK>
struct Part {
    static constexpr int DQ = 0;                 // [C][DK]  dO S^T
    static constexpr int DKH = DQ + C * DK;      // [C][DK]  -mu S^T
    static constexpr int DKB = DKH + C * DK;     // [C][DK]  U dS^T
    static constexpr int AQK = DKB + C * DK;     // [C][C]   <dO_i, U_j>, j <= i (zero above)
    static constexpr int AKK = AQK + C * C;      // [C][C]   -<mu_i, U_j>, j < i (zero elsewhere)
    static constexpr int DB = AKK + C * C;       // [C]      <lam_i, R_i>
    static constexpr int DGC = DB + C;           // [DK]     sum_j S[c][j] dS[c][j]
    static constexpr int FLOATS = DGC + DK;
};

// Workspace, all fp32, per (chunk slot, head): the record, the state at the
// chunk's start [DK][DV], the adjoint at its end [DK][DV], and the sums.
// Regions: rec [slots][H] | ckpt [slots][H] | dckpt [slots][H] | part [slots][H].
template <int DK>
inline size_t ws_floats_per_slot_head(int dv) {
    return (size_t)Rec<DK>::FLOATS + 2 * (size_t)DK * dv + (size_t)Part<DK>::FLOATS;
}

inline size_t backward_workspace_bytes(long long tokens, int H, int dk, int dv, int num_seqs) {
    if (tokens <= 0) return 0;
    const size_t per = dk == 64 ? ws_floats_per_slot_head<64>(dv) : ws_floats_per_slot_head<128>(dv);
    return (size_t)chunk_slots(tokens, num_seqs) * (size_t)H * per * sizeof(float);
}

// Token range of the chunk in `slot`: the owning sequence is the last n whose
// first slot n + floor(t0_n / 64) is <= slot.  False for a slot without a chunk.
__device__ __forceinline__ bool chunk_of_slot(const int32_t *cu_seqlens, int T, int num_seqs, int slot,
                                              long long &cs, int &Lc) {
    int lo = 0, hi = num_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        long long a, b;
        seq_span(cu_seqlens, T, mid, a, b);
        if (mid + a / C <= slot) lo = mid;
        else hi = mid - 1;
    }
    long long t0, t1;
    seq_span(cu_seqlens, T, lo, t0, t1);
    cs = t0 + (long long)(slot - (lo + t0 / C)) * C;
    if (cs < t0 || cs >= t1) return false;
    Lc = (int)min((long long)C, t1 - cs);
    return true;
}

// ------------------------------------------------------------------ tensor-core products

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// d[16 x 8] += A[16 x K] B[K x 8] for one warp.  Element (r, k) of A is
// A[r * ar + k * ak], element (k, n) of B is B[k * bk + n * bn]; K is a multiple
// of 8.  Lane (g = lane / 4, t = lane % 4) holds d rows g and g + 8, columns
// 2t and 2t + 1.  SPLIT sums hi.hi + hi.lo + lo.hi of the tf32 split operands.
template <bool SPLIT>
__device__ __forceinline__ void warp_mma(float (&d)[4], const float *A, int ar, int ak, const float *B, int bk,
                                         int bn, int K) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const float *a_lo = A + g * ar + t * ak, *b_lo = B + t * bk + g * bn;
    for (int k0 = 0; k0 < K; k0 += 8) {
        const float *a = a_lo + k0 * ak, *b = b_lo + k0 * bk;
        const float fa0 = a[0], fa1 = a[8 * ar], fa2 = a[4 * ak], fa3 = a[8 * ar + 4 * ak];
        const float fb0 = b[0], fb1 = b[4 * bk];
        const uint32_t a0 = to_tf32(fa0), a1 = to_tf32(fa1), a2 = to_tf32(fa2), a3 = to_tf32(fa3);
        const uint32_t b0 = to_tf32(fb0), b1 = to_tf32(fb1);
        if (SPLIT) {
            const uint32_t l0 = to_tf32(fa0 - __uint_as_float(a0)), l1 = to_tf32(fa1 - __uint_as_float(a1));
            const uint32_t l2 = to_tf32(fa2 - __uint_as_float(a2)), l3 = to_tf32(fa3 - __uint_as_float(a3));
            const uint32_t m0 = to_tf32(fb0 - __uint_as_float(b0)), m1 = to_tf32(fb1 - __uint_as_float(b1));
            mma_tf32(d, l0, l1, l2, l3, b0, b1);
            mma_tf32(d, a0, a1, a2, a3, m0, m1);
        }
        mma_tf32(d, a0, a1, a2, a3, b0, b1);
    }
}

// Hands the four values a lane holds after warp_mma to epi(row, col, value).
template <typename Epi>
__device__ __forceinline__ void warp_tile_out(const float (&d)[4], int r0, int c0, Epi &&epi) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    epi(r0 + g, c0 + 2 * t, d[0]);
    epi(r0 + g, c0 + 2 * t + 1, d[1]);
    epi(r0 + g + 8, c0 + 2 * t, d[2]);
    epi(r0 + g + 8, c0 + 2 * t + 1, d[3]);
}

// Block product out[M x N] = A1 B1 (+ A2 B2), 16 x 8 output tiles dealt to the
// warps round-robin; every output element goes once through epi(row, col, v).
template <int M, int N, bool SPLIT, typename Epi>
__device__ __forceinline__ void block_mma(const float *A1, int ar1, int ak1, const float *B1, int bk1, int bn1,
                                          int K1, const float *A2, int ar2, int ak2, const float *B2, int bk2,
                                          int bn2, int K2, Epi &&epi) {
    constexpr int NTN = N / 8, TILES = (M / 16) * NTN;
    for (int tile = threadIdx.x >> 5; tile < TILES; tile += NT / 32) {
        const int r0 = (tile / NTN) * 16, c0 = (tile % NTN) * 8;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        warp_mma<SPLIT>(d, A1 + r0 * ar1, ar1, ak1, B1 + c0 * bn1, bk1, bn1, K1);
        if (K2) warp_mma<SPLIT>(d, A2 + r0 * ar2, ar2, ak2, B2 + c0 * bn2, bk2, bn2, K2);
        warp_tile_out(d, r0, c0, epi);
    }
}

// ------------------------------------------------------------------ chunk helpers

// Loads one chunk's q (optional), k and log_alpha rows (zero past Lc) and
// beta, then turns log_alpha into the running sum G (per channel).
template <int DK, typename Tin>
__device__ __forceinline__ void load_chunk_qkg(const Tin *__restrict__ q, const Tin *__restrict__ k,
                                               const float *__restrict__ log_alpha, const float *__restrict__ beta,
                                               long long cs, int Lc, int H, int h, float *sQ, float *sK, float *sG,
                                               float *sB) {
    constexpr int DKP = Pad<DK>::K;
    const int tid = threadIdx.x;
    for (int idx = tid; idx < C * DK; idx += NT) {
        const int i = idx / DK, c = idx % DK;
        float qv = 0.f, kv = 0.f, gv = 0.f;
        if (i < Lc) {
            const long long off = ((cs + i) * H + h) * DK + c;
            if (sQ) qv = Elem<Tin>::load(q + off);
            kv = Elem<Tin>::load(k + off);
            gv = log_alpha[off];
        }
        if (sQ) sQ[i * DKP + c] = qv;
        sK[i * DKP + c] = kv;
        sG[i * DKP + c] = gv;
    }
    for (int i = tid; i < C; i += NT) sB[i] = i < Lc ? beta[(cs + i) * H + h] : 0.f;
    __syncthreads();
    for (int c = tid; c < DK; c += NT) {
        float acc = 0.f;
        for (int i = 0; i < C; ++i) {
            acc += sG[i * DKP + c];
            sG[i * DKP + c] = acc;
        }
    }
    __syncthreads();
}

// Akk (strictly lower) and Aqk (lower with the diagonal), zero elsewhere, with
// the exact pairwise decay.  Row i is paired with row 63 - i for balance.
template <int DK>
__device__ __forceinline__ void chunk_grams(const float *sQ, const float *sK, const float *sG, float *sAkk,
                                            float *sAqk) {
    constexpr int DKP = Pad<DK>::K;
    const int tid = threadIdx.x, l8 = tid & 7, ip = tid >> 3;
    for (int half = 0; half < 2; ++half) {
        const int i = half ? (C - 1 - ip) : ip;
        for (int j = l8; j < C; j += 8) {
            float akk = 0.f, aqk = 0.f;
            if (j <= i) {
                for (int c = 0; c < DK; ++c) {
                    const float kj = sK[j * DKP + c] * expf(sG[i * DKP + c] - sG[j * DKP + c]);
                    akk = fmaf(sK[i * DKP + c], kj, akk);
                    aqk = fmaf(sQ[i * DKP + c], kj, aqk);
                }
            }
            sAkk[i * CP + j] = (j < i) ? akk : 0.f;
            sAqk[i * CP + j] = aqk;
        }
    }
    __syncthreads();
}

// q -> e^G q, k -> e^G k and G -> e^{G_C - G} k; d = e^{G_C}.
template <int DK>
__device__ __forceinline__ void chunk_factors(float *sQ, float *sK, float *sG, float *sD) {
    constexpr int DKP = Pad<DK>::K;
    for (int c = threadIdx.x; c < DK; c += NT) {
        const float gl = sG[(C - 1) * DKP + c];
        sD[c] = expf(gl);
        for (int i = 0; i < C; ++i) {
            const float gi = sG[i * DKP + c];
            const float e = expf(gi);
            const float kc = sK[i * DKP + c];
            sQ[i * DKP + c] *= e;
            sK[i * DKP + c] = kc * e;
            sG[i * DKP + c] = kc * expf(gl - gi);
        }
    }
    __syncthreads();
}

// ------------------------------------------------------------------ prep

template <int DK>
struct PrepSmem {
    static constexpr int DKP = Pad<DK>::K;
    static constexpr int q = 0;                  // [C][DKP] q, then Qh
    static constexpr int k = q + C * DKP;        // [C][DKP] k, then Kh
    static constexpr int g = k + C * DKP;        // [C][DKP] G, then Kb
    static constexpr int akk = g + C * DKP;      // [C][CP]
    static constexpr int aqk = akk + C * CP;     // [C][CP]
    static constexpr int ti = aqk + C * CP;      // [C][CP]  T
    static constexpr int tb = ti + C * CP;       // [C][CP]  Tb
    static constexpr int b = tb + C * CP;        // [C]
    static constexpr int d = b + C;              // [DK]
    static constexpr int total = d + DK;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <int DK, typename Tin>
__global__ void __launch_bounds__(NT, 1)
bwd_prep_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const float *__restrict__ log_alpha,
                const float *__restrict__ beta, const int32_t *__restrict__ cu_seqlens, int T, int H, int num_seqs,
                float *__restrict__ rec) {
    using L = PrepSmem<DK>;
    using R = Rec<DK>;
    constexpr int DKP = L::DKP;
    constexpr bool SPLIT = sizeof(Tin) == 4;
    extern __shared__ float sm[];
    float *sQ = sm + L::q, *sK = sm + L::k, *sG = sm + L::g, *sAkk = sm + L::akk, *sAqk = sm + L::aqk;
    float *sT = sm + L::ti, *sTb = sm + L::tb, *sB = sm + L::b, *sD = sm + L::d;
    const int tid = threadIdx.x, slot = blockIdx.x, h = blockIdx.y;
    long long cs;
    int Lc;
    if (!chunk_of_slot(cu_seqlens, T, num_seqs, slot, cs, Lc)) return;

    load_chunk_qkg<DK, Tin>(q, k, log_alpha, beta, cs, Lc, H, h, sQ, sK, sG, sB);
    chunk_grams<DK>(sQ, sK, sG, sAkk, sAqk);
    chunk_factors<DK>(sQ, sK, sG, sD);
    // T = (I + Diag(beta) Akk)^{-1}, a column of the identity at a time:
    // X_i = [i == col] - beta_i sum_{m<i} Akk[i][m] X_m; 8 lanes per column.
    {
        const int l8 = tid & 7;
        for (int col = tid >> 3; col < C; col += NT / 8) {
            for (int i = 0; i < C; ++i) {
                float part = 0.f;
                for (int m = l8; m < i; m += 8) part = fmaf(sAkk[i * CP + m], sT[m * CP + col], part);
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                part += __shfl_xor_sync(0xffffffffu, part, 2);
                part += __shfl_xor_sync(0xffffffffu, part, 4);
                if (l8 == 0) sT[i * CP + col] = (i == col ? 1.f : 0.f) - sB[i] * part;
                __syncwarp();
            }
        }
    }
    __syncthreads();
    for (int idx = tid; idx < C * C; idx += NT) {
        const int i = idx / C, j = idx % C;
        sTb[i * CP + j] = sT[i * CP + j] * sB[j];
    }
    __syncthreads();
    float *r = rec + ((long long)slot * H + h) * R::FLOATS;
    for (int idx = tid; idx < C * DK; idx += NT) {
        const int i = idx / DK, c = idx % DK;
        r[R::KH + idx] = sK[i * DKP + c];
        r[R::QH + idx] = sQ[i * DKP + c];
        r[R::KB + idx] = sG[i * DKP + c];
    }
    for (int c = tid; c < DK; c += NT) r[R::D + c] = sD[c];
    for (int idx = tid; idx < C * C; idx += NT) {
        const int i = idx / C, j = idx % C;
        r[R::AKK + idx] = sAkk[i * CP + j];
        r[R::AQK + idx] = sAqk[i * CP + j];
        r[R::TI + idx] = sT[i * CP + j];
        r[R::TB + idx] = sTb[i * CP + j];
    }
    // Pt = Aqk Tb;  Kt = Kb^T Tb
    block_mma<C, C, SPLIT>(sAqk, CP, 1, sTb, CP, 1, C, nullptr, 0, 0, nullptr, 0, 0, 0,
                           [&](int i, int j, float x) { r[R::PT + i * C + j] = x; });
    block_mma<DK, C, SPLIT>(sG, 1, DKP, sTb, CP, 1, C, nullptr, 0, 0, nullptr, 0, 0, 0,
                            [&](int c, int j, float x) { r[R::KT + c * C + j] = x; });
}

// ------------------------------------------------------------------ state sweeps

template <int DK>
struct StateSmem {
    static constexpr int DKP = Pad<DK>::K;
    static constexpr int kh = 0;                 // [C][DKP]  Kh
    static constexpr int qh = kh + C * DKP;      // [C][DKP]  Qh (backward)
    static constexpr int kt = qh + C * DKP;      // [DK][CP]  Kt
    static constexpr int pt = kt + DK * CP;      // [C][CP]   Pt (backward)
    static constexpr int s = pt + C * CP;        // [DK][TP]  S or dS
    static constexpr int x = s + DK * TP;        // [C][TP]   V or dO
    static constexpr int y = x + C * TP;         // [C][TP]   W or -mu
    static constexpr int d = y + C * TP;         // [DK]
    static constexpr int total = d + DK;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <int DK, typename Tin>
__global__ void __launch_bounds__(NT, 1)
bwd_state_kernel(const Tin *__restrict__ v, const float *__restrict__ init_state, const Tin *__restrict__ d_o,
                 const float *__restrict__ dfinal, float *__restrict__ dinit_state,
                 const int32_t *__restrict__ cu_seqlens, int T, int H, int DV, const float *__restrict__ rec,
                 float *__restrict__ ckpt, float *__restrict__ dckpt) {
    using L = StateSmem<DK>;
    using R = Rec<DK>;
    constexpr int DKP = L::DKP;
    constexpr bool SPLIT = sizeof(Tin) == 4;
    extern __shared__ float sm[];
    float *sKh = sm + L::kh, *sQh = sm + L::qh, *sKt = sm + L::kt, *sPt = sm + L::pt;
    float *sS = sm + L::s, *sX = sm + L::x, *sY = sm + L::y, *sD = sm + L::d;
    const int tid = threadIdx.x;
    const int ntile = DV / DVT;
    const bool backward = blockIdx.x >= ntile;
    const int tile = blockIdx.x % ntile, col_base = tile * DVT, h = blockIdx.y;
    const int n = seq_for_cta(cu_seqlens, T, (int)gridDim.z);
    long long t0, t1;
    seq_span(cu_seqlens, T, n, t0, t1);
    const long long first = n + t0 / C;
    const int nch = (int)((t1 - t0 + C - 1) / C);
    const long long st_off = ((long long)n * H + h) * DK * DV + col_base;
    const float *src = backward ? dfinal : init_state;
    for (int idx = tid; idx < DK * DVT; idx += NT) {
        const int c = idx / DVT, j = idx % DVT;
        sS[c * TP + j] = src ? src[st_off + (long long)c * DV + j] : 0.f;
    }
    for (int step = 0; step < nch; ++step) {
        const int ci = backward ? nch - 1 - step : step;
        const long long cs = t0 + (long long)ci * C;
        const int Lc = (int)min((long long)C, t1 - cs);
        const long long slot = first + ci;
        const float *rp = rec + (slot * H + h) * R::FLOATS;
        __syncthreads();
        // checkpoint: the state at the chunk's start (forward) or the adjoint at its end
        float *cp = (backward ? dckpt : ckpt) + (slot * H + h) * (long long)DK * DV + col_base;
        for (int idx = tid; idx < DK * DVT; idx += NT) {
            const int c = idx / DVT, j = idx % DVT;
            cp[(long long)c * DV + j] = sS[c * TP + j];
        }
        const Tin *xin = backward ? d_o : v;
        for (int idx = tid; idx < C * DVT; idx += NT) {
            const int i = idx / DVT, j = idx % DVT;
            sX[i * TP + j] = i < Lc ? Elem<Tin>::load(xin + ((cs + i) * H + h) * DV + col_base + j) : 0.f;
        }
        for (int idx = tid; idx < C * DK; idx += NT) {
            const int i = idx / DK, c = idx % DK;
            sKh[i * DKP + c] = rp[R::KH + idx];
            if (backward) sQh[i * DKP + c] = rp[R::QH + idx];
        }
        for (int idx = tid; idx < DK * C; idx += NT) sKt[(idx / C) * CP + idx % C] = rp[R::KT + idx];
        if (backward)
            for (int idx = tid; idx < C * C; idx += NT) sPt[(idx / C) * CP + idx % C] = rp[R::PT + idx];
        for (int c = tid; c < DK; c += NT) sD[c] = rp[R::D + c];
        __syncthreads();
        if (!backward) {
            // W = V - Kh S
            block_mma<C, DVT, SPLIT>(sKh, DKP, 1, sS, TP, 1, DK, nullptr, 0, 0, nullptr, 0, 0, 0,
                                     [&](int i, int j, float x) { sY[i * TP + j] = sX[i * TP + j] - x; });
            __syncthreads();
            // S <- Diag(D) S + Kt W
            block_mma<DK, DVT, SPLIT>(sKt, CP, 1, sY, TP, 1, C, nullptr, 0, 0, nullptr, 0, 0, 0,
                                      [&](int c, int j, float x) { sS[c * TP + j] = sD[c] * sS[c * TP + j] + x; });
        } else {
            // -mu = -(Pt^T dO + Kt^T dS)
            block_mma<C, DVT, SPLIT>(sPt, 1, CP, sX, TP, 1, C, sKt, 1, CP, sS, TP, 1, DK,
                                     [&](int i, int j, float x) { sY[i * TP + j] = -x; });
            __syncthreads();
            // dS <- Diag(D) dS + Qh^T dO + Kh^T (-mu)
            block_mma<DK, DVT, SPLIT>(sQh, 1, DKP, sX, TP, 1, C, sKh, 1, DKP, sY, TP, 1, C,
                                      [&](int c, int j, float x) { sS[c * TP + j] = sD[c] * sS[c * TP + j] + x; });
        }
    }
    __syncthreads();
    if (backward && dinit_state) {
        for (int idx = tid; idx < DK * DVT; idx += NT) {
            const int c = idx / DVT, j = idx % DVT;
            dinit_state[st_off + (long long)c * DV + j] = sS[c * TP + j];
        }
    }
}

// ------------------------------------------------------------------ column-separable terms

template <int DK>
struct PartSmem {
    static constexpr int DKP = Pad<DK>::K;
    static constexpr int kh = 0;                 // [C][DKP]  Kh
    static constexpr int kb = kh + C * DKP;      // [C][DKP]  Kb
    static constexpr int akk = kb + C * DKP;     // [C][CP]
    static constexpr int aqk = akk + C * CP;     // [C][CP]
    static constexpr int ti = aqk + C * CP;      // [C][CP]   T
    static constexpr int tb = ti + C * CP;       // [C][CP]   Tb
    static constexpr int S = tb + C * CP;        // [DK][TP]  state at the chunk's start
    static constexpr int dS = S + DK * TP;       // [DK][TP]  adjoint at its end
    static constexpr int w = dS + DK * TP;       // [C][TP]   v, W, then R
    static constexpr int u = w + C * TP;         // [C][TP]   U
    static constexpr int dout = u + C * TP;      // [C][TP]   dO
    static constexpr int du = dout + C * TP;     // [C][TP]   dU
    static constexpr int lam = du + C * TP;      // [C][TP]   lam, then mu
    static constexpr int b = lam + C * TP;       // [C]
    static constexpr int db = b + C;             // [C]
    static constexpr int total = db + C;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <int DK, typename Tin>
__global__ void __launch_bounds__(NT, 1)
bwd_part_kernel(const Tin *__restrict__ v, const float *__restrict__ beta, const Tin *__restrict__ d_o,
                Tin *__restrict__ dv_out, const int32_t *__restrict__ cu_seqlens, int T, int H, int DV,
                int num_seqs, const float *__restrict__ rec, const float *__restrict__ ckpt,
                const float *__restrict__ dckpt, float *__restrict__ part) {
    using L = PartSmem<DK>;
    using R = Rec<DK>;
    using P = Part<DK>;
    constexpr int DKP = L::DKP;
    constexpr bool SPLIT = sizeof(Tin) == 4;
    constexpr int NW = NT / 32;
    constexpr int TQ = (C / 16) * (DK / 8) / NW;   // [C][DK] output tiles per warp
    constexpr int TA = (C / 16) * (C / 8) / NW;    // [C][C] output tiles per warp
    extern __shared__ float sm[];
    float *sKh = sm + L::kh, *sKb = sm + L::kb, *sAkk = sm + L::akk, *sAqk = sm + L::aqk, *sT = sm + L::ti;
    float *sTb = sm + L::tb, *sS = sm + L::S, *sdS = sm + L::dS, *sW = sm + L::w, *sU = sm + L::u;
    float *sDO = sm + L::dout, *sdU = sm + L::du, *sL = sm + L::lam, *sB = sm + L::b, *sDB = sm + L::db;
    const int tid = threadIdx.x, warp = tid >> 5, slot = blockIdx.x, h = blockIdx.y;
    long long cs;
    int Lc;
    if (!chunk_of_slot(cu_seqlens, T, num_seqs, slot, cs, Lc)) return;
    const float *rp = rec + ((long long)slot * H + h) * R::FLOATS;
    for (int idx = tid; idx < C * DK; idx += NT) {
        const int i = idx / DK, c = idx % DK;
        sKh[i * DKP + c] = rp[R::KH + idx];
        sKb[i * DKP + c] = rp[R::KB + idx];
    }
    for (int idx = tid; idx < C * C; idx += NT) {
        const int i = idx / C, j = idx % C;
        sAkk[i * CP + j] = rp[R::AKK + idx];
        sAqk[i * CP + j] = rp[R::AQK + idx];
        sT[i * CP + j] = rp[R::TI + idx];
        sTb[i * CP + j] = rp[R::TB + idx];
    }
    for (int i = tid; i < C; i += NT) {
        sB[i] = i < Lc ? beta[(cs + i) * H + h] : 0.f;
        sDB[i] = 0.f;
    }
    float a_dq[TQ][4], a_dkh[TQ][4], a_dkb[TQ][4], a_aq[TA][4], a_ak[TA][4], a_gc = 0.f;
#pragma unroll
    for (int r = 0; r < TQ; ++r)
#pragma unroll
        for (int e = 0; e < 4; ++e) a_dq[r][e] = a_dkh[r][e] = a_dkb[r][e] = 0.f;
#pragma unroll
    for (int r = 0; r < TA; ++r)
#pragma unroll
        for (int e = 0; e < 4; ++e) a_aq[r][e] = a_ak[r][e] = 0.f;

    const long long st_base = ((long long)slot * H + h) * DK * DV;
    for (int tile = 0; tile < DV / DVT; ++tile) {
        const int col_base = tile * DVT;
        __syncthreads();   // the previous tile is done with every buffer
        for (int idx = tid; idx < DK * DVT; idx += NT) {
            const int c = idx / DVT, j = idx % DVT;
            sS[c * TP + j] = ckpt[st_base + (long long)c * DV + col_base + j];
            sdS[c * TP + j] = dckpt[st_base + (long long)c * DV + col_base + j];
        }
        for (int idx = tid; idx < C * DVT; idx += NT) {
            const int i = idx / DVT, j = idx % DVT;
            const long long off = ((cs + i) * H + h) * DV + col_base + j;
            sW[i * TP + j] = i < Lc ? Elem<Tin>::load(v + off) : 0.f;
            sDO[i * TP + j] = i < Lc ? Elem<Tin>::load(d_o + off) : 0.f;
        }
        __syncthreads();
        // W = V - Kh S (in place: each element is read and written by its owner only)
        block_mma<C, DVT, SPLIT>(sKh, DKP, 1, sS, TP, 1, DK, nullptr, 0, 0, nullptr, 0, 0, 0,
                                 [&](int i, int j, float x) { sW[i * TP + j] -= x; });
        __syncthreads();
        // U = Tb W;  dU = Aqk^T dO + Kb dS
        block_mma<C, DVT, SPLIT>(sTb, CP, 1, sW, TP, 1, C, nullptr, 0, 0, nullptr, 0, 0, 0,
                                 [&](int i, int j, float x) { sU[i * TP + j] = x; });
        block_mma<C, DVT, SPLIT>(sAqk, 1, CP, sDO, TP, 1, C, sKb, DKP, 1, sdS, TP, 1, DK,
                                 [&](int i, int j, float x) { sdU[i * TP + j] = x; });
        __syncthreads();
        // R = W - Akk U (in place of W);  lam = T^T dU
        block_mma<C, DVT, SPLIT>(sAkk, CP, 1, sU, TP, 1, C, nullptr, 0, 0, nullptr, 0, 0, 0,
                                 [&](int i, int j, float x) { sW[i * TP + j] -= x; });
        block_mma<C, DVT, SPLIT>(sT, 1, CP, sdU, TP, 1, C, nullptr, 0, 0, nullptr, 0, 0, 0,
                                 [&](int i, int j, float x) { sL[i * TP + j] = x; });
        __syncthreads();
        // dbeta: <lam_i, R_i> (one warp per 8 rows; the same lane adds every tile)
        {
            const int lane = tid & 31;
            for (int i = warp * (C / NW); i < (warp + 1) * (C / NW); ++i) {
                float x = sL[i * TP + lane] * sW[i * TP + lane];
                for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                if (lane == 0) sDB[i] += x;
            }
        }
        __syncthreads();
        // mu = beta lam; dV = mu
        for (int idx = tid; idx < C * DVT; idx += NT) {
            const int i = idx / DVT, j = idx % DVT;
            const float mu = sB[i] * sL[i * TP + j];
            sL[i * TP + j] = mu;
            if (i < Lc) Elem<Tin>::store(dv_out + ((cs + i) * H + h) * DV + col_base + j, mu);
        }
        __syncthreads();
        // sums over this tile's columns, kept in registers across tiles:
        // dO S^T, mu S^T, U dS^T ([C][DK]) and dO U^T, mu U^T ([C][C])
#pragma unroll
        for (int r = 0; r < TQ; ++r) {
            const int t2 = warp + r * NW, r0 = (t2 / (DK / 8)) * 16, c0 = (t2 % (DK / 8)) * 8;
            warp_mma<SPLIT>(a_dq[r], sDO + r0 * TP, TP, 1, sS + c0 * TP, 1, TP, DVT);
            warp_mma<SPLIT>(a_dkh[r], sL + r0 * TP, TP, 1, sS + c0 * TP, 1, TP, DVT);
            warp_mma<SPLIT>(a_dkb[r], sU + r0 * TP, TP, 1, sdS + c0 * TP, 1, TP, DVT);
        }
#pragma unroll
        for (int r = 0; r < TA; ++r) {
            const int t2 = warp + r * NW, r0 = (t2 / (C / 8)) * 16, c0 = (t2 % (C / 8)) * 8;
            warp_mma<SPLIT>(a_aq[r], sDO + r0 * TP, TP, 1, sU + c0 * TP, 1, TP, DVT);
            warp_mma<SPLIT>(a_ak[r], sL + r0 * TP, TP, 1, sU + c0 * TP, 1, TP, DVT);
        }
        if (tid < DK)
            for (int j = 0; j < DVT; ++j) a_gc = fmaf(sS[tid * TP + j], sdS[tid * TP + j], a_gc);
    }
    float *pp = part + ((long long)slot * H + h) * P::FLOATS;
#pragma unroll
    for (int r = 0; r < TQ; ++r) {
        const int t2 = warp + r * NW, r0 = (t2 / (DK / 8)) * 16, c0 = (t2 % (DK / 8)) * 8;
        warp_tile_out(a_dq[r], r0, c0, [&](int i, int c, float x) { pp[P::DQ + i * DK + c] = x; });
        warp_tile_out(a_dkh[r], r0, c0, [&](int i, int c, float x) { pp[P::DKH + i * DK + c] = -x; });
        warp_tile_out(a_dkb[r], r0, c0, [&](int i, int c, float x) { pp[P::DKB + i * DK + c] = x; });
    }
#pragma unroll
    for (int r = 0; r < TA; ++r) {
        const int t2 = warp + r * NW, r0 = (t2 / (C / 8)) * 16, c0 = (t2 % (C / 8)) * 8;
        warp_tile_out(a_aq[r], r0, c0, [&](int i, int j, float x) { pp[P::AQK + i * C + j] = j <= i ? x : 0.f; });
        warp_tile_out(a_ak[r], r0, c0, [&](int i, int j, float x) { pp[P::AKK + i * C + j] = j < i ? -x : 0.f; });
    }
    __syncthreads();
    for (int i = tid; i < C; i += NT) pp[P::DB + i] = sDB[i];
    if (tid < DK) pp[P::DGC + tid] = a_gc;
}

// ------------------------------------------------------------------ decay-factor chain rule

template <int DK>
struct ChunkSmem {
    static constexpr int q = 0;                  // [C][DK]
    static constexpr int k = q + C * DK;         // [C][DK]
    static constexpr int g = k + C * DK;         // [C][DK] G
    static constexpr int dk = g + C * DK;        // [C][DK] row terms of dk
    static constexpr int dg = dk + C * DK;       // [C][DK] row terms of dG
    static constexpr int ck = dg + C * DK;       // [C][DK] column terms
    static constexpr int da = ck + C * DK;       // [C][CP] dAqk (j <= i) and dAkk (stored at [j][i], j < i)
    static constexpr int gc = da + C * CP;       // [NT / 2] per row group: sum_i k_i b_i (a dG_C term)
    static constexpr int total = gc + NT / 2;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <int DK, typename Tin>
__global__ void __launch_bounds__(NT, 1)
bwd_chunk_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const float *__restrict__ log_alpha,
                 const float *__restrict__ beta, const int32_t *__restrict__ cu_seqlens, int T, int H, int num_seqs,
                 const float *__restrict__ part, Tin *__restrict__ dq, Tin *__restrict__ dk_out,
                 float *__restrict__ dlog_alpha, float *__restrict__ dbeta) {
    using L = ChunkSmem<DK>;
    using P = Part<DK>;
    extern __shared__ float sm[];
    float *sQ = sm + L::q, *sK = sm + L::k, *sG = sm + L::g, *sDk = sm + L::dk, *sDg = sm + L::dg;
    float *sCk = sm + L::ck, *sDA = sm + L::da, *sGC = sm + L::gc;
    const int tid = threadIdx.x, slot = blockIdx.x, h = blockIdx.y;
    long long cs;
    int Lc;
    if (!chunk_of_slot(cu_seqlens, T, num_seqs, slot, cs, Lc)) return;
    const float *pp = part + ((long long)slot * H + h) * P::FLOATS;

    for (int idx = tid; idx < C * DK; idx += NT) {
        const int i = idx / DK, c = idx % DK;
        float qv = 0.f, kv = 0.f, gv = 0.f;
        if (i < Lc) {
            const long long off = ((cs + i) * H + h) * DK + c;
            qv = Elem<Tin>::load(q + off);
            kv = Elem<Tin>::load(k + off);
            gv = log_alpha[off];
        }
        sQ[idx] = qv;
        sK[idx] = kv;
        sG[idx] = gv;
    }
    // dAqk on and below the diagonal, dAkk transposed above it
    for (int idx = tid; idx < C * C; idx += NT) {
        const int i = idx / C, j = idx % C;
        if (j > i) continue;
        sDA[i * CP + j] = pp[P::AQK + idx];
        if (j < i) sDA[j * CP + i] = pp[P::AKK + idx];
    }
    for (int i = tid; i < Lc; i += NT) dbeta[(cs + i) * H + h] = pp[P::DB + i];
    __syncthreads();
    for (int c = tid; c < DK; c += NT) {
        float acc = 0.f;
        for (int i = 0; i < C; ++i) {
            acc += sG[i * DK + c];
            sG[i * DK + c] = acc;
        }
    }
    __syncthreads();

    // Threads split into DK-wide groups: even groups take row terms (row i),
    // odd groups column terms (column j); with 4 groups (DK = 64) each role
    // alternates rows between its two groups.
    constexpr int NG = NT / DK, NPART = NG / 2;
    const int c = tid % DK, grp = tid / DK, role = grp & 1, prt = grp >> 1;
    const float gC = sG[(C - 1) * DK + c];
    if (role == 0) {
        float kb_sum = 0.f;   // sum_i k_i b_i, a dG_C term
        for (int i = prt; i < C; i += NPART) {
            const float gi = sG[i * DK + c], qi = sQ[i * DK + c], ki = sK[i * DK + c];
            const float eg = expf(gi);
            const float dqh = eg * pp[P::DQ + i * DK + c], a = eg * pp[P::DKH + i * DK + c];
            const float b = expf(gC - gi) * pp[P::DKB + i * DK + c];
            float pq = 0.f, pk = 0.f;
            for (int j = 0; j <= i; ++j) {
                const float kj = sK[j * DK + c] * expf(gi - sG[j * DK + c]);
                pq = fmaf(sDA[i * CP + j], kj, pq);
                if (j < i) pk = fmaf(sDA[j * CP + i], kj, pk);
            }
            if (i < Lc) Elem<Tin>::store(dq + ((cs + i) * H + h) * DK + c, dqh + pq);
            sDk[i * DK + c] = a + b + pk;
            sDg[i * DK + c] = qi * (dqh + pq) + ki * (a - b + pk);
            kb_sum = fmaf(ki, b, kb_sum);
        }
        sGC[prt * DK + c] = kb_sum;
    } else {
        for (int j = prt; j < C; j += NPART) {
            const float gj = sG[j * DK + c];
            float acc = 0.f;
            for (int i = j; i < C; ++i) {
                const float e = expf(sG[i * DK + c] - gj);
                float x = sDA[i * CP + j] * sQ[i * DK + c];
                if (i > j) x = fmaf(sDA[j * CP + i], sK[i * DK + c], x);
                acc = fmaf(x, e, acc);
            }
            sCk[j * DK + c] = acc;
        }
    }
    __syncthreads();
    // dk = row + column terms; dG = row dG - k (column terms); dG_C; dlog_alpha = reverse cumsum
    for (int idx = tid; idx < C * DK; idx += NT) {
        const int i = idx / DK, cc = idx % DK;
        const float ck = sCk[idx];
        if (i < Lc) Elem<Tin>::store(dk_out + ((cs + i) * H + h) * DK + cc, sDk[idx] + ck);
        sDg[idx] -= sK[idx] * ck;
    }
    __syncthreads();
    for (int cc = tid; cc < DK; cc += NT) {
        float acc = expf(sG[(C - 1) * DK + cc]) * pp[P::DGC + cc];
        for (int p2 = 0; p2 < NPART; ++p2) acc += sGC[p2 * DK + cc];
        for (int i = C - 1; i >= 0; --i) {
            acc += sDg[i * DK + cc];
            if (i < Lc) dlog_alpha[((cs + i) * H + h) * DK + cc] = acc;
        }
    }
}

}  // namespace bwd
}  // namespace kda
