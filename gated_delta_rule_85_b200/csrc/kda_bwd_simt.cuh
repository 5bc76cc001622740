// KDA chunked backward: tensor-core products (warp-level mma.sync) with fp32
// accumulation, the rest fp32 on CUDA cores.
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
//     (so U = Tb W with T = (I + Diag(beta) Akk)^{-1}, Tb = T Diag(beta))
//   O = Qh S + Aqk U;  S_next = Diag(D) S + Kb^T U = Diag(D) S + Kt W,  Kt = Kb^T Tb
// Backward of the chunk, given dO and dS (the adjoint of S_next):
//   dU = Aqk^T dO + Kb dS
//   lam = T^T dU   (the adjoint of the forward substitution)
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
//   dG_i = q_i dq_i + k_i (a_i - b_i + the Akk row terms) - k_i (the column terms of dk_i)
//   dG_C += D sum_j S[:, j] dS[:, j] + sum_i k_i b_i;   dlog_alpha_s = sum_{i>=s} dG_i
//
// Kernels, in launch order:
//   bwd_prep_kernel   one CTA per (chunk slot, head): G, Akk, Aqk, the decay
//                     factors, T, Tb, Kt and Pt, written as a record.
//   bwd_state_kernel  one CTA per (direction, 64-column value tile, head,
//                     sequence): the only serial work.  Forward it stores the
//                     state at every chunk start (S <- Diag(D) S + Kt (V - Kh S));
//                     backward the adjoint at every chunk end
//                     (dS <- Diag(D) dS + Qh^T dO - Kh^T (Pt^T dO + Kt^T dS)) and dS_0.
//   bwd_part_kernel   one CTA per (chunk slot, head): everything column-separable
//                     (U = Tb W, R = W - Akk U, lam = T^T dU, mu, dV, and the sums
//                     over the value columns of dQh, dKh, dKb, dAqk, dAkk, dbeta,
//                     S.dS), 32-column value tile by tile.
//   bwd_chunk_kernel  one CTA per (chunk slot, head): the chain rule through the
//                     decay factors; writes dq, dk, dlog_alpha, dbeta.
// Operand precision: fp32 inputs use m16n8k8 tf32 MMAs with each operand split
// into a tf32 high part and remainder, three products summed (hi.hi + hi.lo +
// lo.hi), which keeps fp32 accuracy; bf16 inputs use bf16 m16n8k16 MMAs on the
// state sweeps and column sums (the precision of the forward's tensor-core path)
// and tf32 for the record.  Accumulation is fp32 everywhere.
// Chunk slots as in the two-pass forward: chunk c of sequence n (tokens
// [t0, t1)) is slot n + floor(t0 / 64) + c.
#pragma once

#include "kda_common.cuh"
#include "tc_ptx.cuh"

namespace kda {
namespace bwd {

constexpr int C = 64;      // chunk length
constexpr int DVT = 32;    // value columns per tile
constexpr int NT = 256;    // threads per CTA
constexpr int CHUNK_NT = 512;   // threads per CTA of bwd_chunk_kernel (latency-bound SIMT phases)
constexpr int PREP_NT = 512;    // threads per CTA of bwd_prep_kernel
// threads per CTA of bwd_part_kernel (512 measured no faster, and fp32 inputs'
// split products need more registers than 512 threads leave)
template <typename Tin>
struct PartThreads {
    static constexpr int value = 256;
};
// Padded row strides of shared-memory tiles: 4 mod 32 floats, so the tensor-core
// fragment loads (8 rows x 4 columns per warp) hit 32 distinct banks.
constexpr int TP = DVT + 4;   // [*][DVT]
constexpr int CP = C + 4;     // [*][C]
template <int DK>
struct Pad {
    static constexpr int K = DK + 4;   // [*][DK]
};

inline long long chunk_slots(long long tokens, int num_seqs) { return (tokens + C - 1) / C + num_seqs; }

// Per (chunk slot, head) record of bwd_prep_kernel, in floats.  Rows carry the
// shared-memory padding (stride DK + 4 or C + 4, pad entries unused), so each
// matrix moves between global and shared memory as one bulk copy.
template <int DK>
struct Rec {
    static constexpr int DKP = DK + 4, CPR = C + 4;
    static constexpr int KH = 0;                 // [C][DKP]   e^G k
    static constexpr int QH = KH + C * DKP;      // [C][DKP]   e^G q
    static constexpr int KB = QH + C * DKP;      // [C][DKP]   e^{G_C - G} k
    static constexpr int AKK = KB + C * DKP;     // [C][CPR]   strictly lower (zero elsewhere)
    static constexpr int AQK = AKK + C * CPR;    // [C][CPR]   lower with the diagonal (zero above)
    static constexpr int TI = AQK + C * CPR;     // [C][CPR]   T = (I + Diag(beta) Akk)^{-1}, unit lower
    static constexpr int TB = TI + C * CPR;      // [C][CPR]   Tb = T Diag(beta)
    static constexpr int PT = TB + C * CPR;      // [C][CPR]   Aqk Tb
    static constexpr int KT = PT + C * CPR;      // [DK][CPR]  Kb^T Tb
    static constexpr int D = KT + DK * CPR;      // [DK]       e^{G_C}
    static constexpr int FLOATS = D + DK;
    static constexpr uint32_t ROWS_K = C * DKP * 4, ROWS_C = C * CPR * 4, KT_BYTES = DK * CPR * 4;
};

constexpr long long kWaitLimit = 2000000000ll;   // bounded waits: >= 1 s at any SM clock up to 2 GHz

// Every thread waits for the next phase of a copy barrier; all agree on the
// outcome.  False (and KDA_DEV_WAIT_TIMEOUT flagged) if it did not complete.
__device__ __forceinline__ bool wait_copies(uint32_t mbar, uint32_t &phase) {
    const bool ok = ptx::mbar_wait_bounded(mbar, phase, kWaitLimit);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) {
        if (threadIdx.x == 0) flag_status(KDA_DEV_WAIT_TIMEOUT);
        return false;
    }
    return true;
}

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
// A[r * ar + k * ak], element (k, n) of B is B[k * bk + n * bn]; K (a multiple
// of 8) is a compile-time constant so the k-steps unroll.  Lane (g = lane / 4, t = lane % 4) holds d rows g and g + 8, columns
// 2t and 2t + 1.  SPLIT sums hi.hi + hi.lo + lo.hi of the tf32 split operands.
template <bool SPLIT, int K>
__device__ __forceinline__ void warp_mma(float (&d)[4], const float *A, int ar, int ak, const float *B, int bk,
                                         int bn) {
    static_assert(K % 8 == 0, "K must be a multiple of 8");
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const float *a_lo = A + g * ar + t * ak, *b_lo = B + t * bk + g * bn;
#pragma unroll
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

// d[TW][16 x 8] += A[16 x K] B[K x 8 TW] for one warp: a strip of TW adjacent
// output tiles sharing the A fragment, so TW independent MMAs are in flight per
// k-step instead of one dependent chain.
template <bool SPLIT, int K, int TW>
__device__ __forceinline__ void warp_mma_strip(float (&d)[TW][4], const float *A, int ar, int ak, const float *B,
                                               int bk, int bn) {
    static_assert(K % 8 == 0, "K must be a multiple of 8");
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const float *a_lo = A + g * ar + t * ak, *b_lo = B + t * bk + g * bn;
#pragma unroll
    for (int k0 = 0; k0 < K; k0 += 8) {
        const float *a = a_lo + k0 * ak;
        const float fa0 = a[0], fa1 = a[8 * ar], fa2 = a[4 * ak], fa3 = a[8 * ar + 4 * ak];
        const uint32_t a0 = to_tf32(fa0), a1 = to_tf32(fa1), a2 = to_tf32(fa2), a3 = to_tf32(fa3);
        uint32_t l0 = 0, l1 = 0, l2 = 0, l3 = 0;
        if (SPLIT) {
            l0 = to_tf32(fa0 - __uint_as_float(a0));
            l1 = to_tf32(fa1 - __uint_as_float(a1));
            l2 = to_tf32(fa2 - __uint_as_float(a2));
            l3 = to_tf32(fa3 - __uint_as_float(a3));
        }
#pragma unroll
        for (int w = 0; w < TW; ++w) {
            const float *b = b_lo + k0 * bk + w * 8 * bn;
            const float fb0 = b[0], fb1 = b[4 * bk];
            const uint32_t b0 = to_tf32(fb0), b1 = to_tf32(fb1);
            if (SPLIT) {
                const uint32_t m0 = to_tf32(fb0 - __uint_as_float(b0)), m1 = to_tf32(fb1 - __uint_as_float(b1));
                mma_tf32(d[w], l0, l1, l2, l3, b0, b1);
                mma_tf32(d[w], a0, a1, a2, a3, m0, m1);
            }
            mma_tf32(d[w], a0, a1, a2, a3, b0, b1);
        }
    }
}

// bf16 operands (m16n8k16, fp32 accumulate): the precision of the forward's
// tensor-core path, for bf16 inputs on the serial state sweeps.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two fp32 values (p[0], p[stride]) packed as bf16 (first in the low half).
__device__ __forceinline__ uint32_t pack_bf16x2(const float *p, int stride) {
    float x0, x1;
    if (stride == 1) {
        const float2 v = *reinterpret_cast<const float2 *>(p);
        x0 = v.x;
        x1 = v.y;
    } else {
        x0 = p[0];
        x1 = p[stride];
    }
    __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    return *reinterpret_cast<uint32_t *>(&h);
}

// warp_mma_strip with bf16 operands; K a multiple of 16, pairs along k 8-byte
// aligned when contiguous (even strides and offsets).
template <int K, int TW>
__device__ __forceinline__ void warp_mma_strip_bf16(float (&d)[TW][4], const float *A, int ar, int ak, const float *B,
                                                    int bk, int bn) {
    static_assert(K % 16 == 0, "K must be a multiple of 16");
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const float *a_lo = A + g * ar + 2 * t * ak, *b_lo = B + 2 * t * bk + g * bn;
#pragma unroll
    for (int k0 = 0; k0 < K; k0 += 16) {
        const float *a = a_lo + k0 * ak;
        const uint32_t a0 = pack_bf16x2(a, ak), a1 = pack_bf16x2(a + 8 * ar, ak);
        const uint32_t a2 = pack_bf16x2(a + 8 * ak, ak), a3 = pack_bf16x2(a + 8 * ar + 8 * ak, ak);
#pragma unroll
        for (int w = 0; w < TW; ++w) {
            const float *b = b_lo + k0 * bk + w * 8 * bn;
            mma_bf16_16816(d[w], a0, a1, a2, a3, pack_bf16x2(b, bk), pack_bf16x2(b + 8 * bk, bk));
        }
    }
}

// Block product out[M x N] = A1 B1 (+ A2 B2): each warp takes a strip of one
// 16-row block by TW 8-column tiles; every output element goes once through
// epi(row, col, v).
template <int M, int N, bool SPLIT, int K1, int K2 = 0, int NTH = NT, bool BF = false, typename Epi>
__device__ __forceinline__ void block_mma(const float *A1, int ar1, int ak1, const float *B1, int bk1, int bn1,
                                          const float *A2, int ar2, int ak2, const float *B2, int bk2, int bn2,
                                          Epi &&epi) {
    constexpr int NW = NTH / 32, NTN = N / 8, TILES = (M / 16) * NTN;
    constexpr int TW = TILES >= NW ? TILES / NW : 1;
    static_assert(TILES % NW == 0 || TILES < NW, "tiles must spread evenly over the warps");
    static_assert(NTN % TW == 0, "a strip stays inside one 16-row block");
    constexpr int STRIPS = TILES / TW;
    for (int strip = threadIdx.x >> 5; strip < STRIPS; strip += NW) {
        const int r0 = (strip / (NTN / TW)) * 16, c0 = (strip % (NTN / TW)) * TW * 8;
        float d[TW][4];
#pragma unroll
        for (int w = 0; w < TW; ++w) d[w][0] = d[w][1] = d[w][2] = d[w][3] = 0.f;
        if constexpr (BF) {
            warp_mma_strip_bf16<K1, TW>(d, A1 + r0 * ar1, ar1, ak1, B1 + c0 * bn1, bk1, bn1);
            if constexpr (K2 > 0) warp_mma_strip_bf16<K2, TW>(d, A2 + r0 * ar2, ar2, ak2, B2 + c0 * bn2, bk2, bn2);
        } else {
            warp_mma_strip<SPLIT, K1, TW>(d, A1 + r0 * ar1, ar1, ak1, B1 + c0 * bn1, bk1, bn1);
            if constexpr (K2 > 0) warp_mma_strip<SPLIT, K2, TW>(d, A2 + r0 * ar2, ar2, ak2, B2 + c0 * bn2, bk2, bn2);
        }
#pragma unroll
        for (int w = 0; w < TW; ++w) warp_tile_out(d[w], r0, c0 + 8 * w, epi);
    }
}

// ------------------------------------------------------------------ chunk helpers

// Loads one chunk's q, k and log_alpha rows (zero past Lc) and beta (if sB),
// then turns log_alpha into the running sum G (per channel).  GS: log_alpha is
// one value per (token, head) (Gated DeltaNet), broadcast over the channels.  Every thread
// issues all of its 4-element vector loads before the first shared store.
template <int DK, typename Tin, int NTH = NT, bool GS = false>
__device__ __forceinline__ void load_chunk_qkg(const Tin *__restrict__ q, const Tin *__restrict__ k,
                                               const float *__restrict__ log_alpha, const float *__restrict__ beta,
                                               long long cs, int Lc, int H, int h, float *sQ, float *sK, float *sG,
                                               float *sB) {
    constexpr int DKP = Pad<DK>::K;
    constexpr int NV = C * DK / 4 / NTH;   // 4-element vectors per thread and tensor
    const int tid = threadIdx.x;
    float4 rq[NV], rk[NV], rg[NV];
#pragma unroll
    for (int u = 0; u < NV; ++u) {
        const int e = (tid + u * NTH) * 4, i = e / DK, c = e % DK;
        rq[u] = rk[u] = rg[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < Lc) {
            const long long off = ((cs + i) * H + h) * DK + c;
            rq[u] = load4(q + off);
            rk[u] = load4(k + off);
            if constexpr (GS) {   // one decay rate per (token, head), broadcast over the key channels
                const float gs = log_alpha[(cs + i) * H + h];
                rg[u] = make_float4(gs, gs, gs, gs);
            } else {
                rg[u] = *reinterpret_cast<const float4 *>(log_alpha + off);
            }
        }
    }
    const float bv = (sB && tid < C && tid < Lc) ? beta[(cs + tid) * H + h] : 0.f;
#pragma unroll
    for (int u = 0; u < NV; ++u) {
        const int e = (tid + u * NTH) * 4, i = e / DK, c = e % DK;
        *reinterpret_cast<float4 *>(sQ + i * DKP + c) = rq[u];
        *reinterpret_cast<float4 *>(sK + i * DKP + c) = rk[u];
        *reinterpret_cast<float4 *>(sG + i * DKP + c) = rg[u];
    }
    if (sB && tid < C) sB[tid] = bv;
    __syncthreads();
    for (int c = tid; c < DK; c += NTH) {
        float acc = 0.f;
        for (int i = 0; i < C; ++i) {
            acc += sG[i * DKP + c];
            sG[i * DKP + c] = acc;
        }
    }
    __syncthreads();
}

__device__ __forceinline__ void cp_async16(float *dst, const float *src) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// rows x cols fp32 (cols a multiple of 4; source rows src_ld apart, default
// cols) into shared rows of stride ld, as 16-byte asynchronous copies.
__device__ __forceinline__ void async_rows(float *dst, int ld, const float *src, int rows, int cols,
                                           long long src_ld = -1) {
    const int q4 = cols / 4;
    const long long sld = src_ld < 0 ? cols : src_ld;
    for (int idx = threadIdx.x; idx < rows * q4; idx += blockDim.x) {
        const int r = idx / q4, c4 = (idx % q4) * 4;
        cp_async16(dst + r * ld + c4, src + r * sld + c4);
    }
}

// 16-row sub-blocks of a chunk.  For i in a later block than j, with r the
// first row of i's block (j < r <= i) or s the last row of j's block
// (j <= s < i), the decay factors split into two factors that are both <= 1:
//   e^{G_i - G_j} = e^{G_i - G_r} e^{G_r - G_j} = e^{G_i - G_s} e^{G_s - G_j}
// so the off-diagonal blocks become products of decay-scaled operands on the
// tensor cores; only the 16 x 16 diagonal blocks take the exact pairwise exponent.
constexpr int SB = 16;             // sub-block rows
constexpr int NSB = C / SB;        // sub-blocks per chunk
constexpr int SCR_ROWS = C - SB;   // largest off-diagonal operand (48 rows)
constexpr float DIAG_RANGE = 40.f;   // largest in-block log-decay taken through a block boundary

// True when every channel decays by at most DIAG_RANGE (in log) across each
// 16-row block, so the diagonal blocks can go through the block boundary with a
// factor of at most e^DIAG_RANGE.  Uniform over the CTA (it synchronises).
template <int DK, int NTH>
__device__ __forceinline__ bool diag_blocks_in_range(const float *sG) {
    constexpr int DKP = Pad<DK>::K;
    bool bad = false;
    for (int c = threadIdx.x; c < DK; c += NTH)
#pragma unroll
        for (int b = 0; b < NSB; ++b) bad |= sG[(b * SB) * DKP + c] - sG[(b * SB + SB - 1) * DKP + c] > DIAG_RANGE;
    return !__syncthreads_or(bad);
}

// Akk (strictly lower) and Aqk (lower with the diagonal), zero elsewhere.
// scr holds 2 SB + C rows of stride DKP.  The diagonal blocks take the exact
// pairwise exponent unless `diag` (every block's decay range within DIAG_RANGE),
// in which case they join the tensor-core products through the block boundary.
template <int DK, bool SPLIT, int NTH>
__device__ __forceinline__ void chunk_grams(const float *sQ, const float *sK, const float *sG, float *sAkk,
                                            float *sAqk, float *scr, bool diag) {
    constexpr int DKP = Pad<DK>::K;
    const int tid = threadIdx.x;
    for (int idx = tid; idx < C * CP; idx += NTH) {
        sAkk[idx] = 0.f;
        sAqk[idx] = 0.f;
    }
    __syncthreads();
    if (!diag) {   // diagonal blocks, exact: 8 lanes per (i, j) pair, each lane DK / 8 channels
        constexpr int PAIRS = NSB * SB * (SB + 1) / 2;
        const int l8 = tid & 7;
        static_assert((PAIRS % (NTH / 8)) % 4 == 0, "uniform trip counts within each warp");
        for (int p = tid >> 3; p < PAIRS; p += NTH / 8) {
            const int b = p / (SB * (SB + 1) / 2);
            int rem = p % (SB * (SB + 1) / 2), ii = 0;
            while (rem > ii) rem -= ++ii;
            const int i = b * SB + ii, j = b * SB + rem;   // rem <= ii
            float akk = 0.f, aqk = 0.f;
            for (int c = l8; c < DK; c += 8) {
                const float kj = sK[j * DKP + c] * __expf(sG[i * DKP + c] - sG[j * DKP + c]);
                akk = fmaf(sK[i * DKP + c], kj, akk);
                aqk = fmaf(sQ[i * DKP + c], kj, aqk);
            }
            for (int o = 1; o < 8; o <<= 1) {
                akk += __shfl_xor_sync(0xffffffffu, akk, o);
                aqk += __shfl_xor_sync(0xffffffffu, aqk, o);
            }
            if (l8 == 0) {
                if (j < i) sAkk[i * CP + j] = akk;
                sAqk[i * CP + j] = aqk;
            }
        }
    }
    // rows of block bi against the scaled keys of rows j < r (and, with `diag`,
    // of the block itself, j < r + 16, masked to j < i / j <= i)
    float *sL = scr, *sR = scr + 2 * SB * DKP;   // [k; q] rows of block bi, then k_j e^{G_r - G_j}
    for (int bi = diag ? 0 : 1; bi < NSB; ++bi) {
        const int r = bi * SB, ncol = diag ? r + SB : r;
        __syncthreads();
        for (int idx = tid; idx < SB * DK; idx += NTH) {
            const int ii = idx / DK, c = idx % DK, i = r + ii;
            const float e = __expf(sG[i * DKP + c] - sG[r * DKP + c]);
            sL[ii * DKP + c] = sK[i * DKP + c] * e;
            sL[(SB + ii) * DKP + c] = sQ[i * DKP + c] * e;
        }
        for (int idx = tid; idx < ncol * DK; idx += NTH) {
            const int j = idx / DK, c = idx % DK;
            sR[j * DKP + c] = sK[j * DKP + c] * __expf(sG[r * DKP + c] - sG[j * DKP + c]);
        }
        __syncthreads();
        const int ntn = ncol / 8;
        for (int t = tid >> 5; t < 2 * ntn; t += NTH / 32) {
            const int r0 = (t / ntn) * SB, c0 = (t % ntn) * 8;
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            warp_mma<SPLIT, DK>(d, sL + r0 * DKP, DKP, 1, sR + c0 * DKP, 1, DKP);
            warp_tile_out(d, r0, c0, [&](int row, int j, float x) {
                if (row < SB) {
                    const int i = r + row;
                    if (j < i) sAkk[i * CP + j] = x;
                } else {
                    const int i = r + row - SB;
                    if (j <= i) sAqk[i * CP + j] = x;
                }
            });
        }
    }
    __syncthreads();
}

// q -> e^G q, k -> e^G k and G -> e^{G_C - G} k; d = e^{G_C}.  Every thread keeps
// one channel (NTH is a multiple of DK) and takes every (NTH / DK)-th row; G_C is
// read by all before any row is overwritten.
template <int DK, int NTH>
__device__ __forceinline__ void chunk_factors(float *sQ, float *sK, float *sG, float *sD) {
    constexpr int DKP = Pad<DK>::K, RSTEP = NTH / DK;
    static_assert(NTH % DK == 0, "one channel per thread");
    const int c = threadIdx.x % DK, i0 = threadIdx.x / DK;
    const float gl = sG[(C - 1) * DKP + c];
    if (i0 == 0) sD[c] = __expf(gl);
    __syncthreads();
    for (int i = i0; i < C; i += RSTEP) {
        const float gi = sG[i * DKP + c];
        const float e = __expf(gi);
        const float kc = sK[i * DKP + c];
        sQ[i * DKP + c] *= e;
        sK[i * DKP + c] = kc * e;
        sG[i * DKP + c] = kc * __expf(gl - gi);
    }
    __syncthreads();
}

// Block row BI (rows r..r+15, r = 16 BI) of T = (I + Diag(beta) Akk)^{-1} below
// the diagonal, from its diagonal block and the block rows above:
//   Y = Diag(beta) Akk[r..r+16)[0..r) T[0..r)[0..r)   (in scr)
//   T[r..r+16)[0..r) = -T[r..r+16)[r..r+16) Y
template <bool SPLIT, int BI, int NTH>
__device__ __forceinline__ void t_block_row(const float *sAkk, const float *sB, float *sT, float *scr) {
    constexpr int r = BI * SB;
    __syncthreads();
    block_mma<SB, r, SPLIT, r, 0, NTH>(sAkk + r * CP, CP, 1, sT, CP, 1, nullptr, 0, 0, nullptr, 0, 0,
                               [&](int ii, int j, float x) { scr[ii * CP + j] = sB[r + ii] * x; });
    __syncthreads();
    block_mma<SB, r, SPLIT, SB, 0, NTH>(sT + r * CP + r, CP, 1, scr, CP, 1, nullptr, 0, 0, nullptr, 0, 0,
                                [&](int ii, int j, float x) { sT[(r + ii) * CP + j] = -x; });
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
    static constexpr int scr = tb + C * CP;      // [2 SB + C][DKP] Gram operands
    static constexpr int b = scr + (2 * SB + C) * DKP;   // [C]
    static constexpr int d = b + C;              // [DK]
    static constexpr int total = d + DK;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <int DK, typename Tin, bool GS>
__global__ void __launch_bounds__(PREP_NT, 1)
bwd_prep_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const float *__restrict__ log_alpha,
                const float *__restrict__ beta, const int32_t *__restrict__ cu_seqlens, int T, int H, int num_seqs,
                float *__restrict__ rec) {
    using L = PrepSmem<DK>;
    using R = Rec<DK>;
    constexpr int DKP = L::DKP;
    constexpr bool SPLIT = sizeof(Tin) == 4;
    constexpr int NTH = PREP_NT;
    extern __shared__ __align__(128) float sm[];
    float *sQ = sm + L::q, *sK = sm + L::k, *sG = sm + L::g, *sAkk = sm + L::akk, *sAqk = sm + L::aqk;
    float *sT = sm + L::ti, *sTb = sm + L::tb, *sB = sm + L::b, *sD = sm + L::d;
    const int tid = threadIdx.x, slot = blockIdx.x, h = blockIdx.y;
    long long cs;
    int Lc;
    if (!chunk_of_slot(cu_seqlens, T, num_seqs, slot, cs, Lc)) return;

    load_chunk_qkg<DK, Tin, NTH, GS>(q, k, log_alpha, beta, cs, Lc, H, h, sQ, sK, sG, sB);
    chunk_grams<DK, SPLIT, NTH>(sQ, sK, sG, sAkk, sAqk, sm + L::scr, diag_blocks_in_range<DK, NTH>(sG));
    chunk_factors<DK, NTH>(sQ, sK, sG, sD);
    // T = (I + Diag(beta) Akk)^{-1}: the 16 x 16 diagonal blocks by forward
    // substitution (4 lanes per column, all 64 columns at once), then each block
    // row below the diagonal from the rows above it (t_block_row).
    for (int idx = tid; idx < C * CP; idx += NTH) sT[idx] = 0.f;
    __syncthreads();
    if (tid < NSB * SB * 4) {   // 64 columns x 4 lanes: whole warps, so the shuffles stay full
        const int prob = tid >> 2, l4 = tid & 3, b0 = (prob / SB) * SB, col = prob % SB;
        for (int ii = 0; ii < SB; ++ii) {
            const int i = b0 + ii;
            float part = 0.f;
            for (int m = l4; m < ii; m += 4) part = fmaf(sAkk[i * CP + b0 + m], sT[(b0 + m) * CP + b0 + col], part);
            part += __shfl_xor_sync(0xffffffffu, part, 1);
            part += __shfl_xor_sync(0xffffffffu, part, 2);
            if (l4 == 0) sT[i * CP + b0 + col] = (ii == col ? 1.f : 0.f) - sB[i] * part;
            __syncwarp();
        }
    }
    t_block_row<SPLIT, 1, NTH>(sAkk, sB, sT, sm + L::scr);
    t_block_row<SPLIT, 2, NTH>(sAkk, sB, sT, sm + L::scr);
    t_block_row<SPLIT, 3, NTH>(sAkk, sB, sT, sm + L::scr);
    __syncthreads();
    for (int idx = tid; idx < C * C; idx += NTH) {
        const int i = idx / C, j = idx % C;
        sTb[i * CP + j] = sT[i * CP + j] * sB[j];
    }
    __syncthreads();
    float *r = rec + ((long long)slot * H + h) * R::FLOATS;
    // the shared-memory matrices already have the record's row layout: one bulk store each
    if (tid == 0) {
        ptx::fence_proxy_async_smem();
        ptx::bulk_store(r + R::KH, ptx::smem_u32(sK), R::ROWS_K);
        ptx::bulk_store(r + R::QH, ptx::smem_u32(sQ), R::ROWS_K);
        ptx::bulk_store(r + R::KB, ptx::smem_u32(sG), R::ROWS_K);
        ptx::bulk_store(r + R::AKK, ptx::smem_u32(sAkk), R::ROWS_C);
        ptx::bulk_store(r + R::AQK, ptx::smem_u32(sAqk), R::ROWS_C);
        ptx::bulk_store(r + R::TI, ptx::smem_u32(sT), R::ROWS_C);
        ptx::bulk_store(r + R::TB, ptx::smem_u32(sTb), R::ROWS_C);
        ptx::bulk_store(r + R::D, ptx::smem_u32(sD), DK * 4);
        ptx::bulk_commit();
    }
    // Pt = Aqk Tb;  Kt = Kb^T Tb
    block_mma<C, C, SPLIT, C, 0, NTH>(sAqk, CP, 1, sTb, CP, 1, nullptr, 0, 0, nullptr, 0, 0,
                              [&](int i, int j, float x) { r[R::PT + i * CP + j] = x; });
    block_mma<DK, C, SPLIT, C, 0, NTH>(sG, 1, DKP, sTb, CP, 1, nullptr, 0, 0, nullptr, 0, 0,
                               [&](int c, int j, float x) { r[R::KT + c * CP + j] = x; });
    if (tid == 0) ptx::bulk_wait_read_all();   // shared memory stays valid until the stores have read it
}

// ------------------------------------------------------------------ state sweeps

constexpr int SV = 64;        // value columns per state-sweep CTA
constexpr int SVP = SV + 4;   // padded row stride of [*][SV] tiles

template <int DK>
struct StateSmem {
    static constexpr int DKP = Pad<DK>::K;
    static constexpr int kh = 0;                 // [C][DKP]  Kh
    static constexpr int qh = kh + C * DKP;      // [C][DKP]  Qh (backward)
    static constexpr int kt = qh + C * DKP;      // [DK][CP]  Kt
    static constexpr int pt = kt + DK * CP;      // [C][CP]   Pt (backward)
    static constexpr int s = pt + C * CP;        // [DK][SVP] S or dS
    static constexpr int x = s + DK * SVP;       // [C][SVP]  V or dO
    static constexpr int y = x + C * SVP;        // [C][SVP]  W or -mu
    static constexpr int d = y + C * SVP;        // [DK]      e^{G_C}
    static constexpr int total = d + DK;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

// Each chunk is two products, and each product's record matrices are one group
// of asynchronous copies issued while the other product runs:
//   forward   A: W = V - Kh S            {Kh}          B: S <- Diag(D) S + Kt W     {Kt, D}
//   backward  A: -mu = -(Pt^T dO + Kt^T dS) {Pt, Kt}   B: dS <- Diag(D) dS + Qh^T dO + Kh^T (-mu)  {Qh, Kh, D}
// Groups are committed in the order A(0), B(0), A(1), B(1), ... (empty past the
// last chunk), so "all but the most recent group done" is always the one needed.
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
    constexpr bool BF = sizeof(Tin) == 2;   // bf16 inputs: bf16 operands, as the forward's tensor-core path
    extern __shared__ __align__(128) float sm[];
    float *sKh = sm + L::kh, *sQh = sm + L::qh, *sKt = sm + L::kt, *sPt = sm + L::pt;
    float *sS = sm + L::s, *sX = sm + L::x, *sY = sm + L::y, *sD = sm + L::d;
    const int tid = threadIdx.x;
    const int ntile = DV / SV;
    const bool backward = blockIdx.x >= ntile;
    const int tile = blockIdx.x % ntile, col_base = tile * SV, h = blockIdx.y;
    const int n = seq_for_cta(cu_seqlens, T, (int)gridDim.z);
    long long t0, t1;
    seq_span(cu_seqlens, T, n, t0, t1);
    const long long first = n + t0 / C;
    const int nch = (int)((t1 - t0 + C - 1) / C);
    const long long st_off = ((long long)n * H + h) * DK * DV + col_base;
    const float *src = backward ? dfinal : init_state;
    for (int idx = tid; idx < DK * SV; idx += NT) {
        const int c = idx / SV, j = idx % SV;
        sS[c * SVP + j] = src ? src[st_off + (long long)c * DV + j] : 0.f;
    }
    auto rec_of = [&](int step) {
        const int ci = backward ? nch - 1 - step : step;
        return rec + ((first + ci) * H + h) * (long long)R::FLOATS;
    };
    // one thread issues each group as bulk copies completing on its barrier
    __shared__ __align__(8) uint64_t bars[2];
    const uint32_t bar_a = ptx::smem_u32(&bars[0]), bar_b = ptx::smem_u32(&bars[1]);
    uint32_t ph_a = 0, ph_b = 0;
    bool pend_a = false, pend_b = false;
    if (tid == 0) {
        ptx::mbar_init(bar_a, 1);
        ptx::mbar_init(bar_b, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    auto issue_a = [&](int step) {
        if (step >= nch) return;
        pend_a = true;
        if (tid != 0) return;
        const float *rp = rec_of(step);
        if (backward) {
            ptx::mbar_arrive_expect_tx(bar_a, R::ROWS_C + R::KT_BYTES);
            ptx::bulk_load(ptx::smem_u32(sPt), rp + R::PT, R::ROWS_C, bar_a);
            ptx::bulk_load(ptx::smem_u32(sKt), rp + R::KT, R::KT_BYTES, bar_a);
        } else {
            ptx::mbar_arrive_expect_tx(bar_a, R::ROWS_K);
            ptx::bulk_load(ptx::smem_u32(sKh), rp + R::KH, R::ROWS_K, bar_a);
        }
    };
    auto issue_b = [&](int step) {
        if (step >= nch) return;
        pend_b = true;
        if (tid != 0) return;
        const float *rp = rec_of(step);
        if (backward) {
            ptx::mbar_arrive_expect_tx(bar_b, 2 * R::ROWS_K + DK * 4);
            ptx::bulk_load(ptx::smem_u32(sQh), rp + R::QH, R::ROWS_K, bar_b);
            ptx::bulk_load(ptx::smem_u32(sKh), rp + R::KH, R::ROWS_K, bar_b);
        } else {
            ptx::mbar_arrive_expect_tx(bar_b, R::KT_BYTES + DK * 4);
            ptx::bulk_load(ptx::smem_u32(sKt), rp + R::KT, R::KT_BYTES, bar_b);
        }
        ptx::bulk_load(ptx::smem_u32(sD), rp + R::D, DK * 4, bar_b);
    };
    bool ok = true;
    // V (forward) or dO (backward) rows of a chunk, this thread's share, as raw
    // 16-byte vectors in registers (converted only when stored to shared memory)
    constexpr int XV = 16 / (int)sizeof(Tin);       // elements per vector
    constexpr int XPT = C * SV / XV / NT;           // vectors per thread
    uint4 xr[XPT];
    const Tin *xin = backward ? d_o : v;
    auto load_x = [&](int step) {
        const int ci = backward ? nch - 1 - step : step;
        const long long cs = t0 + (long long)ci * C;
        const int Lc = (int)min((long long)C, t1 - cs);
#pragma unroll
        for (int u = 0; u < XPT; ++u) {
            const int e = (tid + u * NT) * XV, i = e / SV, j = e % SV;
            xr[u] = i < Lc ? *reinterpret_cast<const uint4 *>(xin + ((cs + i) * H + h) * DV + col_base + j)
                           : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    issue_a(0);
    issue_b(0);
    for (int step = 0; step < nch; ++step) {
        const int ci = backward ? nch - 1 - step : step;
        const long long cs = t0 + (long long)ci * C;
        const int Lc = (int)min((long long)C, t1 - cs);
        const long long slot = first + ci;
        __syncthreads();   // S (or dS) final for this chunk; X free
        // checkpoint: the state at the chunk's start (forward) or the adjoint at its end
        float *cp = (backward ? dckpt : ckpt) + (slot * H + h) * (long long)DK * DV + col_base;
        for (int idx = tid; idx < DK * SV / 4; idx += NT) {
            const int c = idx / (SV / 4), j = (idx % (SV / 4)) * 4;
            *reinterpret_cast<float4 *>(cp + (long long)c * DV + j) = *reinterpret_cast<const float4 *>(sS + c * SVP + j);
        }
        if (step == 0) load_x(step);
#pragma unroll
        for (int u = 0; u < XPT; ++u) {
            const int e = (tid + u * NT) * XV, i = e / SV, j = e % SV;
            float *dst = sX + i * SVP + j;
            if constexpr (sizeof(Tin) == 2) {
                const uint32_t w[4] = {xr[u].x, xr[u].y, xr[u].z, xr[u].w};
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[q2]));
                    dst[2 * q2] = f.x;
                    dst[2 * q2 + 1] = f.y;
                }
            } else {
                *reinterpret_cast<uint4 *>(dst) = xr[u];
            }
        }
        pend_a = false;
        if (!(ok = wait_copies(bar_a, ph_a))) break;   // group A of this chunk
        if (!backward)
            block_mma<C, SV, SPLIT, DK, 0, NT, BF>(sKh, DKP, 1, sS, SVP, 1, nullptr, 0, 0, nullptr, 0, 0,
                                    [&](int i, int j, float x) { sY[i * SVP + j] = sX[i * SVP + j] - x; });
        else
            block_mma<C, SV, SPLIT, C, DK, NT, BF>(sPt, 1, CP, sX, SVP, 1, sKt, 1, CP, sS, SVP, 1,
                                    [&](int i, int j, float x) { sY[i * SVP + j] = -x; });
        __syncthreads();   // group A's buffers are free
        issue_a(step + 1);
        if (step + 1 < nch) load_x(step + 1);   // next chunk's V or dO, in flight during product B
        pend_b = false;
        if (!(ok = wait_copies(bar_b, ph_b))) break;   // group B of this chunk
        if (!backward)
            block_mma<DK, SV, SPLIT, C, 0, NT, BF>(sKt, CP, 1, sY, SVP, 1, nullptr, 0, 0, nullptr, 0, 0,
                                     [&](int c, int j, float x) { sS[c * SVP + j] = sD[c] * sS[c * SVP + j] + x; });
        else
            block_mma<DK, SV, SPLIT, C, C, NT, BF>(sQh, 1, DKP, sX, SVP, 1, sKh, 1, DKP, sY, SVP, 1,
                                     [&](int c, int j, float x) { sS[c * SVP + j] = sD[c] * sS[c * SVP + j] + x; });
        __syncthreads();   // group B's buffers are free
        issue_b(step + 1);
    }
    if (!ok) {   // a copy did not arrive: wait (bounded) for any still in flight, then leave
        if (pend_a) ptx::mbar_wait_bounded(bar_a, ph_a, kWaitLimit);
        if (pend_b) ptx::mbar_wait_bounded(bar_b, ph_b, kWaitLimit);
        return;
    }
    __syncthreads();
    if (backward && dinit_state) {
        for (int idx = tid; idx < DK * SV; idx += NT) {
            const int c = idx / SV, j = idx % SV;
            dinit_state[st_off + (long long)c * DV + j] = sS[c * SVP + j];
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
__global__ void __launch_bounds__(PartThreads<Tin>::value, 1)
bwd_part_kernel(const Tin *__restrict__ v, const float *__restrict__ beta, const Tin *__restrict__ d_o,
                Tin *__restrict__ dv_out, const int32_t *__restrict__ cu_seqlens, int T, int H, int DV,
                int num_seqs, const float *__restrict__ rec, const float *__restrict__ ckpt,
                const float *__restrict__ dckpt, float *__restrict__ part) {
    using L = PartSmem<DK>;
    using R = Rec<DK>;
    using P = Part<DK>;
    constexpr int DKP = L::DKP;
    constexpr bool SPLIT = sizeof(Tin) == 4;
    constexpr bool BF = sizeof(Tin) == 2;   // bf16 inputs: bf16 operands
    constexpr int NTH = PartThreads<Tin>::value, NW = NTH / 32;
    // Column sums accumulate in registers across the value tiles: each warp owns a
    // strip of one 16-row block by TQ (TA) adjacent 8-column tiles of the [C][DK]
    // ([C][C]) sums.
    constexpr int TQ = (C / 16) * (DK / 8) / NW;   // [C][DK] output tiles per warp
    constexpr int TA = (C / 16) * (C / 8) / NW;    // [C][C] output tiles per warp
    static_assert((DK / 8) % TQ == 0 && (C / 8) % TA == 0, "strips stay inside one row block");
    const int wq = (int)(threadIdx.x >> 5);
    const int q_r0 = (wq / ((DK / 8) / TQ)) * 16, q_c0 = (wq % ((DK / 8) / TQ)) * TQ * 8;
    const int a_r0 = (wq / ((C / 8) / TA)) * 16, a_c0 = (wq % ((C / 8) / TA)) * TA * 8;
    extern __shared__ __align__(128) float sm[];
    float *sKh = sm + L::kh, *sKb = sm + L::kb, *sAkk = sm + L::akk, *sAqk = sm + L::aqk, *sT = sm + L::ti;
    float *sTb = sm + L::tb, *sS = sm + L::S, *sdS = sm + L::dS, *sW = sm + L::w, *sU = sm + L::u;
    float *sDO = sm + L::dout, *sdU = sm + L::du, *sL = sm + L::lam, *sB = sm + L::b, *sDB = sm + L::db;
    const int tid = threadIdx.x, warp = tid >> 5, slot = blockIdx.x, h = blockIdx.y;
    long long cs;
    int Lc;
    if (!chunk_of_slot(cu_seqlens, T, num_seqs, slot, cs, Lc)) return;
    const float *rp = rec + ((long long)slot * H + h) * R::FLOATS;
    __shared__ __align__(8) uint64_t bar_rec;
    const uint32_t bar = ptx::smem_u32(&bar_rec);
    uint32_t ph = 0;
    if (tid == 0) {
        ptx::mbar_init(bar, 1);
        ptx::fence_mbar_init();
        ptx::mbar_arrive_expect_tx(bar, 2 * R::ROWS_K + 4 * R::ROWS_C);
        ptx::bulk_load(ptx::smem_u32(sKh), rp + R::KH, R::ROWS_K, bar);
        ptx::bulk_load(ptx::smem_u32(sKb), rp + R::KB, R::ROWS_K, bar);
        ptx::bulk_load(ptx::smem_u32(sAkk), rp + R::AKK, R::ROWS_C, bar);
        ptx::bulk_load(ptx::smem_u32(sAqk), rp + R::AQK, R::ROWS_C, bar);
        ptx::bulk_load(ptx::smem_u32(sT), rp + R::TI, R::ROWS_C, bar);
        ptx::bulk_load(ptx::smem_u32(sTb), rp + R::TB, R::ROWS_C, bar);
    }
    for (int i = tid; i < C; i += NTH) {
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
        async_rows(sS, TP, ckpt + st_base + col_base, DK, DVT, DV);
        async_rows(sdS, TP, dckpt + st_base + col_base, DK, DVT, DV);
        cp_async_commit();
        {
            constexpr int NV = C * DVT / 4 / NTH;   // 4-element vectors of V and dO per thread
            float4 rv[NV], rd[NV];
#pragma unroll
            for (int u = 0; u < NV; ++u) {
                const int e = (tid + u * NTH) * 4, i = e / DVT, j = e % DVT;
                rv[u] = rd[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (i < Lc) {
                    const long long off = ((cs + i) * H + h) * DV + col_base + j;
                    rv[u] = load4(v + off);
                    rd[u] = load4(d_o + off);
                }
            }
#pragma unroll
            for (int u = 0; u < NV; ++u) {
                const int e = (tid + u * NTH) * 4, i = e / DVT, j = e % DVT;
                *reinterpret_cast<float4 *>(sW + i * TP + j) = rv[u];
                *reinterpret_cast<float4 *>(sDO + i * TP + j) = rd[u];
            }
        }
        cp_async_wait_all();
        if (tile == 0 && !wait_copies(bar, ph)) {   // the record did not arrive: wait (bounded) once more, leave
            ptx::mbar_wait_bounded(bar, ph ^ 1u, kWaitLimit);
            return;
        }
        __syncthreads();
        // W = V - Kh S (in place: each element is read and written by its owner only)
        block_mma<C, DVT, SPLIT, DK, 0, NTH, BF>(sKh, DKP, 1, sS, TP, 1, nullptr, 0, 0, nullptr, 0, 0,
                                 [&](int i, int j, float x) { sW[i * TP + j] -= x; });
        __syncthreads();
        // U = Tb W;  dU = Aqk^T dO + Kb dS
        block_mma<C, DVT, SPLIT, C, 0, NTH, BF>(sTb, CP, 1, sW, TP, 1, nullptr, 0, 0, nullptr, 0, 0,
                                 [&](int i, int j, float x) { sU[i * TP + j] = x; });
        block_mma<C, DVT, SPLIT, C, DK, NTH, BF>(sAqk, 1, CP, sDO, TP, 1, sKb, DKP, 1, sdS, TP, 1,
                                 [&](int i, int j, float x) { sdU[i * TP + j] = x; });
        __syncthreads();
        // R = W - Akk U (in place of W);  lam = T^T dU
        block_mma<C, DVT, SPLIT, C, 0, NTH, BF>(sAkk, CP, 1, sU, TP, 1, nullptr, 0, 0, nullptr, 0, 0,
                                 [&](int i, int j, float x) { sW[i * TP + j] -= x; });
        block_mma<C, DVT, SPLIT, C, 0, NTH, BF>(sT, 1, CP, sdU, TP, 1, nullptr, 0, 0, nullptr, 0, 0,
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
        for (int idx = tid; idx < C * DVT; idx += NTH) {
            const int i = idx / DVT, j = idx % DVT;
            const float mu = sB[i] * sL[i * TP + j];
            sL[i * TP + j] = mu;
            if (i < Lc) Elem<Tin>::store(dv_out + ((cs + i) * H + h) * DV + col_base + j, mu);
        }
        __syncthreads();
        // sums over this tile's columns, kept in registers across tiles:
        // dO S^T, mu S^T, U dS^T ([C][DK]) and dO U^T, mu U^T ([C][C])
        if constexpr (BF) {
            warp_mma_strip_bf16<DVT, TQ>(a_dq, sDO + q_r0 * TP, TP, 1, sS + q_c0 * TP, 1, TP);
            warp_mma_strip_bf16<DVT, TQ>(a_dkh, sL + q_r0 * TP, TP, 1, sS + q_c0 * TP, 1, TP);
            warp_mma_strip_bf16<DVT, TQ>(a_dkb, sU + q_r0 * TP, TP, 1, sdS + q_c0 * TP, 1, TP);
            warp_mma_strip_bf16<DVT, TA>(a_aq, sDO + a_r0 * TP, TP, 1, sU + a_c0 * TP, 1, TP);
            warp_mma_strip_bf16<DVT, TA>(a_ak, sL + a_r0 * TP, TP, 1, sU + a_c0 * TP, 1, TP);
        } else {
            warp_mma_strip<SPLIT, DVT, TQ>(a_dq, sDO + q_r0 * TP, TP, 1, sS + q_c0 * TP, 1, TP);
            warp_mma_strip<SPLIT, DVT, TQ>(a_dkh, sL + q_r0 * TP, TP, 1, sS + q_c0 * TP, 1, TP);
            warp_mma_strip<SPLIT, DVT, TQ>(a_dkb, sU + q_r0 * TP, TP, 1, sdS + q_c0 * TP, 1, TP);
            warp_mma_strip<SPLIT, DVT, TA>(a_aq, sDO + a_r0 * TP, TP, 1, sU + a_c0 * TP, 1, TP);
            warp_mma_strip<SPLIT, DVT, TA>(a_ak, sL + a_r0 * TP, TP, 1, sU + a_c0 * TP, 1, TP);
        }
        if (tid < DK)
            for (int j = 0; j < DVT; ++j) a_gc = fmaf(sS[tid * TP + j], sdS[tid * TP + j], a_gc);
    }
    float *pp = part + ((long long)slot * H + h) * P::FLOATS;
    {
        const int lane = tid & 31, g = lane >> 2, t = lane & 3;
        auto put = [&](float *base, int ld, const float (&d)[4], int r0, int c0, float sgn) {
            *reinterpret_cast<float2 *>(base + (r0 + g) * ld + c0 + 2 * t) = make_float2(sgn * d[0], sgn * d[1]);
            *reinterpret_cast<float2 *>(base + (r0 + g + 8) * ld + c0 + 2 * t) = make_float2(sgn * d[2], sgn * d[3]);
        };
#pragma unroll
        for (int r = 0; r < TQ; ++r) {
            const int r0 = q_r0, c0 = q_c0 + 8 * r;
            put(pp + P::DQ, DK, a_dq[r], r0, c0, 1.f);
            put(pp + P::DKH, DK, a_dkh[r], r0, c0, -1.f);
            put(pp + P::DKB, DK, a_dkb[r], r0, c0, 1.f);
        }
#pragma unroll
        for (int r = 0; r < TA; ++r) {
            const int r0 = a_r0, c0 = a_c0 + 8 * r;
            // keep j <= i of dAqk and j < i of dAkk; zero the rest
            float aq[4], ak[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = r0 + g + (e >> 1) * 8, j = c0 + 2 * t + (e & 1);
                aq[e] = j <= i ? a_aq[r][e] : 0.f;
                ak[e] = j < i ? -a_ak[r][e] : 0.f;
            }
            put(pp + P::AQK, C, aq, r0, c0, 1.f);
            put(pp + P::AKK, C, ak, r0, c0, 1.f);
        }
    }
    __syncthreads();
    for (int i = tid; i < C; i += NTH) pp[P::DB + i] = sDB[i];
    if (tid < DK) pp[P::DGC + tid] = a_gc;
}

// ------------------------------------------------------------------ decay-factor chain rule

template <int DK>
struct ChunkSmem {
    static constexpr int DKP = Pad<DK>::K;
    static constexpr int q = 0;                  // [C][DKP]
    static constexpr int k = q + C * DKP;        // [C][DKP]
    static constexpr int g = k + C * DKP;        // [C][DKP] G
    static constexpr int acc = g + C * DKP;      // [C][DKP] dq, then dk
    static constexpr int dg = acc + C * DKP;     // [C][DKP] dG
    static constexpr int aq = dg + C * DKP;      // [C][CP]  dAqk (lower with the diagonal)
    static constexpr int ak = aq + C * CP;       // [C][CP]  dAkk (strictly lower)
    static constexpr int scr = ak + C * CP;      // [SCR_ROWS][DKP] decay-scaled operand
    static constexpr int total = scr + SCR_ROWS * DKP;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

// Pair terms of the diagonal 16 x 16 blocks, exact, one thread per (channel,
// block): rows  acc_i += sum_{j<=i} A1[i][j] k_j E_ij (+ k_i times that into dG
// when rows_to_dg), and with A2 (dk phase) the column terms
// acc_j += sum_{i>=j} (A1[i][j] q_i + [i>j] A2[i][j] k_i) E_ij, dG_j -= k_j (that),
// plus the row terms of A2.  Q phase: A1 = dAqk, no A2.  K phase: A1 = dAqk
// (columns only), A2 = dAkk (rows and columns).
template <int DK, bool KPHASE, int NTH>
__device__ __forceinline__ void diag_pair_terms(const float *sQ, const float *sK, const float *sG, const float *sAq,
                                                const float *sAk, float *sAcc, float *sDg) {
    constexpr int DKP = Pad<DK>::K;
    constexpr int NG = NTH / DK;   // thread groups per channel
    const int c = threadIdx.x % DK, grp = threadIdx.x / DK;
    for (int b = grp; b < NSB; b += NG) {
        const int r = b * SB;
        float colacc[SB];
#pragma unroll
        for (int jj = 0; jj < SB; ++jj) colacc[jj] = 0.f;
#pragma unroll
        for (int ii = 0; ii < SB; ++ii) {
            const int i = r + ii;
            const float gi = sG[i * DKP + c], qi = sQ[i * DKP + c], ki = sK[i * DKP + c];
            float row = 0.f;
#pragma unroll
            for (int jj = 0; jj <= ii; ++jj) {
                const int j = r + jj;
                const float e = __expf(gi - sG[j * DKP + c]);
                if (!KPHASE) {
                    row = fmaf(sAq[i * CP + j], sK[j * DKP + c] * e, row);
                } else {
                    const float akk = jj < ii ? sAk[i * CP + j] : 0.f;
                    row = fmaf(akk, sK[j * DKP + c] * e, row);
                    colacc[jj] = fmaf(fmaf(sAq[i * CP + j], qi, akk * ki), e, colacc[jj]);
                }
            }
            sAcc[i * DKP + c] += row;
            if (KPHASE) sDg[i * DKP + c] += ki * row;
        }
        if (KPHASE) {
#pragma unroll
            for (int jj = 0; jj < SB; ++jj) {
                const int j = r + jj;
                sAcc[j * DKP + c] += colacc[jj];
                sDg[j * DKP + c] -= sK[j * DKP + c] * colacc[jj];
            }
        }
    }
}

// Row terms of block bi (rows r..r+15, r = 16 bi) over columns j in [J0, J1), J1 <= r:
// acc_i += e^{G_i - G_r} sum_j A[i][j] (k_j e^{G_r - G_j}); dG_i += k_i (that) when
// to_dg.  Both factors are <= 1.
template <int DK, bool SPLIT, int NTH, int BI, int J0, int J1>
__device__ __forceinline__ void row_terms(const float *sK, const float *sG, const float *sA, float *scr,
                                          float *sAcc, float *sDg, bool to_dg) {
    constexpr int DKP = Pad<DK>::K, r = BI * SB, n = J1 - J0;
    static_assert(n > 0 && n <= SCR_ROWS, "operand fits the scratch");
    __syncthreads();
    for (int idx = threadIdx.x; idx < n * DK; idx += NTH) {
        const int jj = idx / DK, c = idx % DK, j = J0 + jj;
        scr[jj * DKP + c] = sK[j * DKP + c] * __expf(sG[r * DKP + c] - sG[j * DKP + c]);
    }
    __syncthreads();
    block_mma<SB, DK, SPLIT, n, 0, NTH>(sA + r * CP + J0, CP, 1, scr, DKP, 1, nullptr, 0, 0, nullptr, 0, 0,
                                [&](int ii, int c, float x) {
                                    const int i = r + ii;
                                    x *= __expf(sG[i * DKP + c] - sG[r * DKP + c]);
                                    sAcc[i * DKP + c] += x;
                                    if (to_dg) sDg[i * DKP + c] += sK[i * DKP + c] * x;
                                });
}

// Row terms of the blocks below the diagonal.
template <int DK, bool SPLIT, int NTH>
__device__ __forceinline__ void pair_rows(const float *sK, const float *sG, const float *sA, float *scr, float *sAcc,
                                          float *sDg, bool to_dg) {
    static_assert(NSB == 4 && SCR_ROWS == 48, "four 16-row blocks");
    row_terms<DK, SPLIT, NTH, 1, 0, 16>(sK, sG, sA, scr, sAcc, sDg, to_dg);
    row_terms<DK, SPLIT, NTH, 2, 0, 32>(sK, sG, sA, scr, sAcc, sDg, to_dg);
    row_terms<DK, SPLIT, NTH, 3, 0, 48>(sK, sG, sA, scr, sAcc, sDg, to_dg);
    __syncthreads();
}

// Column terms of block bj (columns 16 bj..16 bj+15, last row s) over rows i in
// [I0, I1), I0 > s: acc_j += e^{G_s - G_j} sum_i A[i][j] (X_i e^{G_i - G_s}),
// dG_j -= k_j (that), for (A, X) = (dAqk, q) and (dAkk, k).  Both factors are <= 1.
template <int DK, bool SPLIT, int NTH, int BJ, int I0, int I1>
__device__ __forceinline__ void col_terms(const float *sQ, const float *sK, const float *sG, const float *sAq,
                                          const float *sAk, float *scr, float *sAcc, float *sDg) {
    constexpr int DKP = Pad<DK>::K, s = BJ * SB + SB - 1, n = I1 - I0;
    static_assert(n > 0 && n <= SCR_ROWS, "operand fits the scratch");
    for (int pass = 0; pass < 2; ++pass) {
        const float *X = pass ? sK : sQ;
        const float *A = pass ? sAk : sAq;
        __syncthreads();
        for (int idx = threadIdx.x; idx < n * DK; idx += NTH) {
            const int ii = idx / DK, c = idx % DK, i = I0 + ii;
            scr[ii * DKP + c] = X[i * DKP + c] * __expf(sG[i * DKP + c] - sG[s * DKP + c]);
        }
        __syncthreads();
        block_mma<SB, DK, SPLIT, n, 0, NTH>(A + I0 * CP + BJ * SB, 1, CP, scr, DKP, 1, nullptr, 0, 0, nullptr, 0, 0,
                                    [&](int jj, int c, float x) {
                                        const int j = BJ * SB + jj;
                                        x *= __expf(sG[s * DKP + c] - sG[j * DKP + c]);
                                        sAcc[j * DKP + c] += x;
                                        sDg[j * DKP + c] -= sK[j * DKP + c] * x;
                                    });
    }
}

// Column terms of the blocks below the diagonal.
template <int DK, bool SPLIT, int NTH>
__device__ __forceinline__ void pair_cols(const float *sQ, const float *sK, const float *sG, const float *sAq,
                                          const float *sAk, float *scr, float *sAcc, float *sDg) {
    col_terms<DK, SPLIT, NTH, 0, 16, 64>(sQ, sK, sG, sAq, sAk, scr, sAcc, sDg);
    col_terms<DK, SPLIT, NTH, 1, 32, 64>(sQ, sK, sG, sAq, sAk, scr, sAcc, sDg);
    col_terms<DK, SPLIT, NTH, 2, 48, 64>(sQ, sK, sG, sAq, sAk, scr, sAcc, sDg);
    __syncthreads();
}

// GS: scalar gate (Gated DeltaNet) -- log_alpha and dlog_alpha are [tokens, H];
// the gradient of a rate broadcast over the channels is the sum over them.
template <int DK, typename Tin, bool GS>
__global__ void __launch_bounds__(CHUNK_NT, 1)
bwd_chunk_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const float *__restrict__ log_alpha,
                 const float *__restrict__ beta, const int32_t *__restrict__ cu_seqlens, int T, int H, int num_seqs,
                 const float *__restrict__ part, Tin *__restrict__ dq, Tin *__restrict__ dk_out,
                 float *__restrict__ dlog_alpha, float *__restrict__ dbeta) {
    using L = ChunkSmem<DK>;
    using P = Part<DK>;
    constexpr int DKP = L::DKP;
    constexpr bool SPLIT = sizeof(Tin) == 4;
    constexpr int NTH = CHUNK_NT;
    extern __shared__ __align__(128) float sm[];
    float *sQ = sm + L::q, *sK = sm + L::k, *sG = sm + L::g, *sAcc = sm + L::acc, *sDg = sm + L::dg;
    float *sAq = sm + L::aq, *sAk = sm + L::ak, *scr = sm + L::scr;
    const int tid = threadIdx.x, slot = blockIdx.x, h = blockIdx.y;
    long long cs;
    int Lc;
    if (!chunk_of_slot(cu_seqlens, T, num_seqs, slot, cs, Lc)) return;
    const float *pp = part + ((long long)slot * H + h) * P::FLOATS;
    constexpr int NV = C * DK / 4 / NTH;   // 4-element vectors per thread
    // dAqk (zero above the diagonal) and dAkk (zero on and above it) by async copy
    async_rows(sAq, CP, pp + P::AQK, C, C);
    async_rows(sAk, CP, pp + P::AKK, C, C);
    cp_async_commit();
    for (int i = tid; i < Lc; i += NTH) dbeta[(cs + i) * H + h] = pp[P::DB + i];
    load_chunk_qkg<DK, Tin, NTH, GS>(q, k, log_alpha, nullptr, cs, Lc, H, h, sQ, sK, sG, nullptr);

    // ---- dq = e^G dQh + pair terms of dAqk;  dG = q dq
    {
        float4 r[NV];
#pragma unroll
        for (int u = 0; u < NV; ++u) r[u] = *reinterpret_cast<const float4 *>(pp + P::DQ + (tid + u * NTH) * 4);
#pragma unroll
        for (int u = 0; u < NV; ++u) {
            const int e = (tid + u * NTH) * 4, i = e / DK, c = e % DK;
            const float *g = sG + i * DKP + c;
            *reinterpret_cast<float4 *>(sAcc + i * DKP + c) =
                make_float4(__expf(g[0]) * r[u].x, __expf(g[1]) * r[u].y, __expf(g[2]) * r[u].z, __expf(g[3]) * r[u].w);
        }
    }
    cp_async_wait_all();
    __syncthreads();
    // The diagonal blocks stay exact on CUDA cores here: taking them through the
    // block boundary costs two more scaled operands per phase, which measured slower.
    diag_pair_terms<DK, false, NTH>(sQ, sK, sG, sAq, nullptr, sAcc, nullptr);
    pair_rows<DK, SPLIT, NTH>(sK, sG, sAq, scr, sAcc, nullptr, false);
    // dq out; dk starts at a + b and dG at q dq + k (a - b); sum_i k_i b_i per
    // channel (a dG_C term) goes to scr, one row per group of rows
    {
        float4 ra[NV], rb[NV];
#pragma unroll
        for (int u = 0; u < NV; ++u) {
            ra[u] = *reinterpret_cast<const float4 *>(pp + P::DKH + (tid + u * NTH) * 4);
            rb[u] = *reinterpret_cast<const float4 *>(pp + P::DKB + (tid + u * NTH) * 4);
        }
        float kb[4] = {0.f, 0.f, 0.f, 0.f};
        const int c = (tid * 4) % DK;   // the same 4 channels for every u (NTH * 4 is a multiple of DK)
#pragma unroll
        for (int u = 0; u < NV; ++u) {
            const int e = (tid + u * NTH) * 4, i = e / DK;
            const float ha[4] = {ra[u].x, ra[u].y, ra[u].z, ra[u].w}, hb[4] = {rb[u].x, rb[u].y, rb[u].z, rb[u].w};
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int o = i * DKP + c + v;
                const float x = sAcc[o];
                if (i < Lc) Elem<Tin>::store(dq + ((cs + i) * H + h) * DK + c + v, x);
                const float gi = sG[o], gC = sG[(C - 1) * DKP + c + v];
                const float a = __expf(gi) * ha[v], b = __expf(gC - gi) * hb[v];
                const float kk = sK[o];
                sDg[o] = sQ[o] * x + kk * (a - b);
                sAcc[o] = a + b;
                kb[v] = fmaf(kk, b, kb[v]);
            }
        }
#pragma unroll
        for (int v = 0; v < 4; ++v) scr[((tid * 4) / DK) * DKP + c + v] = kb[v];
    }
    __syncthreads();
    float kb_sum = 0.f;   // this thread's channel (tid < DK) of sum_i k_i b_i
    if (tid < DK)
        for (int gq = 0; gq < NTH * 4 / DK; ++gq) kb_sum += scr[gq * DKP + tid];
    __syncthreads();
    // ---- dk = a + b + pair terms of dAkk (rows) and of dAqk, dAkk (columns)
    diag_pair_terms<DK, true, NTH>(sQ, sK, sG, sAq, sAk, sAcc, sDg);
    pair_rows<DK, SPLIT, NTH>(sK, sG, sAk, scr, sAcc, sDg, true);
    pair_cols<DK, SPLIT, NTH>(sQ, sK, sG, sAq, sAk, scr, sAcc, sDg);
    for (int idx = tid; idx < C * DK; idx += NTH) {
        const int i = idx / DK, c = idx % DK;
        if (i < Lc) Elem<Tin>::store(dk_out + ((cs + i) * H + h) * DK + c, sAcc[i * DKP + c]);
    }
    // ---- dG_C terms, then dlog_alpha_s = sum_{i>=s} dG_i
    for (int c = tid; c < DK; c += NTH) {
        const float gC = sG[(C - 1) * DKP + c];
        float acc = __expf(gC) * pp[P::DGC + c] + kb_sum;
        for (int i = C - 1; i >= 0; --i) {
            acc += sDg[i * DKP + c];
            if constexpr (GS) sDg[i * DKP + c] = acc;
            else if (i < Lc) dlog_alpha[((cs + i) * H + h) * DK + c] = acc;
        }
    }
    if constexpr (GS) {   // dlog_alpha of the shared rate: the sum over the channels, one warp per row
        __syncthreads();
        const int warp = tid >> 5, lane = tid & 31;
        for (int i = warp; i < Lc; i += NTH / 32) {
            float x = 0.f;
            for (int c = lane; c < DK; c += 32) x += sDg[i * DKP + c];
            for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
            if (lane == 0) dlog_alpha[(cs + i) * H + h] = x;
        }
    }
}

}  // namespace bwd
}  // namespace kda
