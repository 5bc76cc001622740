// KDA chunked prefill on sm_100a tensor cores (tcgen05 MMA, fp32 accumulation in TMEM).
//
// Method: the KDA recurrence ("Kimi Delta Attention 徹底解説" (tech-tide.dev),
// § "Kimi Delta Attention の仕組み") regrouped into 64-token chunks; the per-token
// transition (I - beta k k^T) Diag(alpha) is diagonal plus rank one, so a chunk of
// them collapses into a few dense products ("Kimi Linear、独自の土俵でFull
// Attentionを上回る" (remio.ai), § "Kimi Linearがより賢いRecurrent Memoryを使う方法":
// chunkwise algorithm on a diagonal-plus-low-rank transition).
//
// For a chunk starting from state S (dk x dv), G_i = sum_{s<=i} log_alpha_s per channel:
//   Khat = e^G * K, Qhat = e^G * Q, Rk = e^{-G} * K, Kbar = e^{G_last - G} * K
//   Akk = strict_lower(Khat Rk^T), Aqk = lower(Qhat Rk^T)          (Gram, one MMA)
//   X = Khat S, Y = Qhat S                                          (one MMA, state-dependent)
//   T = (I + Diag(beta) Akk)^{-1},  Tb = T Diag(beta)               (fp32, shared memory)
//   Kt = Kbar^T Tb,  Pt = Aqk Tb                                    (one MMA pair)
//   Z = V - X
//   S <- Diag(e^{G_last}) S + Kt Z,   O = Y + Pt Z                   (one MMA pair)
// The e^{-G} factor bounds the usable range: a channel's log-decay summed over one
// chunk must stay >= -80 (checked; KDA_DEV_DECAY_RANGE otherwise).
//
// Mapping: one 128-thread CTA per (value-column tile of DVT, head, sequence) walks
// the sequence's chunks in order.  Thread c owns key channel c (the per-channel
// cumulative decay) and row c of the fp32 state (registers), which is also TMEM
// lane c of every 128-row accumulator.  Thread 0 issues the MMAs; their completion
// is signalled through one mbarrier with bounded waits.  bf16 operands live in
// shared memory in the 128-byte-swizzled K-major layout the MMA descriptors name.
#pragma once

#include <cstdio>

#include "kda_common.cuh"
#include "tc_ptx.cuh"

namespace kda {
namespace tc {

constexpr int C = 64;
constexpr int NT = 128;
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;   // 1 s: far beyond any legitimate MMA latency
constexpr uint32_t TMEM_COLS = 256;
// TMEM column map (fp32 accumulators, lane = row)
constexpr uint32_t COL_GRAM = 0;    // [128 x 64]  rows 0-63 Khat Rk^T, rows 64-127 Qhat Rk^T
constexpr uint32_t COL_XY = 64;     // [128 x DVT] rows 0-63 X, rows 64-127 Y (then O)
constexpr uint32_t COL_KT = 128;    // [128 x 64]  Kt (and Pt rows 64-127 when dk = 64)
constexpr uint32_t COL_PT = 192;    // [128 x 64]  rows 64-127 Pt (dk = 128)
constexpr uint32_t COL_DS = 0;      // [128 x DVT] Kt Z (reuses the Gram columns)

template <int DK, int DVT>
struct Layout {
    static constexpr int KA = DK / 64;                       // 64-element K atoms along dk
    static constexpr int KQ = 0;                             // [KA][128][128 B] Khat (0-63), Qhat (64-127)
    static constexpr int RK = KQ + KA * 128 * 128;           // [KA][64][128 B]  Rk
    static constexpr int SB = RK + KA * 64 * 128;            // [KA][DVT][128 B] S^T (bf16): B operand
    static constexpr int KP = SB + KA * DVT * 128;           // [DK+64][128 B]   Kbar^T -> Kt ; Aqk -> Pt
    static constexpr int TB = KP + (DK + 64) * 128;          // [64][128 B]      Tb^T
    static constexpr int ZT = TB + 64 * 128;                 // [DVT][128 B]     Z^T
    static constexpr int FA = ZT + DVT * 128;                // fp32 [64][65]    Diag(beta) Akk
    static constexpr int FT = FA + 64 * 65 * 4;              // fp32 [64][65]    T
    static constexpr int FM = FT + 64 * 65 * 4;              // fp32 [32][33]    block-product scratch
    static constexpr int FB = FM + 32 * 33 * 4;              // fp32 [64]        beta
    static constexpr int MISC = FB + 64 * 4;                 // mbarrier, TMEM base
    static constexpr int BYTES = MISC + 64;
    static constexpr int ALLOC = BYTES + 1024;               // room to align the base to 1024 B
    static_assert(KQ % 1024 == 0 && RK % 1024 == 0 && SB % 1024 == 0 && KP % 1024 == 0 &&
                      TB % 1024 == 0 && ZT % 1024 == 0,
                  "swizzled tiles must be 1024-byte aligned");
};

// Byte offset of bf16 element (row, k) in a K-major, 128-byte-swizzled tile whose
// K atoms (64 elements each) hold `rows` rows.
__device__ __forceinline__ uint32_t sw128(int row, int k, int rows) {
    const int atom = k >> 6, kk = k & 63;
    return (uint32_t)(atom * rows * 128 + row * 128 + ((((kk >> 3) ^ (row & 7))) << 4) + ((kk & 7) << 1));
}

__device__ __forceinline__ void st_bf16(uint8_t *base, uint32_t off, float x) {
    *reinterpret_cast<__nv_bfloat16 *>(base + off) = __float2bfloat16_rn(x);
}

// Descriptor of the 16-wide K step `s` of a swizzled tile at `addr` with `rows`
// rows per K atom, starting at row r0 (a multiple of 8).
__device__ __forceinline__ uint64_t kdesc(uint32_t addr, int s, int rows, int r0 = 0) {
    return ptx::desc_kmajor_sw128(addr + (uint32_t)((s >> 2) * rows * 128 + r0 * 128 + (s & 3) * 32));
}

// T = (I + A)^{-1} for a 64 x 64 strictly lower A (fp32, row stride 65): the four
// 16 x 16 diagonal blocks by forward substitution, then the block-triangular
// inverse [L11 0; L21 L22]^{-1} = [L11^-1 0; -L22^-1 L21 L11^-1  L22^-1] at 32 and 64.
// Only the lower triangle of T is written.  All 128 threads take part.
__device__ __forceinline__ void invert_unit_lower64(const float *A, float *Tm, float *M, int tid) {
    if (tid < 64) {
        const int o = 16 * (tid >> 4), l = tid & 15;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < i; ++j) acc = fmaf(A[(o + i) * 65 + o + j], x[j], acc);
            x[i] = (i < l) ? 0.f : ((i == l) ? 1.f : -acc);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (i >= l) Tm[(o + i) * 65 + o + l] = x[i];
    }
    __syncthreads();
    // 32-blocks: T[2p+1][2p] = -T[2p+1][2p+1] A[2p+1][2p] T[2p][2p]
#pragma unroll 1
    for (int m = 0; m < 4; ++m) {
        const int oi = tid + 128 * m, p = oi >> 8, r = (oi >> 4) & 15, c = oi & 15;
        const int ro = 32 * p + 16, co = 32 * p;
        float acc = 0.f;
        for (int j = c; j < 16; ++j) acc = fmaf(A[(ro + r) * 65 + co + j], Tm[(co + j) * 65 + co + c], acc);
        M[p * 272 + r * 17 + c] = acc;
    }
    __syncthreads();
#pragma unroll 1
    for (int m = 0; m < 4; ++m) {
        const int oi = tid + 128 * m, p = oi >> 8, r = (oi >> 4) & 15, c = oi & 15;
        const int ro = 32 * p + 16, co = 32 * p;
        float acc = 0.f;
        for (int j = 0; j <= r; ++j) acc = fmaf(Tm[(ro + r) * 65 + ro + j], M[p * 272 + j * 17 + c], acc);
        Tm[(ro + r) * 65 + co + c] = -acc;
    }
    __syncthreads();
    // 64: T[hi][lo] = -T[hi][hi] A[hi][lo] T[lo][lo]
#pragma unroll 1
    for (int m = 0; m < 8; ++m) {
        const int oi = tid + 128 * m, r = oi >> 5, c = oi & 31;
        float acc = 0.f;
        for (int j = c; j < 32; ++j) acc = fmaf(A[(32 + r) * 65 + j], Tm[j * 65 + c], acc);
        M[r * 33 + c] = acc;
    }
    __syncthreads();
#pragma unroll 1
    for (int m = 0; m < 8; ++m) {
        const int oi = tid + 128 * m, r = oi >> 5, c = oi & 31;
        float acc = 0.f;
        for (int j = 0; j <= r; ++j) acc = fmaf(Tm[(32 + r) * 65 + 32 + j], M[j * 33 + c], acc);
        Tm[(32 + r) * 65 + c] = -acc;
    }
    __syncthreads();
}

// Every thread waits for the next completion of the CTA's MMA barrier; all agree
// on the outcome.  Returns false (and flags the device status) on timeout.
__device__ __forceinline__ bool wait_mma(uint32_t mbar, uint32_t &phase) {
    const bool ok = ptx::mbar_wait_bounded(mbar, phase, WAIT_LIMIT_NS);
    phase ^= 1u;
    const bool any_fail = __syncthreads_or(!ok);
    if (any_fail) {
        if (threadIdx.x == 0) flag_status(KDA_DEV_WAIT_TIMEOUT);
        return false;
    }
    ptx::tc_fence_after();
    return true;
}

__device__ __forceinline__ void load16_bf16(const __nv_bfloat16 *p, float (&x)[16]) {
    const uint4 a = reinterpret_cast<const uint4 *>(p)[0];
    const uint4 b = reinterpret_cast<const uint4 *>(p)[1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}

__device__ __forceinline__ void store16_bf16(__nv_bfloat16 *p, const float (&x)[16]) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        __nv_bfloat162 h2 = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t *>(&h2);
    }
    reinterpret_cast<uint4 *>(p)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4 *>(p)[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

template <int DK, int DVT>
__global__ void __launch_bounds__(NT, 1)
chunk_tc_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                const __nv_bfloat16 *__restrict__ v, const float *__restrict__ log_alpha,
                const float *__restrict__ beta, const float *__restrict__ init_state,
                __nv_bfloat16 *__restrict__ o, float *__restrict__ final_state,
                const int32_t *__restrict__ cu_seqlens, int T, int H, int DV) {
    using L = Layout<DK, DVT>;
    static_assert(DVT % 16 == 0 && DVT >= 16 && DVT <= 64, "value tile");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = ptx::smem_u32(sm);
    float *fA = reinterpret_cast<float *>(sm + L::FA);
    float *fT = reinterpret_cast<float *>(sm + L::FT);
    float *fM = reinterpret_cast<float *>(sm + L::FM);
    float *fB = reinterpret_cast<float *>(sm + L::FB);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::MISC + 8);
    const uint32_t mbar = sb + L::MISC;

    const int tid = threadIdx.x, warp = tid >> 5;
    const int col_base = blockIdx.x * DVT, h = blockIdx.y, n = blockIdx.z;

    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), TMEM_COLS);
        ptx::tmem_relinquish();
    }
    if (tid == 0) {
        ptx::mbar_init(mbar, 1);
        ptx::fence_mbar_init();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);   // this warp's TMEM lane quadrant
    uint32_t phase = 0;

    long long t0, t1;
    seq_span(cu_seqlens, T, n, t0, t1);
    const long long st_off = ((long long)n * H + h) * DK * DV + col_base;
    const bool has_row = tid < DK;

    float S[DVT];
#pragma unroll
    for (int j = 0; j < DVT; j += 4) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (has_row && init_state) x = load4(init_state + st_off + (long long)tid * DV + j);
        S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
    }

    bool ok = true;
    for (long long cs = t0; cs < t1; cs += C) {
        const int Lc = (int)min((long long)C, t1 - cs);
        float dch = 1.f;   // e^{G_last} of this thread's channel

        // ---- 1. per-channel decay factors -> bf16 operand tiles; state -> bf16 B operand
        if (has_row) {
            const int c = tid;
            float gsum = 0.f;
            for (int i = 0; i < Lc; ++i) gsum += log_alpha[((cs + i) * H + h) * DK + c];
            if (gsum < -80.f) flag_status(KDA_DEV_DECAY_RANGE);
            dch = expf(gsum);
            float G = 0.f;
            for (int i = 0; i < C; ++i) {
                float qi = 0.f, ki = 0.f, gi = 0.f;
                if (i < Lc) {
                    const long long off = ((cs + i) * H + h) * DK + c;
                    qi = __bfloat162float(q[off]);
                    ki = __bfloat162float(k[off]);
                    gi = log_alpha[off];
                }
                G += gi;
                const float e = __expf(G), er = __expf(-G), eb = __expf(gsum - G);
                st_bf16(sm, L::KQ + sw128(i, c, 128), ki * e);
                st_bf16(sm, L::KQ + sw128(64 + i, c, 128), qi * e);
                st_bf16(sm, L::RK + sw128(i, c, 64), ki * er);
                st_bf16(sm, L::KP + sw128(c, i, DK + 64), ki * eb);
            }
#pragma unroll
            for (int j = 0; j < DVT; ++j) st_bf16(sm, L::SB + sw128(j, c, DVT), S[j]);
        }
        if (tid < C) fB[tid] = tid < Lc ? beta[(cs + tid) * H + h] : 0.f;
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();

        // ---- 2. Gram [Khat; Qhat] Rk^T and [X; Y] = [Khat; Qhat] S
        if (tid == 0) {
            ptx::tc_fence_after();
            constexpr uint32_t ig = ptx::idesc_bf16_f32(128, 64), ix = ptx::idesc_bf16_f32(128, DVT);
#pragma unroll
            for (int s = 0; s < DK / 16; ++s)
                ptx::mma_bf16(tmem + COL_GRAM, kdesc(sb + L::KQ, s, 128), kdesc(sb + L::RK, s, 64), ig, s > 0);
#pragma unroll
            for (int s = 0; s < DK / 16; ++s)
                ptx::mma_bf16(tmem + COL_XY, kdesc(sb + L::KQ, s, 128), kdesc(sb + L::SB, s, DVT), ix, s > 0);
            ptx::mma_commit(mbar);
        }
        if (!(ok = wait_mma(mbar, phase))) break;

        // ---- 3. Gram -> Diag(beta) Akk (fp32) and masked Aqk (bf16); UT transform T
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
            float g16[16];
            ptx::tmem_ld16(tl + COL_GRAM + cc * 16, g16);
            ptx::tmem_wait_ld();
            if (tid < 64) {
                const int i = tid;
                const float bi = fB[i];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int j = cc * 16 + u;
                    fA[i * 65 + j] = (j < i) ? bi * g16[u] : 0.f;
                }
            } else {
                const int i = tid - 64;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int j = cc * 16 + u;
                    st_bf16(sm, L::KP + sw128(DK + i, j, DK + 64), (j <= i) ? g16[u] : 0.f);
                }
            }
        }
        __syncthreads();
        invert_unit_lower64(fA, fT, fM, tid);
        {
            const int j = tid & 63, half = tid >> 6;
            const float bj = fB[j];
#pragma unroll 8
            for (int u = 0; u < 32; ++u) {
                const int l = half * 32 + u;
                st_bf16(sm, L::TB + sw128(j, l, 64), (l >= j) ? fT[l * 65 + j] * bj : 0.f);
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();

        // ---- 4. Kt = Kbar^T Tb, Pt = Aqk Tb
        if (tid == 0) {
            ptx::tc_fence_after();
            constexpr uint32_t ik = ptx::idesc_bf16_f32(128, 64);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                ptx::mma_bf16(tmem + COL_KT, kdesc(sb + L::KP, s, DK + 64), kdesc(sb + L::TB, s, 64), ik, s > 0);
            if (DK == 128) {
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    ptx::mma_bf16(tmem + COL_PT, kdesc(sb + L::KP, s, DK + 64, 64), kdesc(sb + L::TB, s, 64), ik,
                                  s > 0);
            }
            ptx::mma_commit(mbar);
        }
        if (!(ok = wait_mma(mbar, phase))) break;

        // ---- 5. Z = V - X (rows 0-63) -> Z^T operand; Kt, Pt -> bf16 operands
        if (tid < 64) {
            const int j = tid;
#pragma unroll 1
            for (int cc = 0; cc < DVT / 16; ++cc) {
                float x16[16], v16[16];
                ptx::tmem_ld16(tl + COL_XY + cc * 16, x16);
                if (j < Lc)
                    load16_bf16(v + ((cs + j) * H + h) * DV + col_base + cc * 16, v16);
                else
#pragma unroll
                    for (int u = 0; u < 16; ++u) v16[u] = 0.f;
                ptx::tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 16; ++u) st_bf16(sm, L::ZT + sw128(cc * 16 + u, j, DVT), v16[u] - x16[u]);
            }
        }
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
            float k16[16];
            ptx::tmem_ld16(tl + COL_KT + cc * 16, k16);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 16; ++u) st_bf16(sm, L::KP + sw128(tid, cc * 16 + u, DK + 64), k16[u]);
        }
        if (DK == 128 && tid >= 64) {
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                float p16[16];
                ptx::tmem_ld16(tl + COL_PT + cc * 16, p16);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 16; ++u) st_bf16(sm, L::KP + sw128(DK + tid - 64, cc * 16 + u, DK + 64), p16[u]);
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();

        // ---- 6. dS = Kt Z ; O = Y + Pt Z
        if (tid == 0) {
            ptx::tc_fence_after();
            constexpr uint32_t iz = ptx::idesc_bf16_f32(128, DVT);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                ptx::mma_bf16(tmem + COL_DS, kdesc(sb + L::KP, s, DK + 64), kdesc(sb + L::ZT, s, DVT), iz, s > 0);
            if (DK == 128) {
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    ptx::mma_bf16(tmem + COL_XY, kdesc(sb + L::KP, s, DK + 64, 64), kdesc(sb + L::ZT, s, DVT), iz, 1);
            }
            ptx::mma_commit(mbar);
        }
        if (!(ok = wait_mma(mbar, phase))) break;

        // ---- 7. S <- Diag(e^{G_last}) S + dS ; store O rows
#pragma unroll
        for (int cc = 0; cc < DVT / 16; ++cc) {
            float d16[16];
            ptx::tmem_ld16(tl + COL_DS + cc * 16, d16);
            ptx::tmem_wait_ld();
            if (has_row) {
#pragma unroll
                for (int u = 0; u < 16; ++u) S[cc * 16 + u] = fmaf(dch, S[cc * 16 + u], d16[u]);
            }
        }
        if (tid >= 64) {
            const int i = tid - 64;
#pragma unroll 1
            for (int cc = 0; cc < DVT / 16; ++cc) {
                float o16[16];
                ptx::tmem_ld16(tl + COL_XY + cc * 16, o16);
                if (DK == 64) {
                    float p16[16];
                    ptx::tmem_ld16(tl + COL_DS + cc * 16, p16);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int u = 0; u < 16; ++u) o16[u] += p16[u];
                } else {
                    ptx::tmem_wait_ld();
                }
                if (i < Lc) store16_bf16(o + ((cs + i) * H + h) * DV + col_base + cc * 16, o16);
            }
        }
        ptx::tc_fence_before();
    }

    __syncthreads();
    if (ok && final_state && has_row) {
#pragma unroll
        for (int j = 0; j < DVT; j += 4)
            store4(final_state + st_off + (long long)tid * DV + j, make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]));
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, TMEM_COLS);
    }
}

inline size_t workspace_bytes(int num_seqs) {
    (void)num_seqs;
    return 0;
}

template <int DK, int DVT>
int launch_t(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
             const float *init_state, void *o, float *final_state, const int32_t *cu_seqlens, int T, int H,
             int dv, int num_seqs, cudaStream_t st, char *msg, size_t msg_len) {
    constexpr int smem = Layout<DK, DVT>::ALLOC;
    auto kern = chunk_tc_kernel<DK, DVT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) {
        snprintf(msg, msg_len, "cudaFuncSetAttribute(chunk_tc): %s", cudaGetErrorString(e));
        return KDA_ERR_CUDA;
    }
    dim3 grid(dv / DVT, H, num_seqs);
    kern<<<grid, NT, smem, st>>>((const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v,
                                  log_alpha, beta, init_state, (__nv_bfloat16 *)o, final_state, cu_seqlens, T, H,
                                  dv);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        snprintf(msg, msg_len, "chunk_tc launch: %s", cudaGetErrorString(e));
        return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

// Value-tile width: 64 columns when there are enough (sequence, head, tile) work
// items to fill the GPU twice over, else 32 for more CTAs.
inline int launch(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                  const float *init_state, void *o, float *final_state, const int32_t *cu_seqlens, int B, int T,
                  int H, int dk, int dv, int num_seqs, void *workspace, cudaStream_t st, char *msg,
                  size_t msg_len) {
    (void)B;
    (void)workspace;
    const long long items64 = (long long)num_seqs * H * (dv / 64);
    const bool wide = items64 >= 2 * 148;
    if (dk == 128)
        return wide ? launch_t<128, 64>(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, T, H, dv,
                                        num_seqs, st, msg, msg_len)
                    : launch_t<128, 32>(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, T, H, dv,
                                        num_seqs, st, msg, msg_len);
    return wide ? launch_t<64, 64>(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, T, H, dv,
                                   num_seqs, st, msg, msg_len)
                : launch_t<64, 32>(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, T, H, dv,
                                   num_seqs, st, msg, msg_len);
}

}  // namespace tc
}  // namespace kda
