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
// Mapping: one 256-thread CTA per (value-column tile of DVT, head, sequence) walks
// the sequence's chunks in order.  TMA brings each chunk's q, k, log_alpha and v
// tiles into shared memory, the next chunk's while the current one computes.
// All threads build the decayed bf16 operands (two key channels x one token
// segment each); threads 0..dk-1 keep row c of the fp32 state in registers, which
// is also TMEM lane c of every 128-row accumulator.  Thread 0 issues the MMAs;
// completion is signalled through mbarriers with bounded waits.  bf16 operands
// live in shared memory in the 128-byte-swizzled K-major layout the MMA
// descriptors name.
#pragma once

#include <cuda.h>

#include <cstdio>

#include "kda_common.cuh"
#include "tc_ptx.cuh"

namespace kda {
namespace tc {

constexpr int C = 64;
constexpr int NT = 256;
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;   // 1 s: far beyond any legitimate latency
constexpr uint32_t TMEM_COLS = 256;
// TMEM column map (fp32 accumulators, lane = row)
constexpr uint32_t COL_GRAM = 0;    // [128 x 64]  rows 0-63 Khat Rk^T, rows 64-127 Qhat Rk^T
constexpr uint32_t COL_XY = 64;     // [128 x DVT] rows 0-63 X, rows 64-127 Y (then O)
constexpr uint32_t COL_KT = 128;    // [128 x 64]  Kt (and Pt rows 64-127 when dk = 64)
constexpr uint32_t COL_PT = 192;    // [128 x 64]  rows 64-127 Pt (dk = 128)
constexpr uint32_t COL_DS = 0;      // [128 x DVT] Kt Z (reuses the Gram columns)
constexpr int AS = 68;              // fp32 row stride of the 64 x 64 scratch matrices (16-byte rows)

template <int DK, int DVT>
struct Layout {
    static constexpr int KA = DK / 64;                       // 64-element K atoms along dk
    // bf16 MMA operands, 128-byte swizzled, 1024-byte aligned
    static constexpr int KQ = 0;                             // [KA][128][128 B] Khat (0-63), Qhat (64-127)
    static constexpr int RK = KQ + KA * 128 * 128;           // [KA][64][128 B]  Rk
    static constexpr int SB = RK + KA * 64 * 128;            // [KA][DVT][128 B] S^T (bf16): B operand
    static constexpr int KP = SB + KA * DVT * 128;           // [DK+64][128 B]   Kbar^T -> Kt ; Aqk -> Pt
    static constexpr int TB = KP + (DK + 64) * 128;          // [64][128 B]      Tb^T
    static constexpr int ZT = TB + 64 * 128;                 // [DVT][128 B]     Z^T
    // dense TMA input tiles; the fp32 scratch of the UT transform aliases them
    static constexpr int QIN = ZT + DVT * 128;               // bf16 [64][DK]
    static constexpr int KIN = QIN + 64 * DK * 2;            // bf16 [64][DK]
    static constexpr int GIN = KIN + 64 * DK * 2;            // fp32 [64][DK]
    static constexpr int IN_BYTES = 64 * DK * 8;
    static constexpr int FA = QIN;                           // fp32 [64][AS]   Diag(beta) Akk
    static constexpr int FT = FA + 64 * AS * 4;              // fp32 [64][AS]   T
    static constexpr int FM = FT + 64 * AS * 4;              // fp32 [32][36]   block-product scratch
    static constexpr int SCR_BYTES = 2 * 64 * AS * 4 + 32 * 36 * 4;
    static constexpr int SPAN = IN_BYTES > SCR_BYTES ? IN_BYTES : SCR_BYTES;
    static constexpr int VIN = QIN + SPAN;                   // bf16 [2][64][DVT]
    static constexpr int FB = VIN + 2 * 64 * DVT * 2;        // fp32 [2][64]    beta
    static constexpr int FD = FB + 2 * 64 * 4;               // fp32 [DK]       e^{G_last}
    static constexpr int NSEG = NT / (DK / 2);               // token segments in the factor stage
    static constexpr int FSEG = FD + DK * 4;                 // fp32 [NSEG][DK] segment sums of log_alpha
    static constexpr int MISC = FSEG + NSEG * DK * 4;        // mbarriers, TMEM base, flags
    static constexpr int BYTES = MISC + 64;
    static constexpr int ALLOC = BYTES + 1024;               // room to align the base to 1024 B
    static_assert(KQ % 1024 == 0 && RK % 1024 == 0 && SB % 1024 == 0 && KP % 1024 == 0 &&
                      TB % 1024 == 0 && ZT % 1024 == 0 && QIN % 1024 == 0 && VIN % 128 == 0,
                  "tile alignment");
    static_assert(ALLOC <= 232448, "shared memory budget");
};

// Byte offset of bf16 element (row, k) in a K-major, 128-byte-swizzled tile whose
// K atoms (64 elements each) hold `rows` rows.
__device__ __forceinline__ uint32_t sw128(int row, int k, int rows) {
    const int atom = k >> 6, kk = k & 63;
    return (uint32_t)(atom * rows * 128 + row * 128 + ((((kk >> 3) ^ (row & 7))) << 4) + ((kk & 7) << 1));
}
// Byte offset of the 16-byte group holding elements (row, 8g .. 8g+7) of a one-atom (64-wide) tile.
__device__ __forceinline__ uint32_t sw128_chunk(int row, int g) {
    return (uint32_t)(row * 128 + ((g ^ (row & 7)) << 4));
}

__device__ __forceinline__ void st_bf16(uint8_t *base, uint32_t off, float x) {
    *reinterpret_cast<__nv_bfloat16 *>(base + off) = __float2bfloat16_rn(x);
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ void st_bf16x2(uint8_t *base, uint32_t off, float a, float b) {
    *reinterpret_cast<uint32_t *>(base + off) = pack_bf16(a, b);
}
// Eight consecutive values of a row as one 16-byte swizzled store.
__device__ __forceinline__ void st_bf16x8(uint8_t *base, uint32_t off, const float *x) {
    *reinterpret_cast<uint4 *>(base + off) =
        make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
}

__device__ __forceinline__ float exp2_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Descriptor of the 16-wide K step `s` of a swizzled tile at `addr` with `rows`
// rows per K atom, starting at row r0 (a multiple of 8).
__device__ __forceinline__ uint64_t kdesc(uint32_t addr, int s, int rows, int r0 = 0) {
    return ptx::desc_kmajor_sw128(addr + (uint32_t)((s >> 2) * rows * 128 + r0 * 128 + (s & 3) * 32));
}

// T = (I + A)^{-1} for a 64 x 64 strictly lower A (fp32, row stride AS): the four
// 16 x 16 diagonal blocks by forward substitution, then the block-triangular
// inverse [L11 0; L21 L22]^{-1} = [L11^-1 0; -L22^-1 L21 L11^-1  L22^-1] at 32 and
// 64, each block product register-tiled over 256 threads.  The lower triangle
// of T and the zero upper triangles of its four 16 x 16 diagonal blocks are
// written; nothing reads T above those blocks.
__device__ __forceinline__ void invert_unit_lower64(const float *A, float *Tm, float *M, int tid) {
    if (tid < 64) {
        const int o = 16 * (tid >> 4), l = tid & 15;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < i; ++j) acc = fmaf(A[(o + i) * AS + o + j], x[j], acc);
            x[i] = (i < l) ? 0.f : ((i == l) ? 1.f : -acc);
        }
        // the whole block column, zeros above the diagonal included: the vectorised
        // block products below read a few of those entries
#pragma unroll
        for (int i = 0; i < 16; ++i) Tm[(o + i) * AS + o + l] = x[i];
    }
    __syncthreads();
    {   // M_p = A[2p+1][2p] T[2p][2p]; then T[2p+1][2p] = -T[2p+1][2p+1] M_p   (p = 0, 1)
        const int p = tid >> 7, r = (tid >> 3) & 15, c = (tid & 7) * 2;
        const int ro = 32 * p + 16, co = 32 * p;
        float a0 = 0.f, a1 = 0.f;
        for (int j = c; j < 16; ++j) {
            const float a = A[(ro + r) * AS + co + j];
            const float2 t = *reinterpret_cast<const float2 *>(Tm + (co + j) * AS + co + c);
            a0 = fmaf(a, t.x, a0);
            a1 = fmaf(a, t.y, a1);
        }
        *reinterpret_cast<float2 *>(M + p * 16 * 36 + r * 36 + c) = make_float2(a0, a1);
        __syncthreads();
        float b0 = 0.f, b1 = 0.f;
        for (int j = 0; j <= r; ++j) {
            const float t = Tm[(ro + r) * AS + ro + j];
            const float2 m = *reinterpret_cast<const float2 *>(M + p * 16 * 36 + j * 36 + c);
            b0 = fmaf(t, m.x, b0);
            b1 = fmaf(t, m.y, b1);
        }
        *reinterpret_cast<float2 *>(Tm + (ro + r) * AS + co + c) = make_float2(-b0, -b1);
    }
    __syncthreads();
    {   // M = A[hi][lo] T[lo][lo]; then T[hi][lo] = -T[hi][hi] M   (32 x 32 blocks)
        const int r = tid >> 3, c = (tid & 7) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = c; j < 32; ++j) {
            const float a = A[(32 + r) * AS + j];
            const float4 t = *reinterpret_cast<const float4 *>(Tm + j * AS + c);
            acc.x = fmaf(a, t.x, acc.x); acc.y = fmaf(a, t.y, acc.y);
            acc.z = fmaf(a, t.z, acc.z); acc.w = fmaf(a, t.w, acc.w);
        }
        *reinterpret_cast<float4 *>(M + r * 36 + c) = acc;
        __syncthreads();
        float4 b = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j <= r; ++j) {
            const float t = Tm[(32 + r) * AS + 32 + j];
            const float4 m = *reinterpret_cast<const float4 *>(M + j * 36 + c);
            b.x = fmaf(t, m.x, b.x); b.y = fmaf(t, m.y, b.y);
            b.z = fmaf(t, m.z, b.z); b.w = fmaf(t, m.w, b.w);
        }
        *reinterpret_cast<float4 *>(Tm + (32 + r) * AS + c) = make_float4(-b.x, -b.y, -b.z, -b.w);
    }
    __syncthreads();
}

// Every thread waits for the next completion of an mbarrier; all agree on the
// outcome (a shared "failed" flag from warp-local waits is folded in).  Returns
// false, and flags the device status, on timeout.
__device__ __forceinline__ bool wait_all(uint32_t mbar, uint32_t &phase, int local_fail = 0) {
    const bool ok = ptx::mbar_wait_bounded(mbar, phase, WAIT_LIMIT_NS);
    phase ^= 1u;
    if (__syncthreads_or((!ok) || local_fail)) {
        if (threadIdx.x == 0) flag_status(KDA_DEV_WAIT_TIMEOUT);
        return false;
    }
    ptx::tc_fence_after();
    return true;
}

__device__ __forceinline__ void unpack_bf16x8(uint4 u, float *x) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}

template <int DK, int DVT>
__global__ void __launch_bounds__(NT, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_v,
                const float *__restrict__ beta, const float *__restrict__ init_state,
                __nv_bfloat16 *__restrict__ o, float *__restrict__ final_state,
                const int32_t *__restrict__ cu_seqlens, int T, int H, int DV) {
    using L = Layout<DK, DVT>;
    static_assert(DVT % 16 == 0 && DVT >= 16 && DVT <= 64, "value tile");
    constexpr int NPAIR = DK / 2, NSEG = L::NSEG, SEGLEN = C / NSEG;
    constexpr float LOG2E = 1.4426950408889634f;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = ptx::smem_u32(sm);
    float *fA = reinterpret_cast<float *>(sm + L::FA);
    float *fT = reinterpret_cast<float *>(sm + L::FT);
    float *fM = reinterpret_cast<float *>(sm + L::FM);
    float *fB = reinterpret_cast<float *>(sm + L::FB);
    float *fD = reinterpret_cast<float *>(sm + L::FD);
    float *fSeg = reinterpret_cast<float *>(sm + L::FSEG);
    const uint32_t bar_mma = sb + L::MISC, bar_in = sb + L::MISC + 8;
    const uint32_t bar_v0 = sb + L::MISC + 16;          // + 8 * buffer
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::MISC + 32);
    int *fail_flag = reinterpret_cast<int *>(sm + L::MISC + 36);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int col_base = blockIdx.x * DVT, h = blockIdx.y, n = blockIdx.z;

    long long t0, t1;
    seq_span(cu_seqlens, T, n, t0, t1);
    const int nck = (int)((t1 - t0 + C - 1) / C);

    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), TMEM_COLS);
        ptx::tmem_relinquish();
    }
    if (tid == 0) {
        ptx::mbar_init(bar_mma, 1);
        ptx::mbar_init(bar_in, 1);
        ptx::mbar_init(bar_v0, 1);
        ptx::mbar_init(bar_v0 + 8, 1);
        *fail_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_g);
        ptx::prefetch_tmap(&tm_v);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);   // this warp's TMEM lane quadrant
    uint32_t ph_mma = 0, ph_in = 0, ph_v[2] = {0u, 0u};

    auto issue_inputs = [&](int ci) {   // thread 0 only
        const int z = (int)(t0 + (long long)ci * C);
        ptx::mbar_arrive_expect_tx(bar_in, (uint32_t)L::IN_BYTES);
        ptx::tma_load_3d(sb + L::QIN, &tm_q, bar_in, 0, h, z);
        ptx::tma_load_3d(sb + L::KIN, &tm_k, bar_in, 0, h, z);
        ptx::tma_load_3d(sb + L::GIN, &tm_g, bar_in, 0, h, z);
    };
    auto issue_v = [&](int ci) {        // thread 0 only
        const int z = (int)(t0 + (long long)ci * C);
        const uint32_t bar = bar_v0 + 8u * (uint32_t)(ci & 1);
        ptx::mbar_arrive_expect_tx(bar, (uint32_t)(C * DVT * 2));
        ptx::tma_load_3d(sb + L::VIN + (uint32_t)((ci & 1) * C * DVT * 2), &tm_v, bar, col_base, h, z);
    };

    const bool has_row = tid < DK;
    const long long st_off = ((long long)n * H + h) * DK * DV + col_base;
    float S[DVT];
#pragma unroll
    for (int j = 0; j < DVT; j += 4) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (has_row && init_state) x = load4(init_state + st_off + (long long)tid * DV + j);
        S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
    }
    if (nck > 0) {
        if (tid == 0) {
            issue_inputs(0);
            issue_v(0);
        }
        if (tid < C) {
            const int L0 = (int)min((long long)C, t1 - t0);
            fB[tid] = tid < L0 ? beta[(t0 + tid) * H + h] : 0.f;
        }
        if (has_row) {
#pragma unroll
            for (int j = 0; j < DVT; ++j) st_bf16(sm, L::SB + sw128(j, tid, DVT), S[j]);
        }
    }

    bool ok = true;
    for (int ci = 0; ci < nck; ++ci) {
        const long long cs = t0 + (long long)ci * C;
        const int Lc = (int)min((long long)C, t1 - cs);
        const int buf = ci & 1;
        float beta_next = 0.f;
        if (ci + 1 < nck) {
            if (tid == 0) issue_v(ci + 1);
            if (tid < C) {
                const int Ln = (int)min((long long)C, t1 - cs - C);
                beta_next = tid < Ln ? beta[(cs + C + tid) * H + h] : 0.f;
            }
        }

        // ---- 1. decay factors -> bf16 operand tiles (two channels x one token segment per thread)
        if (!(ok = wait_all(bar_in, ph_in))) break;
        {
            const int pr = tid % NPAIR, seg = tid / NPAIR, c0 = 2 * pr;
            const float *gin = reinterpret_cast<const float *>(sm + L::GIN);
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int u = 0; u < SEGLEN; ++u) {
                const int i = seg * SEGLEN + u;
                if (i < Lc) {
                    const float2 g2 = *reinterpret_cast<const float2 *>(gin + i * DK + c0);
                    s0 += g2.x;
                    s1 += g2.y;
                }
            }
            fSeg[seg * DK + c0] = s0;
            fSeg[seg * DK + c0 + 1] = s1;
            __syncthreads();
            float G0 = 0.f, G1 = 0.f, tot0 = 0.f, tot1 = 0.f;
#pragma unroll
            for (int s = 0; s < NSEG; ++s) {
                const float a = fSeg[s * DK + c0], b = fSeg[s * DK + c0 + 1];
                if (s < seg) { G0 += a; G1 += b; }
                tot0 += a;
                tot1 += b;
            }
            const float d0 = expf(tot0), d1 = expf(tot1);
            if (seg == 0) {
                fD[c0] = d0;
                fD[c0 + 1] = d1;
                if (tot0 < -80.f || tot1 < -80.f) flag_status(KDA_DEV_DECAY_RANGE);
            }
            const __nv_bfloat162 *qin = reinterpret_cast<const __nv_bfloat162 *>(sm + L::QIN);
            const __nv_bfloat162 *kin = reinterpret_cast<const __nv_bfloat162 *>(sm + L::KIN);
#pragma unroll
            for (int u = 0; u < SEGLEN; u += 2) {
                float kb0[2], kb1[2];
#pragma unroll
                for (int w = 0; w < 2; ++w) {
                    const int i = seg * SEGLEN + u + w;
                    float2 q2 = make_float2(0.f, 0.f), k2 = make_float2(0.f, 0.f), g2 = make_float2(0.f, 0.f);
                    if (i < Lc) {
                        q2 = __bfloat1622float2(qin[(i * DK + c0) >> 1]);
                        k2 = __bfloat1622float2(kin[(i * DK + c0) >> 1]);
                        g2 = *reinterpret_cast<const float2 *>(gin + i * DK + c0);
                    }
                    G0 += g2.x;
                    G1 += g2.y;
                    const float e0 = exp2_fast(G0 * LOG2E), e1 = exp2_fast(G1 * LOG2E);
                    const float r0 = exp2_fast(-G0 * LOG2E), r1 = exp2_fast(-G1 * LOG2E);
                    st_bf16x2(sm, L::KQ + sw128(i, c0, 128), k2.x * e0, k2.y * e1);
                    st_bf16x2(sm, L::KQ + sw128(64 + i, c0, 128), q2.x * e0, q2.y * e1);
                    st_bf16x2(sm, L::RK + sw128(i, c0, 64), k2.x * r0, k2.y * r1);
                    kb0[w] = k2.x * (d0 * r0);
                    kb1[w] = k2.y * (d1 * r1);
                }
                const int i0 = seg * SEGLEN + u;
                st_bf16x2(sm, L::KP + sw128(c0, i0, DK + 64), kb0[0], kb0[1]);
                st_bf16x2(sm, L::KP + sw128(c0 + 1, i0, DK + 64), kb1[0], kb1[1]);
            }
        }
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
            ptx::mma_commit(bar_mma);
        }
        if (!(ok = wait_all(bar_mma, ph_mma))) break;

        // ---- 3. Gram -> Diag(beta) Akk (fp32) and masked Aqk (bf16); Z = V - X; UT transform
        if (warp < 4) {
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                float g32[32];
                ptx::tmem_ld32(tl + COL_GRAM + hh * 32, g32);
                ptx::tmem_wait_ld();
                if (tid < 64) {
                    const int i = tid;
                    const float bi = fB[buf * C + i];
#pragma unroll
                    for (int u = 0; u < 32; u += 4) {
                        const int j = hh * 32 + u;
                        float4 a;
                        a.x = (j + 0 < i) ? bi * g32[u + 0] : 0.f;
                        a.y = (j + 1 < i) ? bi * g32[u + 1] : 0.f;
                        a.z = (j + 2 < i) ? bi * g32[u + 2] : 0.f;
                        a.w = (j + 3 < i) ? bi * g32[u + 3] : 0.f;
                        *reinterpret_cast<float4 *>(fA + i * AS + j) = a;
                    }
                } else {
                    const int i = tid - 64;
#pragma unroll
                    for (int u = 0; u < 32; ++u) g32[u] = (hh * 32 + u <= i) ? g32[u] : 0.f;
#pragma unroll
                    for (int gq = 0; gq < 4; ++gq)
                        st_bf16x8(sm, L::KP + (uint32_t)(DK + i) * 128 + ((((hh * 4 + gq) ^ ((DK + i) & 7))) << 4),
                                  g32 + gq * 8);
                }
            }
        } else if (warp < 6) {
            // X rows (TMEM lanes 0-63) -> Z = V - X -> Z^T
            int lf = 0;
            if (!ptx::mbar_wait_bounded(bar_v0 + 8u * (uint32_t)buf, ph_v[buf], WAIT_LIMIT_NS)) lf = 1;
            if (lf) *fail_flag = 1;
            const int j = (warp - 4) * 32 + lane;
            const uint8_t *vin = sm + L::VIN + buf * C * DVT * 2;
#pragma unroll 1
            for (int cc = 0; cc < DVT / 16; ++cc) {
                float x16[16], v16[16];
                ptx::tmem_ld16(tl + COL_XY + cc * 16, x16);
                if (j < Lc) {
                    unpack_bf16x8(*reinterpret_cast<const uint4 *>(vin + (j * DVT + cc * 16) * 2), v16);
                    unpack_bf16x8(*reinterpret_cast<const uint4 *>(vin + (j * DVT + cc * 16 + 8) * 2), v16 + 8);
                } else {
#pragma unroll
                    for (int u = 0; u < 16; ++u) v16[u] = 0.f;
                }
                ptx::tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 16; ++u) st_bf16(sm, L::ZT + sw128(cc * 16 + u, j, DVT), v16[u] - x16[u]);
            }
        }
        ph_v[buf] ^= 1u;
        __syncthreads();
        invert_unit_lower64(fA, fT, fM, tid);
        {   // Tb^T[j][l] = T[l][j] beta_j   (l >= j)
            const int j = tid & 63, lq = tid >> 6;
            const float bj = fB[buf * C + j];
            float t16[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int l = lq * 16 + u;
                t16[u] = (l >= j) ? fT[l * AS + j] * bj : 0.f;
            }
            st_bf16x8(sm, L::TB + sw128_chunk(j, 2 * lq), t16);
            st_bf16x8(sm, L::TB + sw128_chunk(j, 2 * lq + 1), t16 + 8);
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();

        // ---- 4. Kt = Kbar^T Tb, Pt = Aqk Tb ; next chunk's inputs (scratch is free now)
        if (tid == 0) {
            if (ci + 1 < nck) issue_inputs(ci + 1);
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
            ptx::mma_commit(bar_mma);
        }
        if (!(ok = wait_all(bar_mma, ph_mma, *fail_flag))) break;

        // ---- 5. Kt, Pt -> bf16 A operands
        if (warp < 4) {
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                float k32[32];
                ptx::tmem_ld32(tl + COL_KT + hh * 32, k32);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int gq = 0; gq < 4; ++gq)
                    st_bf16x8(sm, L::KP + (uint32_t)tid * 128 + ((((hh * 4 + gq) ^ (tid & 7))) << 4), k32 + gq * 8);
            }
        } else if (DK == 128 && warp >= 6) {
            const int i = (warp - 6) * 32 + lane;
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                float p32[32];
                ptx::tmem_ld32(tl + COL_PT + hh * 32, p32);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int gq = 0; gq < 4; ++gq)
                    st_bf16x8(sm, L::KP + (uint32_t)(DK + i) * 128 + ((((hh * 4 + gq) ^ ((DK + i) & 7))) << 4),
                              p32 + gq * 8);
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
            ptx::mma_commit(bar_mma);
        }
        if (!(ok = wait_all(bar_mma, ph_mma))) break;

        // ---- 7. S <- Diag(e^{G_last}) S + dS (and its bf16 copy for the next chunk); store O rows
        if (warp < 4) {
            const float dch = has_row ? fD[tid] : 0.f;
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
            if (has_row && ci + 1 < nck) {
#pragma unroll
                for (int j = 0; j < DVT; ++j) st_bf16(sm, L::SB + sw128(j, tid, DVT), S[j]);
            }
        } else if (warp >= 6) {
            const int i = (warp - 6) * 32 + lane;
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
                if (i < Lc) {
                    __nv_bfloat16 *dst = o + ((cs + i) * H + h) * DV + col_base + cc * 16;
                    reinterpret_cast<uint4 *>(dst)[0] = make_uint4(pack_bf16(o16[0], o16[1]), pack_bf16(o16[2], o16[3]),
                                                                   pack_bf16(o16[4], o16[5]), pack_bf16(o16[6], o16[7]));
                    reinterpret_cast<uint4 *>(dst)[1] =
                        make_uint4(pack_bf16(o16[8], o16[9]), pack_bf16(o16[10], o16[11]),
                                   pack_bf16(o16[12], o16[13]), pack_bf16(o16[14], o16[15]));
                }
            }
        }
        if (tid < C && ci + 1 < nck) fB[(buf ^ 1) * C + tid] = beta_next;
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

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                    const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [tokens, H, inner] row-major tensor -> box (box_inner, 1, 64 tokens).
inline bool make_tmap(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize, long long tokens,
                      int H, int inner, int box_inner) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)H, (cuuint64_t)tokens};
    cuuint64_t strides[2] = {(cuuint64_t)inner * esize, (cuuint64_t)inner * esize * H};
    cuuint32_t box[3] = {(cuuint32_t)box_inner, 1u, (cuuint32_t)C};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK, int DVT>
int launch_t(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
             const float *init_state, void *o, float *final_state, const int32_t *cu_seqlens, long long tokens,
             int T, int H, int dv, int num_seqs, cudaStream_t st, char *msg, size_t msg_len) {
    CUtensorMap tq, tk, tg, tv;
    if (!make_tmap(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, DK, DK) ||
        !make_tmap(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, DK, DK) ||
        !make_tmap(&tg, log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, tokens, H, DK, DK) ||
        !make_tmap(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, dv, DVT)) {
        snprintf(msg, msg_len, "building TMA descriptors failed (driver entry point cuTensorMapEncodeTiled)");
        return KDA_ERR_CUDA;
    }
    constexpr int smem = Layout<DK, DVT>::ALLOC;
    auto kern = chunk_tc_kernel<DK, DVT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) {
        snprintf(msg, msg_len, "cudaFuncSetAttribute(chunk_tc): %s", cudaGetErrorString(e));
        return KDA_ERR_CUDA;
    }
    dim3 grid(dv / DVT, H, num_seqs);
    kern<<<grid, NT, smem, st>>>(tq, tk, tg, tv, beta, init_state, (__nv_bfloat16 *)o, final_state, cu_seqlens,
                                  T, H, dv);
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
    (void)workspace;
    const long long tokens = (long long)B * T;
    if (tokens == 0) {
        // no tokens: the final state is the initial state (or zeros)
        if (final_state) {
            const size_t bytes = (size_t)num_seqs * H * dk * dv * sizeof(float);
            cudaError_t e = init_state ? cudaMemcpyAsync(final_state, init_state, bytes, cudaMemcpyDeviceToDevice, st)
                                       : cudaMemsetAsync(final_state, 0, bytes, st);
            if (e != cudaSuccess) {
                snprintf(msg, msg_len, "state copy: %s", cudaGetErrorString(e));
                return KDA_ERR_CUDA;
            }
        }
        return KDA_OK;
    }
    if (tokens > 0x7fffffffLL) {
        snprintf(msg, msg_len, "B*T=%lld exceeds the 2^31 token limit of the TMA coordinates", tokens);
        return KDA_ERR_UNSUPPORTED;
    }
    const long long items64 = (long long)num_seqs * H * (dv / 64);
    const bool wide = items64 >= 2 * 148;
#define KDA_TC(DKv, DVTv)                                                                                   \
    return launch_t<DKv, DVTv>(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, tokens, T, \
                               H, dv, num_seqs, st, msg, msg_len)
    if (dk == 128) {
        if (wide) KDA_TC(128, 64);
        KDA_TC(128, 32);
    }
    if (wide) KDA_TC(64, 64);
    KDA_TC(64, 32);
#undef KDA_TC
}

}  // namespace tc
}  // namespace kda
