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
constexpr long long WAIT_LIMIT_CYCLES = 2000000000ll;   // >= 1 s at any SM clock up to 2 GHz: far beyond any legitimate latency
constexpr uint32_t TMEM_COLS = 512;
// TMEM column map (fp32 accumulators, lane = row)
constexpr uint32_t COL_GRAM = 0;    // [128 x 64]  rows 0-63 Kp Kbar^T, rows 64-127 Qp Kbar^T
constexpr uint32_t COL_XY = 64;     // [128 x DVT] rows 0-63 X, rows 64-127 Y, then O (same MMA as the Gram)
constexpr uint32_t COL_KT = 192;    // [128 x 64]  Kt (lanes 0..dk-1)
constexpr uint32_t COL_PT = 256;    // [128 x 64]  Pt (lanes 64-127)
constexpr uint32_t COL_DS = 320;    // [128 x DVT] Kt Z (lanes 0..dk-1)
constexpr int AS = 68;              // fp32 row stride of the 64 x 64 scratch matrices (16-byte rows)

template <int DK, int DVT>
struct Layout {
    static constexpr int KA = DK / 64;                       // 64-element K atoms along dk
    // bf16 MMA operands, 128-byte swizzled, 1024-byte aligned
    static constexpr int KQ = 0;                             // [KA][128][128 B] Kp (0-63), Qp (64-127)
    static constexpr int KSR = 64 + DVT;                     // rows of the combined B operand
    static constexpr int KS = KQ + KA * 128 * 128;           // [KA][64+DVT][128 B] rows 0-63 Kbar (tokens),
                                                             //   rows 64.. (e^{G_last} S)^T (value columns)
    static constexpr int KP = KS + KA * KSR * 128;           // [DK+64][128 B]   Kt (0..DK-1), Aqk -> Pt (DK..)
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
    static constexpr int VIN = QIN + SPAN;                   // bf16 [64][DVT]
    static constexpr int FB = VIN + 64 * DVT * 2;            // fp32 [2][64]    beta
    static constexpr int NSEG = NT / (DK / 4);               // token segments in the factor stage
    static constexpr int FSEG = FB + 2 * 64 * 4;             // fp32 [NSEG][DK] segment sums of log_alpha
    static constexpr int MISC = FSEG + NSEG * DK * 4;        // mbarriers, TMEM base, flags
    static constexpr int BYTES = MISC + 64;
    static constexpr int ALLOC = BYTES + 1024;               // room to align the base to 1024 B
    static_assert(KQ % 1024 == 0 && KS % 1024 == 0 && KP % 1024 == 0 && TB % 1024 == 0 && ZT % 1024 == 0 &&
                      QIN % 1024 == 0 && VIN % 128 == 0,
                  "tile alignment");
    static_assert(ALLOC <= 232448, "shared memory budget");
};

// Byte offset of bf16 element (row, k) in a 128-byte-swizzled tile whose 64-wide
// K atoms hold `rows` rows each.
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
// Four consecutive values of a row as one 8-byte store (8-byte aligned offsets).
__device__ __forceinline__ void st_bf16x4(uint8_t *base, uint32_t off, float a, float b, float c, float d) {
    *reinterpret_cast<uint2 *>(base + off) = make_uint2(pack_bf16(a, b), pack_bf16(c, d));
}
__device__ __forceinline__ float4 ld_bf16x4(const uint8_t *p) {
    const uint2 r = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&r.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&r.y));
    return make_float4(a.x, a.y, b.x, b.y);
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

// Descriptor of the 16-wide K step `s` of a K-major swizzled tile at `addr` with
// `rows` rows per K atom, starting at row r0 (a multiple of 8).
__device__ __forceinline__ uint64_t kdesc(uint32_t addr, int s, int rows, int r0 = 0) {
    return ptx::desc_kmajor_sw128(addr + (uint32_t)((s >> 2) * rows * 128 + r0 * 128 + (s & 3) * 32));
}

__device__ __forceinline__ uint32_t f2tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// d (16 x 8 fragment of one warp) += X (16 x 8K, row-major, stride sx) * Y (8K x 8,
// row-major, stride sy) on the tensor cores with tf32 inputs and fp32
// accumulation (m16n8k8 fragments: lane = 4 g + t).
template <int KSTEPS>
__device__ __forceinline__ void warp_mm16x8_tf32(float (&d)[4], const float *X, int sx, const float *Y, int sy,
                                                 int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
        const int k0 = ks * 8;
        const uint32_t a0 = f2tf32(X[g * sx + k0 + t]), a1 = f2tf32(X[(g + 8) * sx + k0 + t]);
        const uint32_t a2 = f2tf32(X[g * sx + k0 + t + 4]), a3 = f2tf32(X[(g + 8) * sx + k0 + t + 4]);
        const uint32_t b0 = f2tf32(Y[(k0 + t) * sy + g]), b1 = f2tf32(Y[(k0 + t + 4) * sy + g]);
        asm volatile(
            "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
}

__device__ __forceinline__ void warp_store16x8(float *Z, int sz, const float (&d)[4], float sign, int lane) {
    const int g = lane >> 2, t = lane & 3;
    *reinterpret_cast<float2 *>(Z + g * sz + 2 * t) = make_float2(sign * d[0], sign * d[1]);
    *reinterpret_cast<float2 *>(Z + (g + 8) * sz + 2 * t) = make_float2(sign * d[2], sign * d[3]);
}

// The same 16 x 8 tile of T (rows r0.., columns c0..) as Tb^T entries:
// Tb^T[c][r] = sign * T[r][c] * beta_c, bf16, into the swizzled operand tile.
__device__ __forceinline__ void warp_store16x8_tbt(uint8_t *tb, int r0, int c0, const float (&d)[4], float sign,
                                                  const float *beta, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int ca = c0 + 2 * t, cb = ca + 1;
    const float ba = sign * beta[ca], bb = sign * beta[cb];
    st_bf16(tb, sw128(ca, r0 + g, 64), d[0] * ba);
    st_bf16(tb, sw128(cb, r0 + g, 64), d[1] * bb);
    st_bf16(tb, sw128(ca, r0 + g + 8, 64), d[2] * ba);
    st_bf16(tb, sw128(cb, r0 + g + 8, 64), d[3] * bb);
}

// Diagonal 16 x 16 blocks of T = (I + A)^{-1} (A strictly lower, fp32, row stride
// AS) by forward substitution: 64 threads, one block column each, zeros above the
// diagonal included.
__device__ __forceinline__ void invert_diag_blocks(const float *A, float *Tm, uint8_t *tb, const float *beta,
                                                   int t64) {
    const int o = 16 * (t64 >> 4), l = t64 & 15;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int j4 = 0; j4 < 16; j4 += 4) {
            if (j4 < i) {
                const float4 a = *reinterpret_cast<const float4 *>(A + (o + i) * AS + o + j4);
                if (j4 + 0 < i) acc = fmaf(a.x, x[j4 + 0], acc);
                if (j4 + 1 < i) acc = fmaf(a.y, x[j4 + 1], acc);
                if (j4 + 2 < i) acc = fmaf(a.z, x[j4 + 2], acc);
                if (j4 + 3 < i) acc = fmaf(a.w, x[j4 + 3], acc);
            }
        }
        x[i] = (i < l) ? 0.f : ((i == l) ? 1.f : -acc);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) Tm[(o + i) * AS + o + l] = x[i];
    // Tb^T[o+l][o+i] = T[o+i][o+l] beta_{o+l}: one 32-byte row segment of the bf16 operand
    const float bl = beta[o + l];
    float t16[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) t16[i] = x[i] * bl;
    st_bf16x8(tb, sw128_chunk(o + l, o / 8), t16);
    st_bf16x8(tb, sw128_chunk(o + l, o / 8 + 1), t16 + 8);
}

// The rest of T once its diagonal blocks are in place and blocks (0,1) and (2,3)
// are zero: the block-triangular inverse [L11 0; L21 L22]^{-1} =
// [L11^-1 0; -L22^-1 L21 L11^-1  L22^-1] at 32 (two pairs of 16-blocks) and at 64,
// each block product one 16 x 8 tile per warp on the tensor cores (tf32 inputs,
// fp32 accumulation).  All 256 threads take part.
__device__ __forceinline__ void invert_merge_blocks(const float *A, float *Tm, float *M, uint8_t *tb,
                                                    const float *beta, int warp, int lane) {
    if (warp < 4) {   // M_p = A[2p+1][2p] T[2p][2p]
        const int p = warp >> 1, nt = warp & 1, ro = 32 * p + 16, co = 32 * p;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        warp_mm16x8_tf32<2>(d, A + ro * AS + co, AS, Tm + co * AS + co + 8 * nt, AS, lane);
        warp_store16x8(M + p * 16 * 36 + 8 * nt, 36, d, 1.f, lane);
    }
    __syncthreads();
    if (warp < 4) {   // T[2p+1][2p] = -T[2p+1][2p+1] M_p
        const int p = warp >> 1, nt = warp & 1, ro = 32 * p + 16, co = 32 * p;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        warp_mm16x8_tf32<2>(d, Tm + ro * AS + ro, AS, M + p * 16 * 36 + 8 * nt, 36, lane);
        warp_store16x8(Tm + ro * AS + co + 8 * nt, AS, d, -1.f, lane);
        warp_store16x8_tbt(tb, ro, co + 8 * nt, d, -1.f, beta, lane);
    }
    __syncthreads();
    const int mt = warp >> 2, nt = warp & 3;
    {   // M = A[hi][lo] T[lo][lo]
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        warp_mm16x8_tf32<4>(d, A + (32 + 16 * mt) * AS, AS, Tm + 8 * nt, AS, lane);
        warp_store16x8(M + 16 * mt * 36 + 8 * nt, 36, d, 1.f, lane);
    }
    __syncthreads();
    {   // T[hi][lo] = -T[hi][hi] M
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        warp_mm16x8_tf32<4>(d, Tm + (32 + 16 * mt) * AS + 32, AS, M + 8 * nt, 36, lane);
        warp_store16x8_tbt(tb, 32 + 16 * mt, 8 * nt, d, -1.f, beta, lane);
    }
}

// Every thread waits for the next completion of an mbarrier; all agree on the
// outcome (a shared "failed" flag from warp-local waits is folded in).  Returns
// false, and flags the device status, on timeout.
__device__ __forceinline__ bool wait_all(uint32_t mbar, uint32_t &phase, int local_fail = 0) {
    const bool ok = ptx::mbar_wait_bounded(mbar, phase, WAIT_LIMIT_CYCLES);
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

// Threads are grouped by TMEM lane quadrant: warp w reads lanes 32 (w % 4) ..
// 32 (w % 4) + 31.  State row r (= key channel = TMEM lane) is held by the two
// warps with w % 4 == r / 32, one per half of the value tile's columns.
// GS: scalar gate (Gated DeltaNet), read from g_scalar [tokens, H] instead of the
// per-channel log_alpha tile that tm_g describes.
template <int DK, int DVT, bool GS>
__global__ void __launch_bounds__(NT, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_v,
                const float *__restrict__ beta, const float *__restrict__ init_state,
                __nv_bfloat16 *__restrict__ o, float *__restrict__ final_state,
                const int32_t *__restrict__ cu_seqlens, int T, int H, int DV, const int32_t *__restrict__ slots,
                int num_slots, const float *__restrict__ g_scalar) {
    using L = Layout<DK, DVT>;
    static_assert(DVT % 32 == 0 && DVT >= 32 && DVT <= 128, "value tile");
    constexpr int NCG = DK / 4, NSEG = L::NSEG, SEGLEN = C / NSEG;   // factor stage: 4 channels x SEGLEN tokens
    constexpr int CPT = DVT / 2;                              // state / output columns per thread
    constexpr float LOG2E = 1.4426950408889634f;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = ptx::smem_u32(sm);
    float *fA = reinterpret_cast<float *>(sm + L::FA);
    float *fT = reinterpret_cast<float *>(sm + L::FT);
    float *fM = reinterpret_cast<float *>(sm + L::FM);
    float *fB = reinterpret_cast<float *>(sm + L::FB);
    float *fSeg = reinterpret_cast<float *>(sm + L::FSEG);
    const uint32_t bar_mma = sb + L::MISC, bar_in = sb + L::MISC + 8, bar_v = sb + L::MISC + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::MISC + 32);
    int *fail_flag = reinterpret_cast<int *>(sm + L::MISC + 36);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const int col_base = blockIdx.x * DVT, h = blockIdx.y;
    const int n = seq_for_cta(cu_seqlens, T, (int)gridDim.z);

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
        ptx::mbar_init(bar_v, 1);
        *fail_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        if constexpr (!GS) ptx::prefetch_tmap(&tm_g);
        ptx::prefetch_tmap(&tm_v);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);   // this warp's TMEM lane quadrant
    uint32_t ph_mma = 0, ph_in = 0, ph_v = 0;
    int n_in = 0, n_v = 0, n_commit = 0;   // thread 0: arms of bar_in, bar_v and MMA commits

    auto issue_inputs = [&](int ci) {   // thread 0 only
        const int z = (int)(t0 + (long long)ci * C);
        ++n_in;
        ptx::mbar_arrive_expect_tx(bar_in, (uint32_t)(GS ? L::IN_BYTES / 2 : L::IN_BYTES));
        ptx::tma_load_3d(sb + L::QIN, &tm_q, bar_in, 0, h, z);
        ptx::tma_load_3d(sb + L::KIN, &tm_k, bar_in, 0, h, z);
        if constexpr (!GS) ptx::tma_load_3d(sb + L::GIN, &tm_g, bar_in, 0, h, z);
    };
    auto issue_v = [&](int ci) {        // thread 0 only
        const int z = (int)(t0 + (long long)ci * C);
        ++n_v;
        ptx::mbar_arrive_expect_tx(bar_v, (uint32_t)(C * DVT * 2));
        ptx::tma_load_3d(sb + L::VIN, &tm_v, bar_v, col_base, h, z);
    };

    // state rows held by this thread: row = key channel = TMEM lane
    const int srow = quad * 32 + lane;
    const bool has_row = srow < DK;
    const int scol = half * CPT;
    const int row = state_row(slots, num_slots, n);
    const long long st_off = ((long long)(row < 0 ? 0 : row) * H + h) * DK * DV + col_base + scol;
    float S[CPT];
#pragma unroll
    for (int j = 0; j < CPT; j += 4) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (has_row && init_state && row >= 0) x = load4(init_state + st_off + (long long)srow * DV + j);
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
    }

    bool ok = true;
    for (int ci = 0; ci < nck; ++ci) {
        const long long cs = t0 + (long long)ci * C;
        const int Lc = (int)min((long long)C, t1 - cs);
        const int buf = ci & 1;
        float beta_next = 0.f;
        if (ci + 1 < nck && tid < C) {
            const int Ln = (int)min((long long)C, t1 - cs - C);
            beta_next = tid < Ln ? beta[(cs + C + tid) * H + h] : 0.f;
        }

        // ---- 1. decay factors (one exp per element) -> Kp, Qp, Kbar; e^{G_last} S -> bf16 operand
        if (!(ok = wait_all(bar_in, ph_in))) break;
        float dch = 0.f;   // e^{G_last} of this thread's state row
        {
            const int cg = tid % NCG, seg = tid / NCG, c0 = 4 * cg, i0 = seg * SEGLEN;
            const float *gin = reinterpret_cast<const float *>(sm + L::GIN);
            const uint8_t *qin = sm + L::QIN, *kin = sm + L::KIN;
            float al[SEGLEN][4];
            float4 sg = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int u = 0; u < SEGLEN; ++u) {
                float4 g4 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (i0 + u < Lc) {
                    if constexpr (GS) {
                        const float gs = __ldg(g_scalar + (cs + i0 + u) * H + h);
                        g4 = make_float4(gs, gs, gs, gs);
                    } else {
                        g4 = *reinterpret_cast<const float4 *>(gin + (i0 + u) * DK + c0);
                    }
                }
                sg.x += g4.x; sg.y += g4.y; sg.z += g4.z; sg.w += g4.w;
                al[u][0] = g4.x; al[u][1] = g4.y; al[u][2] = g4.z; al[u][3] = g4.w;
            }
            *reinterpret_cast<float4 *>(fSeg + seg * DK + c0) = sg;
            __syncthreads();
            float pre[4] = {0.f, 0.f, 0.f, 0.f}, tot[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int s2 = 0; s2 < NSEG; ++s2) {
                const float4 x = *reinterpret_cast<const float4 *>(fSeg + s2 * DK + c0);
                const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (s2 < seg) pre[e] += xv[e];
                    tot[e] += xv[e];
                }
            }
            if (seg == 0 && (tot[0] < -80.f || tot[1] < -80.f || tot[2] < -80.f || tot[3] < -80.f))
                flag_status(KDA_DEV_DECAY_RANGE);
            if (has_row) {
                float tr = 0.f;
#pragma unroll
                for (int s2 = 0; s2 < NSEG; ++s2) tr += fSeg[s2 * DK + srow];
                dch = expf(tr);
            }
#pragma unroll
            for (int u = 0; u < SEGLEN; ++u)
#pragma unroll
                for (int e = 0; e < 4; ++e) al[u][e] = exp2_fast(al[u][e] * LOG2E);
            const float sgv[4] = {sg.x, sg.y, sg.z, sg.w};
            // forward: ef = e^{G_i - G_last} (>= 1; bounded by e^80 under the range precondition)
            float ef[4], eb[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                ef[e] = exp2_fast((pre[e] - tot[e]) * LOG2E);
                eb[e] = exp2_fast((tot[e] - pre[e] - sgv[e]) * LOG2E);
            }
#pragma unroll
            for (int u = 0; u < SEGLEN; ++u) {
                const int i = i0 + u;
                float4 q4 = make_float4(0.f, 0.f, 0.f, 0.f), k4 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (i < Lc) {
                    q4 = ld_bf16x4(qin + (i * DK + c0) * 2);
                    k4 = ld_bf16x4(kin + (i * DK + c0) * 2);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) ef[e] *= al[u][e];
                st_bf16x4(sm, L::KQ + sw128(i, c0, 128), k4.x * ef[0], k4.y * ef[1], k4.z * ef[2], k4.w * ef[3]);
                st_bf16x4(sm, L::KQ + sw128(64 + i, c0, 128), q4.x * ef[0], q4.y * ef[1], q4.z * ef[2],
                          q4.w * ef[3]);
            }
            // backward: eb = e^{G_last - G_i} (<= 1)
#pragma unroll
            for (int u = SEGLEN - 1; u >= 0; --u) {
                const int i = i0 + u;
                float4 k4 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (i < Lc) k4 = ld_bf16x4(kin + (i * DK + c0) * 2);
                st_bf16x4(sm, L::KS + sw128(i, c0, L::KSR), k4.x * eb[0], k4.y * eb[1], k4.z * eb[2], k4.w * eb[3]);
#pragma unroll
                for (int e = 0; e < 4; ++e) eb[e] *= al[u][e];
            }
        }
        if (has_row) {
#pragma unroll
            for (int j = 0; j < CPT; ++j) st_bf16(sm, L::KS + sw128(64 + scol + j, srow, L::KSR), dch * S[j]);
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();

        // ---- 2. [Gram | X; Y] = [Kp; Qp] [Kbar; e^{G_last} S^T]^T in one N = 64 + DVT MMA chain
        if (tid == 0) {
            ptx::tc_fence_after();
            constexpr uint32_t ig = ptx::idesc_bf16_f32(128, 64 + DVT);
#pragma unroll
            for (int s = 0; s < DK / 16; ++s)
                ptx::mma_bf16(tmem + COL_GRAM, kdesc(sb + L::KQ, s, 128), kdesc(sb + L::KS, s, L::KSR), ig, s > 0);
            ptx::mma_commit(bar_mma);
            ++n_commit;
        }
        if (!(ok = wait_all(bar_mma, ph_mma))) break;

        // ---- 3. Gram -> Diag(beta) Akk (fp32) -> diagonal blocks of T (warps 0-1);
        //        masked Aqk -> bf16 (warps 2-3); Z = V - X (warps 4-5); zero blocks of T (6-7)
        if (warp < 2) {
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                float g32[32];
                ptx::tmem_ld32(tl + COL_GRAM + hh * 32, g32);
                ptx::tmem_wait_ld();
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
            }
            asm volatile("bar.sync 1, 64;" ::: "memory");   // rows of A from both warps
            invert_diag_blocks(fA, fT, sm + L::TB, fB + buf * C, tid);
        } else if (warp < 4) {
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                float g32[32];
                ptx::tmem_ld32(tl + COL_GRAM + hh * 32, g32);
                ptx::tmem_wait_ld();
                const int i = tid - 64;
#pragma unroll
                for (int u = 0; u < 32; ++u) g32[u] = (hh * 32 + u <= i) ? g32[u] : 0.f;
#pragma unroll
                for (int gq = 0; gq < 4; ++gq)
                    st_bf16x8(sm, L::KP + sw128_chunk(DK + i, hh * 4 + gq), g32 + gq * 8);
            }
        } else if (warp < 6) {
            // X rows (TMEM lanes 0-63) -> Z = V - X -> Z^T
            if (!ptx::mbar_wait_bounded(bar_v, ph_v, WAIT_LIMIT_CYCLES)) *fail_flag = 1;
            const int j = quad * 32 + lane;
            const uint8_t *vin = sm + L::VIN;
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
        } else {
            // blocks (0,1) and (2,3) of T are read by the merge products as zeros;
            // Tb^T is zero below its block diagonal (six 16 x 16 blocks, 16-byte stores)
            const int t = tid - 192;
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int e = t + 64 * m, blk = e >> 8, r = (e >> 4) & 15, c = e & 15;
                fT[(32 * blk + r) * AS + 32 * blk + 16 + c] = 0.f;
            }
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int m = 0; m < 3; ++m) {
                const int e = t + 64 * m;                  // 0..191: 6 blocks x 16 rows x 2 groups
                const int blk = e >> 5, r = (e >> 1) & 15, gh = e & 1;
                const int bi = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);   // row block of Tb^T
                const int bj = blk < 3 ? 0 : (blk < 5 ? 1 : 2);               // column block (< bi)
                *reinterpret_cast<uint4 *>(sm + L::TB + sw128_chunk(16 * bi + r, 2 * bj + gh)) = z;
            }
        }
        ph_v ^= 1u;
        __syncthreads();
        if (tid == 0 && ci + 1 < nck && !*fail_flag) issue_v(ci + 1);   // V tile consumed
        invert_merge_blocks(fA, fT, fM, sm + L::TB, fB + buf * C, warp, lane);
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();

        // ---- 4. Kt = Kbar^T Tb (Kbar read MN-major), Pt = Aqk Tb ; next chunk's inputs
        if (tid == 0) {
            if (ci + 1 < nck) issue_inputs(ci + 1);
            ptx::tc_fence_after();
            constexpr uint32_t ikt = ptx::idesc_bf16_f32(128, 64, true, false);
            constexpr uint32_t ipt = ptx::idesc_bf16_f32(128, 64);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                ptx::mma_bf16(tmem + COL_KT, ptx::desc_mnmajor_sw128(sb + L::KS + s * 2048, L::KSR * 128, 1024),
                              kdesc(sb + L::TB, s, 64), ikt, s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                ptx::mma_bf16(tmem + COL_PT, kdesc(sb + L::KP, s, DK + 64, DK - 64), kdesc(sb + L::TB, s, 64), ipt,
                              s > 0);
            ptx::mma_commit(bar_mma);
            ++n_commit;
        }
        if (!(ok = wait_all(bar_mma, ph_mma, *fail_flag))) break;

        // ---- 5. Kt, Pt -> bf16 A operands
        if (warp < DK / 32) {
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                float k32[32];
                ptx::tmem_ld32(tl + COL_KT + hh * 32, k32);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int gq = 0; gq < 4; ++gq) st_bf16x8(sm, L::KP + sw128_chunk(srow, hh * 4 + gq), k32 + gq * 8);
            }
        } else if (warp >= 6) {
            const int i = (quad - 2) * 32 + lane;
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                float p32[32];
                ptx::tmem_ld32(tl + COL_PT + hh * 32, p32);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int gq = 0; gq < 4; ++gq) st_bf16x8(sm, L::KP + sw128_chunk(DK + i, hh * 4 + gq), p32 + gq * 8);
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();

        // ---- 6. dS = Kt Z ; O = Y + Pt Z (accumulated onto the Y rows of [X; Y])
        if (tid == 0) {
            ptx::tc_fence_after();
            constexpr uint32_t iz = ptx::idesc_bf16_f32(128, DVT);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                ptx::mma_bf16(tmem + COL_DS, kdesc(sb + L::KP, s, DK + 64), kdesc(sb + L::ZT, s, DVT), iz, s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                ptx::mma_bf16(tmem + COL_XY, kdesc(sb + L::KP, s, DK + 64, DK - 64), kdesc(sb + L::ZT, s, DVT), iz, 1);
            ptx::mma_commit(bar_mma);
            ++n_commit;
        }
        if (!(ok = wait_all(bar_mma, ph_mma))) break;

        // ---- 7. S <- Diag(e^{G_last}) S + dS ; store O rows (TMEM lanes 64-127)
        if (has_row) {
#pragma unroll
            for (int cc = 0; cc < CPT / 16; ++cc) {
                float d16[16];
                ptx::tmem_ld16(tl + COL_DS + scol + cc * 16, d16);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 16; ++u) S[cc * 16 + u] = fmaf(dch, S[cc * 16 + u], d16[u]);
            }
        }
        if (quad >= 2) {
            const int i = (quad - 2) * 32 + lane;
#pragma unroll 1
            for (int cc = 0; cc < CPT / 16; ++cc) {
                float o16[16];
                ptx::tmem_ld16(tl + COL_XY + scol + cc * 16, o16);
                ptx::tmem_wait_ld();
                if (i < Lc) {
                    __nv_bfloat16 *dst = o + ((cs + i) * H + h) * DV + col_base + scol + cc * 16;
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

    if (!ok && tid == 0) {   // a wait timed out: let the copies and MMAs in flight land (bounded), then leave
        if (n_in > 0) ptx::mbar_wait_bounded(bar_in, (uint32_t)((n_in - 1) & 1), WAIT_LIMIT_CYCLES);
        if (n_v > 0) ptx::mbar_wait_bounded(bar_v, (uint32_t)((n_v - 1) & 1), WAIT_LIMIT_CYCLES);
        if (n_commit > 0) ptx::mbar_wait_bounded(bar_mma, (uint32_t)((n_commit - 1) & 1), WAIT_LIMIT_CYCLES);
    }
    __syncthreads();
    if (ok && final_state && has_row && row >= 0) {
#pragma unroll
        for (int j = 0; j < CPT; j += 4)
            store4(final_state + st_off + (long long)srow * DV + j, make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]));
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, TMEM_COLS);
    }
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

template <int DK, int DVT, bool GS>
int launch_t(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
             const float *init_state, void *o, float *final_state, const int32_t *cu_seqlens, long long tokens,
             int T, int H, int dv, int num_seqs, const int32_t *slots, int num_slots, cudaStream_t st, char *msg,
             size_t msg_len) {
    CUtensorMap tq, tk, tg, tv;
    if (!make_tmap(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, DK, DK) ||
        !make_tmap(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, DK, DK) ||
        (!GS && !make_tmap(&tg, log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, tokens, H, DK, DK)) ||
        !make_tmap(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, dv, DVT)) {
        snprintf(msg, msg_len, "building TMA descriptors failed (driver entry point cuTensorMapEncodeTiled)");
        return KDA_ERR_CUDA;
    }
    if (GS) tg = tq;   // unused: the scalar gate is read directly
    constexpr int smem = Layout<DK, DVT>::ALLOC;
    auto kern = chunk_tc_kernel<DK, DVT, GS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) {
        snprintf(msg, msg_len, "cudaFuncSetAttribute(chunk_tc): %s", cudaGetErrorString(e));
        return KDA_ERR_CUDA;
    }
    dim3 grid(dv / DVT, H, num_seqs);
    kern<<<grid, NT, smem, st>>>(tq, tk, tg, tv, beta, init_state, (__nv_bfloat16 *)o, final_state, cu_seqlens,
                                  T, H, dv, slots, num_slots, GS ? log_alpha : nullptr);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        snprintf(msg, msg_len, "chunk_tc launch: %s", cudaGetErrorString(e));
        return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

// No tokens: the final state is the initial state (or zeros).
inline int state_passthrough(const float *init_state, float *final_state, int num_seqs, int H, int dk, int dv,
                             cudaStream_t st, char *msg, size_t msg_len) {
    if (!final_state) return KDA_OK;
    const size_t bytes = (size_t)num_seqs * H * dk * dv * sizeof(float);
    cudaError_t e = init_state ? cudaMemcpyAsync(final_state, init_state, bytes, cudaMemcpyDeviceToDevice, st)
                               : cudaMemsetAsync(final_state, 0, bytes, st);
    if (e != cudaSuccess) {
        snprintf(msg, msg_len, "state copy: %s", cudaGetErrorString(e));
        return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

inline int launch_fused(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                        const float *init_state, void *o, float *final_state, const int32_t *cu_seqlens,
                        long long tokens, int T, int H, int dk, int dv, int num_seqs, const int32_t *slots,
                        int num_slots, bool gate_scalar, cudaStream_t st, char *msg, size_t msg_len) {
    // Value-tile width: the widest tile (fewest duplicated per-chunk operand
    // builds) that still gives at least two CTAs per SM; else 32 columns.
    const long long chains = (long long)num_seqs * H;
    int dvt = 32;
    for (int cand = dv; cand >= 32; cand /= 2)
        if (chains * (dv / cand) >= 2 * 148) { dvt = cand; break; }
#define KDA_TC(DKv, DVTv)                                                                                      \
    return gate_scalar ? launch_t<DKv, DVTv, true>(q, k, v, log_alpha, beta, init_state, o, final_state,      \
                                                   cu_seqlens, tokens, T, H, dv, num_seqs, slots, num_slots,  \
                                                   st, msg, msg_len)                                          \
                       : launch_t<DKv, DVTv, false>(q, k, v, log_alpha, beta, init_state, o, final_state,     \
                                                    cu_seqlens, tokens, T, H, dv, num_seqs, slots, num_slots, \
                                                    st, msg, msg_len)
    if (dk == 128) {
        if (dvt == 128) KDA_TC(128, 128);
        if (dvt == 64) KDA_TC(128, 64);
        KDA_TC(128, 32);
    }
    if (dvt == 128) KDA_TC(64, 128);
    if (dvt == 64) KDA_TC(64, 64);
    KDA_TC(64, 32);
#undef KDA_TC
}

}  // namespace tc
}  // namespace kda
