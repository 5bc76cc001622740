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
//   Khat = e^G * K, Qhat = e^G * Q, Kbar = e^{G_last - G} * K        (every factor <= 1)
//   Akk = strict_lower(Khat-Gram), Aqk = lower(Qhat-Gram)            (entries sum_c x_ic k_jc e^{G_ic - G_jc})
//   X = Khat S, Y = Qhat S                                          (state-dependent)
//   T = (I + Diag(beta) Akk)^{-1},  Tb = T Diag(beta)               (fp32, shared memory)
//   Kt = Kbar^T Tb,  Pt = Aqk Tb                                    (one MMA pair)
//   Z = V - X
//   S <- Diag(e^{G_last}) S + Kt Z,   O = Y + Pt Z                   (one MMA pair)
// The Gram's pairwise factors e^{G_ic - G_jc} are split into bf16 operands in two
// tiers (see DECAY_LIM below), exact for any log_alpha <= 0.
//
// Mapping: one 256-thread CTA per (value-column tile of DVT, head, sequence) walks
// the sequence's chunks in order.  TMA brings each chunk's q, k, log_alpha and v
// tiles into shared memory, the next chunk's while the current one computes.
// All threads build the decayed bf16 operands (four key channels x one token
// segment each); threads 0..dk-1 keep row c of the fp32 state in registers, which
// is also TMEM lane c of every 128-row accumulator.  Thread 0 issues the MMAs;
// completion is signalled through mbarriers with bounded waits.  bf16 operands
// live in shared memory in the 128-byte-swizzled K-major layout the MMA
// descriptors name.
#pragma once

#include <cuda.h>

#include <algorithm>
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
constexpr uint32_t COL_GRAM = 0;    // [128 x 64]  tier A: rows 0-63 (e^G K)(e^{-G} K)^T, rows 64-127 with Q
constexpr uint32_t COL_XY = 64;     // [128 x DVT] rows 0-63 X, rows 64-127 Y, then O (same MMA as the Gram)
constexpr uint32_t COL_KT = 192;    // [128 x 64]  Kt (lanes 0..dk-1)
constexpr uint32_t COL_PT = 256;    // [128 x 64]  Pt (lanes 64-127)
constexpr uint32_t COL_DS = 320;    // [128 x DVT] Kt Z (lanes 0..dk-1)
constexpr uint32_t COL_BT = 192;    // tier B: block b's Gram [128 x 16 (b+1)] at COL_BT + bt_row0(b) (in KT..DS, free then)
constexpr int AS = 68;              // fp32 row stride of the 64 x 64 scratch matrices (16-byte rows)
constexpr float DECAY_LIM = 80.f;

// First row of block b's operand in the tier-B operand region (tiles of 16 (b + 1)
// rows: 0, 16, 48, 96) -- also its TMEM column offset.
__host__ __device__ constexpr int bt_row0(int b) { return 8 * b * (b + 1); }
constexpr int BT_ROWS = 160;   // bt_row0(4)


template <int DK, int DVT>
struct Layout {
    static constexpr int KA = DK / 64;                       // 64-element K atoms along dk
    // bf16 MMA operands, 128-byte swizzled, 1024-byte aligned
    static constexpr int KQ = 0;                             // [KA][128][128 B] e^G K (0-63), e^G Q (64-127);
                                                             //   tier B: the block-relative rows first
    static constexpr int KB = KQ + KA * 128 * 128;           // [KA][64][128 B] tier A e^{-G} K, tier B Kbar (tokens)
    static constexpr int SB = KB + KA * 64 * 128;            // bf16 S, MN-major (key rows = K, value columns = N)
    static constexpr int RX = SB + DK * DVT * 2;             // Kt/Pt, Tb^T, Z; tier B: block operands B_0..B_3
    static constexpr int KP = RX;                            //   [DK+64][128 B] Kt (0..DK-1), Aqk -> Pt (DK..)
    static constexpr int TB = KP + (DK + 64) * 128;          //   [64][128 B]    Tb^T
    static constexpr int ZT = TB + 64 * 128;                 //   bf16 Z, MN-major (tokens = K, value columns = N)
    static constexpr int RX_USE = ZT + DVT * 128 - RX;
    static constexpr int BT_BYTES = KA * BT_ROWS * 128;
    static constexpr int RX_BYTES = ((RX_USE > BT_BYTES ? RX_USE : BT_BYTES) + 1023) / 1024 * 1024;
    // dense TMA input tiles; the fp32 scratch of the UT transform aliases them
    static constexpr int QIN = RX + RX_BYTES;                // bf16 [64][DK]
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
    static constexpr int BAD = FSEG + NSEG * DK * 4;         // u32 [4][DK/32]  (block, channel) pairs left to diag_fixup
    static constexpr int MISC = BAD + 4 * (DK / 32) * 4;     // mbarriers, TMEM base, flags
    static constexpr int BYTES = MISC + 64;
    static constexpr int ALLOC = BYTES + 1024;               // room to align the base to 1024 B
    static_assert(KQ % 1024 == 0 && KB % 1024 == 0 && SB % 1024 == 0 && KP % 1024 == 0 && TB % 1024 == 0 &&
                      ZT % 1024 == 0 &&
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

// bf16 MN-major operand of DVT columns (N) by `krows` rows (K): rows of 64 bytes
// (32 columns, 64-byte swizzle) at DVT = 32, else 128 bytes (64 columns, 128-byte
// swizzle) per column block; a thread that holds consecutive columns of one row
// writes them as 16-byte groups.
template <int DVT>
struct MnOp {
    static constexpr int RB = DVT >= 64 ? 128 : 64, NB = RB / 2;
    // byte offset of the 16-byte group holding columns n .. n+7 of row k
    static __device__ __forceinline__ uint32_t off(int k, int n, int krows) {
        const int blk = n / NB, g = (n % NB) / 8;
        const int sg = RB == 128 ? (g ^ (k & 7)) : (g ^ ((k >> 1) & 3));
        return (uint32_t)(blk * krows * RB + k * RB + sg * 16);
    }
    // descriptor of K step s (16 rows)
    static __device__ __forceinline__ uint64_t desc(uint32_t addr, int s, int krows) {
        return RB == 128 ? ptx::desc_mnmajor_sw128(addr + s * 16 * RB, krows * RB, 8 * RB)
                         : ptx::desc_mnmajor_sw64(addr + s * 16 * RB, krows * RB, 8 * RB);
    }
};

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
template <bool KEEP_T = false>
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
        // KEEP_T: T[hi][lo] into Tm too (this step reads only columns 32.. of Tm)
        if constexpr (KEEP_T) warp_store16x8(Tm + (32 + 16 * mt) * AS + 8 * nt, AS, d, -1.f, lane);
    }
}

// ------------------------------------------------------------------ exact decay factors
//
// The Gram matrices need e^{G_i - G_j} (i >= j, G the per-channel cumulative log
// decay of the chunk), which is at most 1 but may be as small as the data makes it
// (a channel can forget everything in one token).  It is split into two bf16 MMA
// operands, one factor per side, in one of two tiers chosen per chunk:
//   tier A (every channel's chunk decay >= -DECAY_LIM): rows e^{G_i} x_i (<= 1)
//       against e^{-G_j} k_j (<= e^DECAY_LIM), one product of N = 64;
//   tier B (otherwise): 16-token blocks.  Row i of block b is scaled relative to
//       the block's start, e^{G_i - G_s(b)} x_i (<= 1), against the block's own
//       operand B_b = e^{G_s(b) - G_j} k_j for j < 16 (b + 1): <= 1 for earlier
//       blocks; inside block b the factor is e^{in-block decay}, used when that
//       decay is >= -DECAY_LIM, and otherwise (a (block, channel) "bad" pair)
//       the channel is left out of B_b and its 16 x 16 diagonal terms are added
//       exactly in fp32 from running products of alpha (diag_fixup).
// Every operand factor stays within e^{+-DECAY_LIM} (bf16 and fp32 reach e^88).
// Byte offset of block b's operand tile ([KA][16 (b + 1)][128 B]) in the region.
__device__ __forceinline__ uint32_t bt_off(int b, int KA) { return (uint32_t)(KA * 128 * bt_row0(b)); }

// Tier-B Gram readout: 32 columns [32 hh, 32 hh + 32) of this lane's row r (0..63
// within the k or the q rows), taken from the accumulator of the row's own 16-row
// block.  The accumulator of block b sits at TMEM column col0 + bt_row0(b) and is
// 16 (b + 1) wide; columns beyond it read a neighbour, but lie above the diagonal
// and are masked by the caller.  quad: the warp's TMEM lane quadrant.
__device__ __forceinline__ void gram_tier_b_ld32(uint32_t tl, uint32_t col0, int quad, int hh, int r,
                                                 float (&v)[32]) {
    const int bl = (quad & 1) * 2;   // the warp's rows cover blocks bl and bl + 1
    if (hh == 1 && bl == 0) {        // rows 0..31: columns 32.. are above the diagonal
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] = 0.f;
        return;
    }
    const bool lo = (r >> 4) == bl;
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        float a[16], c[16];
        ptx::tmem_ld16(tl + col0 + bt_row0(bl) + 32 * hh + 16 * p, a);
        ptx::tmem_ld16(tl + col0 + bt_row0(bl + 1) + 32 * hh + 16 * p, c);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; ++u) v[16 * p + u] = lo ? a[u] : c[u];
    }
}

// Adds fx (this lane's exact terms for columns 16 rb .. 16 rb + 15) into the
// diagonal columns of its block's tier-B accumulator.  Warp-collective: the warp's
// lanes cover blocks bl and bl + 1, so both column ranges are read and written back.
__device__ __forceinline__ void diag_add(uint32_t tl, uint32_t col0, int quad, int rb, const float (&fx)[16]) {
    const int bl = (quad & 1) * 2;
    const uint32_t ca = tl + col0 + bt_row0(bl) + 16 * bl, cb = tl + col0 + bt_row0(bl + 1) + 16 * (bl + 1);
    float va[16], vb[16];
    ptx::tmem_ld16(ca, va);
    ptx::tmem_ld16(cb, vb);
    ptx::tmem_wait_ld();
    uint32_t ua[16], ub[16];
    const bool lo = rb == bl;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        ua[u] = __float_as_uint(lo ? va[u] + fx[u] : va[u]);
        ub[u] = __float_as_uint(lo ? vb[u] : vb[u] + fx[u]);
    }
    ptx::tmem_st16(ca, ua);
    ptx::tmem_st16(cb, ub);
    ptx::tmem_wait_st();
}

// Exact diagonal-block terms of the channels left out of a tier-B operand: for
// row i of block b and each channel c set in mask (NW words), for j = 16 b .. i,
//   fx[j - 16 b] += x_ic k_jc prod_{t = j+1..i} alpha_tc
// accumulated in fp32 from running products.  alpha(t, c), kv(t, c) and xv(c)
// read the chunk's inputs (k and x zero, alpha anything, past the chunk end).
template <int NW, class FA, class FK, class FX>
__device__ __forceinline__ void diag_fixup(float (&fx)[16], const uint32_t *mask, int b, int i, FA alpha, FK kv,
                                           FX xv) {
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) fx[jj] = 0.f;
    const int j0 = 16 * b, il = i - j0;
#pragma unroll 1
    for (int w = 0; w < NW; ++w) {
        uint32_t m = mask[w];
#pragma unroll 1
        while (m) {
            const int c = 32 * w + __ffs(m) - 1;
            m &= m - 1;
            const float x = xv(c);
            float P = 1.f;
#pragma unroll
            for (int hb = 1; hb >= 0; --hb) {   // j from i down to 16 b, eight at a time
                float a[8], kk[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const bool on = 8 * hb + jj <= il;
                    a[jj] = on ? alpha(j0 + 8 * hb + jj, c) : 0.f;
                    kk[jj] = on ? kv(j0 + 8 * hb + jj, c) : 0.f;
                }
#pragma unroll
                for (int jj = 7; jj >= 0; --jj) {
                    if (8 * hb + jj <= il) {
                        fx[8 * hb + jj] = fmaf(x * kk[jj], P, fx[8 * hb + jj]);
                        P *= a[jj];
                    }
                }
            }
        }
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
    constexpr int SPB = 16 / SEGLEN, NW = DK / 32;
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
    uint32_t *bad = reinterpret_cast<uint32_t *>(sm + L::BAD);
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

        // ---- 1. decay factors (one exp per element) -> the Gram operands (tier A or B), Kbar; S -> bf16 operand
        if (!(ok = wait_all(bar_in, ph_in))) break;
        float dch = 0.f;   // e^{G_last} of this thread's state row
        bool tier_b;
        {
            const int cg = tid % NCG, seg = tid / NCG, c0 = 4 * cg, i0 = seg * SEGLEN, blk = seg / SPB;
            const float *gin = reinterpret_cast<const float *>(sm + L::GIN);
            const uint8_t *qin = sm + L::QIN, *kin = sm + L::KIN;
            float al[SEGLEN][4];
            float4 sg = make_float4(0.f, 0.f, 0.f, 0.f);
            if (tid < 4 * NW) bad[tid] = 0u;
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
            // every segment sum >= -DECAY_LIM / NSEG proves every chunk sum >= -DECAY_LIM (tier A)
            constexpr float SEG_LIM = -DECAY_LIM / NSEG;
            const bool maybe_strong =
                __syncthreads_or(sg.x < SEG_LIM || sg.y < SEG_LIM || sg.z < SEG_LIM || sg.w < SEG_LIM) != 0;
            // pre = G before this segment, tot = G_last, gsb = G before this thread's 16-token block
            float pre[4] = {0.f, 0.f, 0.f, 0.f}, tot[4] = {0.f, 0.f, 0.f, 0.f}, gsb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int s2 = 0; s2 < NSEG; ++s2) {
                const float4 x = *reinterpret_cast<const float4 *>(fSeg + s2 * DK + c0);
                const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (s2 < seg) pre[e] += xv[e];
                    if (s2 < blk * SPB) gsb[e] += xv[e];
                    tot[e] += xv[e];
                }
            }
            auto g_before = [&](int b, float (&gb)[4]) {   // G before block b (b = 4: G_last)
#pragma unroll
                for (int e = 0; e < 4; ++e) gb[e] = 0.f;
#pragma unroll
                for (int s2 = 0; s2 < NSEG; ++s2) {
                    if (s2 >= b * SPB) break;
                    const float4 x = *reinterpret_cast<const float4 *>(fSeg + s2 * DK + c0);
                    gb[0] += x.x; gb[1] += x.y; gb[2] += x.z; gb[3] += x.w;
                }
            };
            const bool strong =
                tot[0] < -DECAY_LIM || tot[1] < -DECAY_LIM || tot[2] < -DECAY_LIM || tot[3] < -DECAY_LIM;
            tier_b = maybe_strong && __syncthreads_or(strong) != 0;   // uniform over the CTA
            if (tier_b && seg == 0) {
#pragma unroll 1
                for (int b = 0; b < 4; ++b) {
                    float ga[4], gz[4];
                    g_before(b, ga);
                    g_before(b + 1, gz);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (gz[e] - ga[e] < -DECAY_LIM) atomicOr(&bad[b * NW + (c0 + e) / 32], 1u << ((c0 + e) & 31));
                }
            }
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
            // forward: rows e^{G_i - ref} [k_i; q_i] (<= 1), ref = 0 (tier A) or the block start (tier B)
            {
                float ef[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) ef[e] = exp2_fast((pre[e] - (tier_b ? gsb[e] : 0.f)) * LOG2E);
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
            }
            // backward: rows e^{ref - G_j} k_j of a tile of `rows` rows (e0 at this segment's end)
            auto store_cols = [&](uint32_t tile, int rows, float (&e0)[4]) {
#pragma unroll
                for (int u = SEGLEN - 1; u >= 0; --u) {
                    const int i = i0 + u;
                    float4 k4 = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (i < Lc) k4 = ld_bf16x4(kin + (i * DK + c0) * 2);
                    st_bf16x4(sm, tile + sw128(i, c0, rows), k4.x * e0[0], k4.y * e0[1], k4.z * e0[2], k4.w * e0[3]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) e0[e] *= al[u][e];
                }
            };
            {
                float eb[4];   // tier A: e^{-G_j} (<= e^{DECAY_LIM}); tier B: Kbar, e^{G_last - G_j} (<= 1)
#pragma unroll
                for (int e = 0; e < 4; ++e) eb[e] = exp2_fast(((tier_b ? tot[e] : 0.f) - pre[e] - sgv[e]) * LOG2E);
                store_cols(L::KB, 64, eb);
            }
            if (tier_b) {
#pragma unroll 1
                for (int b = blk; b < 4; ++b) {   // block b's operand holds tokens j < 16 (b + 1)
                    float ga[4], gz[4], eB[4];
                    g_before(b, ga);
                    g_before(b + 1, gz);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const bool out = b == blk && gz[e] - ga[e] < -DECAY_LIM;   // bad pair: diag_fixup
                        eB[e] = out ? 0.f : exp2_fast(fminf(ga[e] - pre[e] - sgv[e], DECAY_LIM) * LOG2E);
                    }
                    store_cols(L::RX + bt_off(b, DK / 64), 16 * (b + 1), eB);
                }
            }
        }
        if (has_row) {
#pragma unroll
            for (int g = 0; g < CPT / 8; ++g)
                *reinterpret_cast<uint4 *>(sm + L::SB + MnOp<DVT>::off(srow, scol + 8 * g, DK)) =
                    make_uint4(pack_bf16(S[8 * g], S[8 * g + 1]), pack_bf16(S[8 * g + 2], S[8 * g + 3]),
                               pack_bf16(S[8 * g + 4], S[8 * g + 5]), pack_bf16(S[8 * g + 6], S[8 * g + 7]));
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();

        if (!tier_b) {
            // ---- 2. Gram = [e^G K; e^G Q] (e^{-G} K)^T and [X; Y] = [e^G K; e^G Q] S (S MN-major)
            if (tid == 0) {
                ptx::tc_fence_after();
                constexpr uint32_t ig = ptx::idesc_bf16_f32(128, 64);
                constexpr uint32_t ixy = ptx::idesc_bf16_f32(128, DVT, false, true);
#pragma unroll
                for (int s = 0; s < DK / 16; ++s)
                    ptx::mma_bf16(tmem + COL_GRAM, kdesc(sb + L::KQ, s, 128), kdesc(sb + L::KB, s, 64), ig, s > 0);
#pragma unroll
                for (int s = 0; s < DK / 16; ++s)
                    ptx::mma_bf16(tmem + COL_XY, kdesc(sb + L::KQ, s, 128), MnOp<DVT>::desc(sb + L::SB, s, DK), ixy,
                                  s > 0);
                ptx::mma_commit(bar_mma);
                ++n_commit;
            }
            if (!(ok = wait_all(bar_mma, ph_mma))) break;
        } else {
            // ---- 2B. Gram from the block-relative rows and the four block operands, then the
            //          chunk-start rows e^G [K; Q] for [X; Y] = [e^G K; e^G Q] S
            if (tid == 0) {
                ptx::tc_fence_after();
#pragma unroll 1
                for (int b = 0; b < 4; ++b) {
                    const int rows = 16 * (b + 1);
                    const uint32_t ib = ptx::idesc_bf16_f32(128, rows);
#pragma unroll
                    for (int s = 0; s < DK / 16; ++s)
                        ptx::mma_bf16(tmem + COL_BT + bt_row0(b), kdesc(sb + L::KQ, s, 128),
                                      kdesc(sb + L::RX + bt_off(b, DK / 64), s, rows), ib, s > 0);
                }
                ptx::mma_commit(bar_mma);
                ++n_commit;
            }
            if (!(ok = wait_all(bar_mma, ph_mma))) break;
            {
                const int cg = tid % NCG, seg = tid / NCG, c0 = 4 * cg, i0 = seg * SEGLEN;
                const float *gin = reinterpret_cast<const float *>(sm + L::GIN);
                const uint8_t *qin = sm + L::QIN, *kin = sm + L::KIN;
                float ef[4] = {0.f, 0.f, 0.f, 0.f};   // G before this segment, then e^{G_i}
#pragma unroll
                for (int s2 = 0; s2 < NSEG; ++s2) {
                    if (s2 >= seg) break;
                    const float4 x = *reinterpret_cast<const float4 *>(fSeg + s2 * DK + c0);
                    ef[0] += x.x; ef[1] += x.y; ef[2] += x.z; ef[3] += x.w;
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) ef[e] = exp2_fast(ef[e] * LOG2E);
#pragma unroll
                for (int u = 0; u < SEGLEN; ++u) {
                    const int i = i0 + u;
                    float4 q4 = make_float4(0.f, 0.f, 0.f, 0.f), k4 = make_float4(0.f, 0.f, 0.f, 0.f);
                    float4 g4 = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (i < Lc) {
                        q4 = ld_bf16x4(qin + (i * DK + c0) * 2);
                        k4 = ld_bf16x4(kin + (i * DK + c0) * 2);
                        if constexpr (GS) {
                            const float gs = __ldg(g_scalar + (cs + i) * H + h);
                            g4 = make_float4(gs, gs, gs, gs);
                        } else {
                            g4 = *reinterpret_cast<const float4 *>(gin + i * DK + c0);
                        }
                    }
                    ef[0] *= exp2_fast(g4.x * LOG2E); ef[1] *= exp2_fast(g4.y * LOG2E);
                    ef[2] *= exp2_fast(g4.z * LOG2E); ef[3] *= exp2_fast(g4.w * LOG2E);
                    st_bf16x4(sm, L::KQ + sw128(i, c0, 128), k4.x * ef[0], k4.y * ef[1], k4.z * ef[2], k4.w * ef[3]);
                    st_bf16x4(sm, L::KQ + sw128(64 + i, c0, 128), q4.x * ef[0], q4.y * ef[1], q4.z * ef[2],
                              q4.w * ef[3]);
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                ptx::tc_fence_after();
                constexpr uint32_t ixy = ptx::idesc_bf16_f32(128, DVT, false, true);
#pragma unroll
                for (int s = 0; s < DK / 16; ++s)
                    ptx::mma_bf16(tmem + COL_XY, kdesc(sb + L::KQ, s, 128), MnOp<DVT>::desc(sb + L::SB, s, DK), ixy,
                                  s > 0);
                ptx::mma_commit(bar_mma);
                ++n_commit;
            }
            // bad (block, channel) pairs: exact diagonal terms into the Gram accumulator,
            // from the input tiles (still intact: the scratch overwrites them only in step 3)
            if (warp < 4) {
                const int r = tid & 63, rb = r >> 4;
                const uint32_t *mk = bad + rb * NW;
                bool fix = false;
#pragma unroll
                for (int w = 0; w < NW; ++w) fix |= mk[w] != 0u;
                if (__any_sync(0xffffffffu, fix)) {
                    float fx[16];
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) fx[jj] = 0.f;
                    if (fix) {
                        const float *gin = reinterpret_cast<const float *>(sm + L::GIN);
                        const __nv_bfloat16 *qin = reinterpret_cast<const __nv_bfloat16 *>(sm + L::QIN);
                        const __nv_bfloat16 *kin = reinterpret_cast<const __nv_bfloat16 *>(sm + L::KIN);
                        auto kval = [&](int t, int c) -> float { return t < Lc ? __bfloat162float(kin[t * DK + c]) : 0.f; };
                        auto alpha = [&](int t, int c) -> float {
                            if (t >= Lc) return 1.f;
                            float g;
                            if constexpr (GS) g = __ldg(g_scalar + (cs + t) * H + h);
                            else g = gin[t * DK + c];
                            return exp2_fast(g * LOG2E);
                        };
                        auto xval = [&](int c) -> float {
                            if (r >= Lc) return 0.f;
                            return __bfloat162float((warp < 2 ? kin : qin)[r * DK + c]);
                        };
                        diag_fixup<NW>(fx, mk, rb, r, alpha, kval, xval);
                    }
                    diag_add(tl, COL_BT, quad, rb, fx);
                }
            }
            if (!(ok = wait_all(bar_mma, ph_mma))) break;   // [X; Y]; also orders the fixups before step 3
        }

        // ---- 3. Gram -> Diag(beta) Akk (fp32) -> diagonal blocks of T (warps 0-1);
        //        masked Aqk -> bf16 (warps 2-3); Z = V - X (warps 4-5); zero blocks of T (6-7)
        if (warp < 2) {
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                float g32[32];
                if (!tier_b) {
                    ptx::tmem_ld32(tl + COL_GRAM + hh * 32, g32);
                    ptx::tmem_wait_ld();
                } else {
                    gram_tier_b_ld32(tl, COL_BT, quad, hh, tid, g32);
                }
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
                if (!tier_b) {
                    ptx::tmem_ld32(tl + COL_GRAM + hh * 32, g32);
                    ptx::tmem_wait_ld();
                } else {
                    gram_tier_b_ld32(tl, COL_BT, quad, hh, tid - 64, g32);
                }
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
                for (int g = 0; g < 2; ++g)
                    *reinterpret_cast<uint4 *>(sm + L::ZT + MnOp<DVT>::off(j, cc * 16 + 8 * g, C)) = make_uint4(
                        pack_bf16(v16[8 * g] - x16[8 * g], v16[8 * g + 1] - x16[8 * g + 1]),
                        pack_bf16(v16[8 * g + 2] - x16[8 * g + 2], v16[8 * g + 3] - x16[8 * g + 3]),
                        pack_bf16(v16[8 * g + 4] - x16[8 * g + 4], v16[8 * g + 5] - x16[8 * g + 5]),
                        pack_bf16(v16[8 * g + 6] - x16[8 * g + 6], v16[8 * g + 7] - x16[8 * g + 7]));
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
                ptx::mma_bf16(tmem + COL_KT, ptx::desc_mnmajor_sw128(sb + L::KB + s * 2048, 64 * 128, 1024),
                              kdesc(sb + L::TB, s, 64), ikt, s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                ptx::mma_bf16(tmem + COL_PT, kdesc(sb + L::KP, s, DK + 64, DK - 64), kdesc(sb + L::TB, s, 64), ipt,
                              s > 0);
            ptx::mma_commit(bar_mma);
            ++n_commit;
        }
        if (!(ok = wait_all(bar_mma, ph_mma, *fail_flag))) break;

        // ---- 5. Kt, Pt -> bf16 A operands (tier A: Kt rows take the factor e^{G_last})
        if (warp < DK / 32) {
            const float dr = tier_b ? 1.f : dch;
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                float k32[32];
                ptx::tmem_ld32(tl + COL_KT + hh * 32, k32);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 32; ++u) k32[u] *= dr;
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
            constexpr uint32_t iz = ptx::idesc_bf16_f32(128, DVT, false, true);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                ptx::mma_bf16(tmem + COL_DS, kdesc(sb + L::KP, s, DK + 64), MnOp<DVT>::desc(sb + L::ZT, s, C), iz, s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                ptx::mma_bf16(tmem + COL_XY, kdesc(sb + L::KP, s, DK + 64, DK - 64), MnOp<DVT>::desc(sb + L::ZT, s, C), iz,
                              1);
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
                      int H, int inner, int box_inner,
                      CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)H, (cuuint64_t)tokens};
    cuuint64_t strides[2] = {(cuuint64_t)inner * esize, (cuuint64_t)inner * esize * H};
    cuuint32_t box[3] = {(cuuint32_t)box_inner, 1u, (cuuint32_t)C};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
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
