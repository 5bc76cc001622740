// KDA chunked prefill in two passes, for inputs with few (sequence, head) chains.
//
// Same chunk algebra as chunk_tc_kernel (kda_chunk_tc.cuh; "Kimi Linear、独自の土俵で
// Full Attentionを上回る" (remio.ai), § "Kimi Linearがより賢いRecurrent Memoryを使う方法":
// chunkwise algorithm on a diagonal-plus-low-rank transition).  Everything of a
// chunk that does not involve the state -- the decay factors, the Gram matrix, the
// UT transform T = (I + Diag(beta) Akk)^{-1} and the products Kt = Kbar^T Tb,
// Pt = Aqk Tb -- depends on that chunk's inputs alone; its decay factors are exact
// for any log_alpha <= 0 (the two tiers described in kda_chunk_tc.cuh).  The fused
// kernel builds it inside the serial walk over chunks, once per value-column tile.  Here
//
//   pass 1, chunk_intra_kernel: one CTA per (chunk, head), all chunks at once,
//       writes the bf16 operands [e^G K; e^G Q], [Kt; Pt] and e^{G_last} of the chunk to
//       a workspace record laid out byte for byte like the shared-memory tiles the
//       second pass feeds to the tensor cores;
//   pass 2, chunk_inter_kernel: one CTA per (value tile, head, sequence) walks
//       the chunks in order with only the state-dependent work left on the
//       serial path: X; Y = [e^G K; e^G Q] S, Z = V - X,
//       S <- Diag(e^{G_last}) S + Kt Z, O = Y + Pt Z.
//
// Chunk slots: chunk c of sequence n (tokens [t0, t1)) is record
// n + floor(t0 / 64) + c, unique and below ceil(total tokens / 64) + N for any
// token ranges; a dense batch uses t0 = n T.
#pragma once

#include <cstring>

#include "kda_chunk_tc.cuh"

namespace kda {
namespace tc {

// Workspace record of one (chunk slot, head).
template <int DK>
struct Rec {
    static constexpr int KA = DK / 64;
    static constexpr int KQ = 0;                          // [KA][128][128 B]  e^G K (rows 0-63), e^G Q (rows 64-127)
    static constexpr int KP = KA * 128 * 128;             // [DK+64][128 B]    Kt (rows 0..DK-1), Pt (DK..DK+63)
    static constexpr int DCH = KP + (DK + 64) * 128;      // fp32 [DK]         e^{G_last}
    static constexpr int BYTES = (DCH + DK * 4 + 1023) / 1024 * 1024;
};

// What the backward needs of a chunk beyond the record (first pass with BX): bf16
// 64 x 64 tiles, row i of 128 bytes with a 128-byte swizzle, fp32 values rounded once.
struct BwdX {
    static constexpr int AKK = 0;        // Akk[i][j], j < i (zero elsewhere), without beta
    static constexpr int AQK = 8192;     // Aqk[i][j], j <= i (zero above)
    static constexpr int TI = 16384;     // T = (I + Diag(beta) Akk)^{-1}, unit lower (zero above)
    static constexpr int BYTES = 24576;
};

// Backward workspace unit of one (chunk slot, head), dk = dv = 128 (kda_bwd_tc.cuh):
// the record and the extras from the first pass, the state at the chunk's start
// (forward sweep) and its adjoint at the chunk's end (adjoint sweep), both bf16
// [DV/64][DK][128 B] with a 128-byte swizzle.
template <int DK>
struct BwdUnit {
    static constexpr int DV = 128;
    static constexpr int REC = 0;
    static constexpr int BXO = Rec<DK>::BYTES;
    static constexpr int SC = BXO + BwdX::BYTES;
    static constexpr int DSC = SC + DK * DV * 2;
    static constexpr int BYTES = DSC + DK * DV * 2;
    static_assert(BXO % 1024 == 0 && SC % 1024 == 0 && DSC % 1024 == 0 && BYTES % 1024 == 0, "tile alignment");
};

inline long long chunk_slots(long long tokens, int num_seqs) { return (tokens + C - 1) / C + num_seqs; }

// Workspace: the records [slot][H] of the first pass.
inline size_t two_pass_workspace_bytes(long long tokens, int H, int dk, int num_seqs) {
    if (tokens <= 0) return 0;
    const size_t rec = dk == 64 ? (size_t)Rec<64>::BYTES : (size_t)Rec<128>::BYTES;
    return (size_t)chunk_slots(tokens, num_seqs) * (size_t)H * rec;
}

// First token of sequence n (clamped like seq_span).
__device__ __forceinline__ long long seq_begin(const int32_t *cu_seqlens, int T, int n) {
    return cu_seqlens ? (long long)min(max(cu_seqlens[n], 0), T) : (long long)n * T;
}

// ------------------------------------------------------------------ pass 1

// Chunk of `slot`: the last sequence n whose first slot n + floor(t0_n / 64) is
// <= slot owns it.  False for a slot without a chunk (uniform over the CTA).
__device__ __forceinline__ bool slot_chunk(const int32_t *cu_seqlens, int T, int num_seqs, int slot, long long &cs,
                                           int &Lc) {
    int lo = 0, hi = num_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (mid + seq_begin(cu_seqlens, T, mid) / C <= slot) lo = mid;
        else hi = mid - 1;
    }
    long long t0, t1;
    seq_span(cu_seqlens, T, lo, t0, t1);
    cs = t0 + (long long)(slot - (lo + t0 / C)) * C;
    if (cs < t0 || cs >= t1) return false;
    Lc = (int)min((long long)C, t1 - cs);
    return true;
}


template <int DK>
struct IntraLayout {
    static constexpr int KA = DK / 64;
    static constexpr int KQ_BYTES = KA * 128 * 128;
    static constexpr int BT_BYTES = KA * BT_ROWS * 128;
    static constexpr int SCR_BYTES = 2 * 64 * AS * 4 + 32 * 36 * 4;
    static constexpr int RG_BYTES = ((BT_BYTES > SCR_BYTES ? BT_BYTES : SCR_BYTES) + 1023) / 1024 * 1024;
    static constexpr int KQ = 0;                          // [KA][128][128 B] e^G K (rows 0-63), e^G Q (64-127);
                                                          //   tier B: the block-relative rows first
    static constexpr int RG = KQ + KQ_BYTES;              // tier B: block operands B_0..B_3; after the Gram:
    static constexpr int FA = RG;                         //   fp32 [64][AS] Diag(beta) Akk
    static constexpr int FT = FA + 64 * AS * 4;           //   fp32 [64][AS] T
    static constexpr int FM = FT + 64 * AS * 4;           //   fp32 [32][36] block products
    static constexpr int KB = RG + RG_BYTES;              // [KA][64][128 B] tier A: e^{-G} K; tier B: Kbar
    static constexpr int TB = KB + KA * 64 * 128;         // [64][128 B]      Tb^T
    static constexpr int AQ = TB + 64 * 128;              // [64][128 B]      masked Aqk (rows 64-127 of [Tb^T; Aqk])
    static constexpr int FB = AQ + 64 * 128;              // fp32 [64]        beta
    static constexpr int FD = FB + 64 * 4;                // fp32 [DK]        e^{G_last}
    static constexpr int FN = FD + DK * 4;                // fp32 [2][64]     prologue: 1/|q_i|, 1/|k_i|
    static constexpr int NSEG = NT / (DK / 4);
    static constexpr int FSEG = FN + 2 * 64 * 4;          // fp32 [NSEG][DK]  segment sums of log_alpha
    static constexpr int BAD = FSEG + NSEG * DK * 4;      // u32 [4][DK/32]   (block, channel) pairs left to diag_fixup
    static constexpr int MISC = BAD + 4 * (DK / 32) * 4;  // mbarrier, TMEM base
    static constexpr int BYTES = MISC + 64;
    static constexpr int ALLOC = BYTES + 1024;
    static_assert(RG % 1024 == 0 && KB % 1024 == 0 && TB % 1024 == 0 && AQ % 1024 == 0, "tile alignment");
    static_assert(2 * (ALLOC + 1024) <= 233472, "two CTAs per SM");
};

constexpr uint32_t INTRA_TMEM_COLS = 256;
constexpr uint32_t ICOL_GRAM = 0;     // tier A: [128 x 64] rows 0-63 (e^G K)(e^{-G} K)^T, rows 64-127 with Q
constexpr uint32_t ICOL_BT = 64;      // tier B: block b's [128 x 16 (b+1)] at ICOL_BT + bt_row0(b)
constexpr uint32_t ICOL_KT = 64;      // [128 x 64] Kt (lanes 0..dk-1), after the Gram is read
constexpr uint32_t ICOL_PT = 128;     // [128 x 64] Pt (lanes 64-127)

__device__ __forceinline__ float4 scale4(float4 a, float s) { return make_float4(a.x * s, a.y * s, a.z * s, a.w * s); }

__device__ __forceinline__ uint2 float4_to_bf16x4(float4 a) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(a.x, a.y), hi = __floats2bfloat162_rn(a.z, a.w);
    return make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
}

__device__ __forceinline__ float4 bf16x4_to_float4(uint2 r) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&r.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&r.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ void st_global_bf16x8(uint8_t *p, const float *x) {
    *reinterpret_cast<uint4 *>(p) =
        make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
}

// Tier B of the first pass, lanes of warps 0-3 (row r of the k rows, warps 0-1, or of
// the q rows, warps 2-3): the exact diagonal terms of the bad (block, channel) pairs
// of the row's block, read from the inputs in global memory and added into the
// Gram accumulator.  Kept out of line: it runs only for chunks that decay by more
// than e^DECAY_LIM within 16 tokens.
template <int DK, bool GS, bool PRO>
__device__ __noinline__ void intra_fixup(uint32_t tl, int quad, int warp, int r, int Lc, long long cs, int H, int h,
                                         const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                                         const float *__restrict__ log_alpha, const uint32_t *bad, const float *fN) {
    constexpr int NW = DK / 32;
    constexpr float LOG2E = 1.4426950408889634f;
    const int rb = r >> 4;
    const uint32_t *mk = bad + rb * NW;
    bool fix = false;
#pragma unroll
    for (int w = 0; w < NW; ++w) fix |= mk[w] != 0u;
    if (!__any_sync(0xffffffffu, fix)) return;
    float fx[16];
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) fx[jj] = 0.f;
    if (fix) {
        // chunk token t, channel c of a [tokens, H, DK] input: base + t * tstride + c
        const long long tstride = (long long)H * DK, base = (cs * H + h) * DK;
        auto kval = [&](int t, int c) -> float {
            if (t >= Lc) return 0.f;
            const float x = __bfloat162float(k[base + t * tstride + c]);
            if constexpr (PRO) return __bfloat162float(__float2bfloat16_rn(x * fN[64 + t]));
            return x;
        };
        auto alpha = [&](int t, int c) -> float {
            if (t >= Lc) return 1.f;
            float g;
            if constexpr (GS) g = log_alpha[(cs + t) * H + h];
            else if constexpr (PRO)
                g = neg_softplus(__bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(log_alpha)[base + t * tstride + c]));
            else g = log_alpha[base + t * tstride + c];
            return exp2_fast(g * LOG2E);
        };
        auto xval = [&](int c) -> float {
            if (r >= Lc) return 0.f;
            if (warp < 2) return kval(r, c);
            const float x = __bfloat162float(q[base + r * tstride + c]);
            if constexpr (PRO) return __bfloat162float(__float2bfloat16_rn(x * fN[r]));
            return x;
        };
        diag_fixup<NW>(fx, mk, rb, r, alpha, kval, xval);
    }
    diag_add(tl, ICOL_BT, quad, rb, fx);
}

// GS: scalar gate, log_alpha [tokens, H] (Gated DeltaNet).  PRO: fused input
// prologue -- q and k are raw (scaled here to unit norm over the key axis) and
// log_alpha points to the bf16 gate pre-activation x [tokens, H, DK],
// log_alpha = -softplus(x).
// One (chunk slot, head) of the first pass.  TB = false: tier A only -- a chunk
// that needs tier B is left at once (returns 1) for intra_chunk_strong.  TB = true:
// tier B.  All threads of the CTA call it; ph_mma carries the MMA mbarrier phase.
// Returns 0 when done (or the slot has no chunk) and -1 when a bounded wait ran out.
template <int DK, bool GS, bool PRO, bool TB, bool BX>
__device__ __forceinline__ int intra_chunk(int slot, int h, const __nv_bfloat16 *__restrict__ q,
                                           const __nv_bfloat16 *__restrict__ k,
                                           const float *__restrict__ log_alpha, const float *__restrict__ beta,
                                           const int32_t *__restrict__ cu_seqlens, int T, int H, int num_seqs,
                                           uint8_t *__restrict__ ws, uint8_t *sm, uint32_t tmem,
                                           uint32_t &ph_mma) {
    using L = IntraLayout<DK>;
    using R = Rec<DK>;
    constexpr int NCG = DK / 4, NSEG = L::NSEG, SEGLEN = C / NSEG, SPB = 16 / SEGLEN, NW = DK / 32;
    constexpr float LOG2E = 1.4426950408889634f;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;

    // the sequence owning this slot: the last n whose first slot n + floor(t0_n / 64) is <= slot
    int lo = 0, hi = num_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (mid + seq_begin(cu_seqlens, T, mid) / C <= slot) lo = mid;
        else hi = mid - 1;
    }
    long long t0, t1;
    seq_span(cu_seqlens, T, lo, t0, t1);
    const long long cs = t0 + (long long)(slot - (lo + t0 / C)) * C;
    if (cs < t0 || cs >= t1) return 0;   // slot without a chunk
    const int Lc = (int)min((long long)C, t1 - cs);
    const uint32_t sb = ptx::smem_u32(sm);
    float *fA = reinterpret_cast<float *>(sm + L::FA);
    float *fT = reinterpret_cast<float *>(sm + L::FT);
    float *fM = reinterpret_cast<float *>(sm + L::FM);
    float *fB = reinterpret_cast<float *>(sm + L::FB);
    float *fD = reinterpret_cast<float *>(sm + L::FD);
    float *fN = reinterpret_cast<float *>(sm + L::FN);
    float *fSeg = reinterpret_cast<float *>(sm + L::FSEG);
    uint32_t *bad = reinterpret_cast<uint32_t *>(sm + L::BAD);
    const uint32_t bar_mma = sb + L::MISC;
    // BX: ws holds backward units (record, then the extras)
    uint8_t *rec = ws + ((size_t)slot * H + h) * (size_t)(BX ? BwdUnit<DK>::BYTES : R::BYTES);
    uint8_t *xr = rec + BwdUnit<DK>::BXO;

    if (tid < C) fB[tid] = tid < Lc ? beta[(cs + tid) * H + h] : 0.f;
    if (tid < 4 * NW) bad[tid] = 0u;

    // ---- 1. decay factors -> the Gram operands (tier A or B), Kbar, e^{G_last}
    const int cg = tid % NCG, seg = tid / NCG, c0 = 4 * cg, i0 = seg * SEGLEN, blk = seg / SPB;
    float al[SEGLEN][4];
    uint2 qv[SEGLEN], kv[SEGLEN];
    float4 sg = make_float4(0.f, 0.f, 0.f, 0.f);
    {
        // all loads first, unconditionally (rows past Lc read the last valid row
        // and are zeroed afterwards), so every one is in flight before any is used
        float4 gv[SEGLEN];
#pragma unroll
        for (int u = 0; u < SEGLEN; ++u) {
            const long long row = cs + min(i0 + u, Lc - 1);
            const long long off = (row * H + h) * DK + c0;
            if constexpr (GS) {
                const float gs = __ldg(log_alpha + row * H + h);
                gv[u] = make_float4(gs, gs, gs, gs);
            } else if constexpr (PRO) {
                const uint2 xr = __ldcs(reinterpret_cast<const uint2 *>(reinterpret_cast<const __nv_bfloat16 *>(log_alpha) + off));
                gv[u] = make_float4(__uint_as_float(xr.x), __uint_as_float(xr.y), 0.f, 0.f);   // raw bf16 pairs
            } else {
                gv[u] = __ldcs(reinterpret_cast<const float4 *>(log_alpha + off));
            }
            qv[u] = __ldcs(reinterpret_cast<const uint2 *>(q + off));
            kv[u] = __ldcs(reinterpret_cast<const uint2 *>(k + off));
        }
#pragma unroll
        for (int u = 0; u < SEGLEN; ++u) {
            float4 g4 = gv[u];
            if constexpr (PRO) {
                const float4 x4 = bf16x4_to_float4(make_uint2(__float_as_uint(g4.x), __float_as_uint(g4.y)));
                g4 = make_float4(neg_softplus(x4.x), neg_softplus(x4.y), neg_softplus(x4.z), neg_softplus(x4.w));
            }
            if (i0 + u >= Lc) {
                g4 = make_float4(0.f, 0.f, 0.f, 0.f);
                qv[u] = make_uint2(0u, 0u);
                kv[u] = make_uint2(0u, 0u);
            }
            sg.x += g4.x; sg.y += g4.y; sg.z += g4.z; sg.w += g4.w;
            al[u][0] = g4.x; al[u][1] = g4.y; al[u][2] = g4.z; al[u][3] = g4.w;
        }
    }
    // prologue: q and k rows to unit norm (a row's DK channels live in NCG
    // consecutive lanes of one warp), rounded back to bf16 -- the same values as
    // normalising in fp32 and then casting, as prepared inputs are made
    if constexpr (PRO) {
#pragma unroll
        for (int u = 0; u < SEGLEN; ++u) {
            const float4 a = bf16x4_to_float4(qv[u]), b = bf16x4_to_float4(kv[u]);
            float sq = a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
            float sk = b.x * b.x + b.y * b.y + b.z * b.z + b.w * b.w;
#pragma unroll
            for (int o = NCG / 2; o > 0; o >>= 1) {
                sq += __shfl_xor_sync(0xffffffffu, sq, o);
                sk += __shfl_xor_sync(0xffffffffu, sk, o);
            }
            const float iq = inv_row_norm(sq), ik = inv_row_norm(sk);
            if (cg == 0) {
                fN[i0 + u] = iq;
                fN[64 + i0 + u] = ik;
            }
            qv[u] = float4_to_bf16x4(scale4(a, iq));
            kv[u] = float4_to_bf16x4(scale4(b, ik));
        }
    }
    *reinterpret_cast<float4 *>(fSeg + seg * DK + c0) = sg;
    // every segment sum >= -DECAY_LIM / NSEG proves every chunk sum >= -DECAY_LIM (tier A)
    constexpr float SEG_LIM = -DECAY_LIM / NSEG;
    const bool maybe_strong = __syncthreads_or(sg.x < SEG_LIM || sg.y < SEG_LIM || sg.z < SEG_LIM || sg.w < SEG_LIM) != 0;
    // prefix sums over the segments: pre = G before this segment, tot = G_last,
    // gsb = G before this thread's own 16-token block
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
    // G before block b (b = 0..4; G_last at 4) for this thread's channels, from the segment sums
    auto g_before = [&](int b, float (&gb)[4]) {
#pragma unroll
        for (int e = 0; e < 4; ++e) gb[e] = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < NSEG; ++s2) {
            if (s2 >= b * SPB) break;
            const float4 x = *reinterpret_cast<const float4 *>(fSeg + s2 * DK + c0);
            gb[0] += x.x; gb[1] += x.y; gb[2] += x.z; gb[3] += x.w;
        }
    };
    constexpr bool tier_b = TB;
    if constexpr (!TB) {
        if (maybe_strong) {
            const bool strong =
                tot[0] < -DECAY_LIM || tot[1] < -DECAY_LIM || tot[2] < -DECAY_LIM || tot[3] < -DECAY_LIM;
            if (__syncthreads_or(strong)) return 1;   // uniform over the CTA: tier B
        }
    }
    const float sgv[4] = {sg.x, sg.y, sg.z, sg.w};
    if (seg == 0) {
        const float4 d4 = make_float4(expf(tot[0]), expf(tot[1]), expf(tot[2]), expf(tot[3]));
        *reinterpret_cast<float4 *>(rec + R::DCH + c0 * 4) = d4;
        *reinterpret_cast<float4 *>(fD + c0) = d4;
        if (tier_b) {
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
    }
#pragma unroll
    for (int u = 0; u < SEGLEN; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) al[u][e] = exp2_fast(al[u][e] * LOG2E);

    // rows e^{G_i - ref} x_i (<= 1) of the A operand; ref = 0 (tier A / the record) or the block start (tier B)
    // rows e^{G_i - ref} x_i: ref = 0 into the A tile (tier A, the record's image) or
    // the block start (tier B); to_rec: ref = 0 straight into the workspace record
    // (tier B, whose A tile holds the block-relative rows)
    auto store_rows = [&](bool rel_block, bool to_rec) {
        float ef[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) ef[e] = exp2_fast((pre[e] - (rel_block ? gsb[e] : 0.f)) * LOG2E);
#pragma unroll
        for (int u = 0; u < SEGLEN; ++u) {
            const int i = i0 + u;
            const float4 q4 = bf16x4_to_float4(qv[u]);
            const float4 k4 = bf16x4_to_float4(kv[u]);
#pragma unroll
            for (int e = 0; e < 4; ++e) ef[e] *= al[u][e];
            const uint2 kr = make_uint2(pack_bf16(k4.x * ef[0], k4.y * ef[1]), pack_bf16(k4.z * ef[2], k4.w * ef[3]));
            const uint2 qr = make_uint2(pack_bf16(q4.x * ef[0], q4.y * ef[1]), pack_bf16(q4.z * ef[2], q4.w * ef[3]));
            uint8_t *dst = to_rec ? rec + R::KQ : sm + L::KQ;
            *reinterpret_cast<uint2 *>(dst + sw128(i, c0, 128)) = kr;
            *reinterpret_cast<uint2 *>(dst + sw128(64 + i, c0, 128)) = qr;
        }
    };
    // rows e^{ref - G_j} k_j, j in this segment, into a 64-column-atom tile of `rows` rows;
    // e0 = e^{ref - G at the segment end} per channel, multiplied by alpha going back
    auto store_cols = [&](uint32_t tile, int rows, float (&e0)[4]) {
#pragma unroll
        for (int u = SEGLEN - 1; u >= 0; --u) {
            const int i = i0 + u;
            const float4 k4 = bf16x4_to_float4(kv[u]);
            st_bf16x4(sm, tile + sw128(i, c0, rows), k4.x * e0[0], k4.y * e0[1], k4.z * e0[2], k4.w * e0[3]);
#pragma unroll
            for (int e = 0; e < 4; ++e) e0[e] *= al[u][e];
        }
    };
    if constexpr (!TB) {
        store_rows(false, false);
        float er[4];   // e^{-G_j}: at most e^{DECAY_LIM} in a tier-A chunk
#pragma unroll
        for (int e = 0; e < 4; ++e) er[e] = exp2_fast(-(pre[e] + sgv[e]) * LOG2E);
        store_cols(L::KB, 64, er);
    } else {
        store_rows(true, false);
        store_rows(false, true);
        float eb[4];   // Kbar: e^{G_last - G_j} <= 1
#pragma unroll
        for (int e = 0; e < 4; ++e) eb[e] = exp2_fast((tot[e] - pre[e] - sgv[e]) * LOG2E);
        store_cols(L::KB, 64, eb);
#pragma unroll 1
        for (int b = blk; b < 4; ++b) {   // block b's operand holds tokens j < 16 (b + 1)
            float ga[4], gz[4], eB[4];    // e^{G_s(b) - G_j}: <= 1 before block b, <= e^{DECAY_LIM} inside it
            g_before(b, ga);
            g_before(b + 1, gz);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const bool out = b == blk && gz[e] - ga[e] < -DECAY_LIM;   // bad pair: left to diag_fixup
                eB[e] = out ? 0.f : exp2_fast(fminf(ga[e] - pre[e] - sgv[e], DECAY_LIM) * LOG2E);
            }
            store_cols(L::RG + bt_off(b, DK / 64), 16 * (b + 1), eB);
        }
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);

    // ---- 2. Gram; in tier A the tile is the record's e^G K / e^G Q image, stored meanwhile
    if (tid == 0) {
        if constexpr (!TB) {
            ptx::bulk_store(rec + R::KQ, sb + L::KQ, (uint32_t)L::KQ_BYTES);
            ptx::bulk_commit();
            constexpr uint32_t ig = ptx::idesc_bf16_f32(128, 64);
#pragma unroll
            for (int s = 0; s < DK / 16; ++s)
                ptx::mma_bf16(tmem + ICOL_GRAM, kdesc(sb + L::KQ, s, 128), kdesc(sb + L::KB, s, 64), ig, s > 0);
        } else {
#pragma unroll 1
            for (int b = 0; b < 4; ++b) {
                const int rows = 16 * (b + 1);
                const uint32_t ib = ptx::idesc_bf16_f32(128, rows);
#pragma unroll
                for (int s = 0; s < DK / 16; ++s)
                    ptx::mma_bf16(tmem + ICOL_BT + bt_row0(b), kdesc(sb + L::KQ, s, 128),
                                  kdesc(sb + L::RG + bt_off(b, DK / 64), s, rows), ib, s > 0);
            }
        }
        ptx::mma_commit(bar_mma);
    }
    bool ok = wait_all(bar_mma, ph_mma);

    if (ok) {
        // ---- 3. Diag(beta) Akk -> diagonal blocks of T (warps 0-1); masked Aqk (warps 2-3);
        //         zero blocks of T and Tb^T (warps 6-7)
        if (warp < 4) {
            const int r = tid & 63, rb = r >> 4;   // token row of this lane, its 16-row block
            if constexpr (TB) intra_fixup<DK, GS, PRO>(tl, quad, warp, r, Lc, cs, H, h, q, k, log_alpha, bad, fN);
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                float g32[32];
                if constexpr (!TB) {
                    ptx::tmem_ld32(tl + ICOL_GRAM + hh * 32, g32);
                    ptx::tmem_wait_ld();
                } else {
                    gram_tier_b_ld32(tl, ICOL_BT, quad, hh, r, g32);
                }
                if (warp < 2) {
                    const int i = r;
                    const float bi = fB[i];
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
                    if constexpr (BX) {
#pragma unroll
                        for (int u = 0; u < 32; ++u) g32[u] = (hh * 32 + u < i) ? g32[u] : 0.f;
#pragma unroll
                        for (int gq = 0; gq < 4; ++gq)
                            st_global_bf16x8(xr + BwdX::AKK + sw128_chunk(i, hh * 4 + gq), g32 + gq * 8);
                    }
                } else {
                    const int i = r;
#pragma unroll
                    for (int u = 0; u < 32; ++u) g32[u] = (hh * 32 + u <= i) ? g32[u] : 0.f;
#pragma unroll
                    for (int gq = 0; gq < 4; ++gq) st_bf16x8(sm, L::AQ + sw128_chunk(i, hh * 4 + gq), g32 + gq * 8);
                    if constexpr (BX) {
#pragma unroll
                        for (int gq = 0; gq < 4; ++gq)
                            st_global_bf16x8(xr + BwdX::AQK + sw128_chunk(i, hh * 4 + gq), g32 + gq * 8);
                    }
                }
            }
            if (warp < 2) {
                asm volatile("bar.sync 1, 64;" ::: "memory");
                invert_diag_blocks(fA, fT, sm + L::TB, fB, tid);
            }
        } else if (warp >= 6) {
            const int t = tid - 192;
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int e = t + 64 * m, blk2 = e >> 8, r = (e >> 4) & 15, c = e & 15;
                fT[(32 * blk2 + r) * AS + 32 * blk2 + 16 + c] = 0.f;
            }
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int m = 0; m < 3; ++m) {
                const int e = t + 64 * m;
                const int blk2 = e >> 5, r = (e >> 1) & 15, gh = e & 1;
                const int bi = blk2 < 3 ? blk2 + 1 : (blk2 < 5 ? blk2 - 1 : 3);
                const int bj = blk2 < 3 ? 0 : (blk2 < 5 ? 1 : 2);
                *reinterpret_cast<uint4 *>(sm + L::TB + sw128_chunk(16 * bi + r, 2 * bj + gh)) = z;
            }
        }
        __syncthreads();
        invert_merge_blocks<BX>(fA, fT, fM, sm + L::TB, fB, warp, lane);
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();

        // ---- 4. Kt = (KB tile)^T Tb (read MN-major); Pt = Aqk Tb from the M = 128 operand [Tb^T; Aqk]
        if (tid == 0) {
            ptx::tc_fence_after();
            constexpr uint32_t ikt = ptx::idesc_bf16_f32(128, 64, true, false);
            constexpr uint32_t ipt = ptx::idesc_bf16_f32(128, 64);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                ptx::mma_bf16(tmem + ICOL_KT, ptx::desc_mnmajor_sw128(sb + L::KB + s * 2048, 64 * 128, 1024),
                              kdesc(sb + L::TB, s, 64), ikt, s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                ptx::mma_bf16(tmem + ICOL_PT, kdesc(sb + L::TB, s, 128), kdesc(sb + L::TB, s, 64), ipt, s > 0);
            ptx::mma_commit(bar_mma);
        }
        if constexpr (BX) {   // T rows while the products run: 16 columns per thread
            const int row = tid >> 2;
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
                const int g8 = (tid & 3) * 2 + gg;
                float t8[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) t8[u] = (8 * g8 + u <= row) ? fT[row * AS + 8 * g8 + u] : 0.f;
                st_global_bf16x8(xr + BwdX::TI + sw128_chunk(row, g8), t8);
            }
        }
        ok = wait_all(bar_mma, ph_mma);
    }

    if (ok) {
        // ---- 5. Kt, Pt -> bf16 images in the record (each thread one 64-byte half row);
        //         tier A's KB tile is e^{-G} K, so its Kt rows take the factor e^{G_last}
        uint8_t *kp = rec + R::KP;
        if (quad < DK / 32) {
            float x[32];
            ptx::tmem_ld32(tl + ICOL_KT + half * 32, x);
            ptx::tmem_wait_ld();
            const int row = quad * 32 + lane;
            if constexpr (!TB) {
                const float dr = fD[row];
#pragma unroll
                for (int u = 0; u < 32; ++u) x[u] *= dr;
            }
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) st_global_bf16x8(kp + sw128_chunk(row, half * 4 + gq), x + gq * 8);
        }
        if (quad >= 2) {
            float x[32];
            ptx::tmem_ld32(tl + ICOL_PT + half * 32, x);
            ptx::tmem_wait_ld();
            const int row = DK + (quad - 2) * 32 + lane;
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) st_global_bf16x8(kp + sw128_chunk(row, half * 4 + gq), x + gq * 8);
        }
    }
    if (tid == 0) {
        if (!ok) ptx::mbar_wait_bounded(bar_mma, ph_mma ^ 1u, WAIT_LIMIT_CYCLES);   // MMAs still in flight
        ptx::bulk_wait_all();
    }
    return ok ? 0 : -1;
}

// Tier B of one chunk, kept out of line so that its code does not weigh on the
// register allocation of the common (tier-A) path.
template <int DK, bool GS, bool PRO, bool BX>
__device__ __noinline__ int intra_chunk_strong(int slot, int h, const __nv_bfloat16 *__restrict__ q,
                                               const __nv_bfloat16 *__restrict__ k,
                                               const float *__restrict__ log_alpha, const float *__restrict__ beta,
                                               const int32_t *__restrict__ cu_seqlens, int T, int H, int num_seqs,
                                               uint8_t *__restrict__ ws, uint8_t *sm, uint32_t tmem,
                                               uint32_t *ph_mma) {
    uint32_t ph = *ph_mma;
    const int r = intra_chunk<DK, GS, PRO, true, BX>(slot, h, q, k, log_alpha, beta, cu_seqlens, T, H, num_seqs, ws,
                                                     sm, tmem, ph);
    *ph_mma = ph;
    return r;
}

// First pass: persistent, two CTAs per SM taking (chunk slot, head) items in turn
// (slot fastest); tier A inline, tier B out of line.  While an item runs, thread 0
// prefetches the next item's q, k and gate rows into L2 (tensor-map prefetches; no
// completion is awaited), so its loads find them there.  tm_g covers the
// per-channel gate (fp32 log_alpha, or the bf16 pre-activation with PRO); the
// scalar gate of GS is not prefetched.
// BX (the backward): ws holds [slot][H] BwdUnit; the extras go beside each record.
template <int DK, bool GS, bool PRO, bool BX = false>
__global__ void __launch_bounds__(NT, 2)
chunk_intra_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_g, const __nv_bfloat16 *__restrict__ q,
                   const __nv_bfloat16 *__restrict__ k, const float *__restrict__ log_alpha,
                   const float *__restrict__ beta, const int32_t *__restrict__ cu_seqlens, int T, int H, int num_seqs,
                   int nslots, uint8_t *__restrict__ ws) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t bar_mma = ptx::smem_u32(sm) + IntraLayout<DK>::MISC;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + IntraLayout<DK>::MISC + 8);
    if ((threadIdx.x >> 5) == 0) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), INTRA_TMEM_COLS);
        ptx::tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        ptx::mbar_init(bar_mma, 1);
        ptx::fence_mbar_init();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint32_t ph_mma = 0;
    const int n_items = nslots * H;
    for (int it = (int)blockIdx.x; it < n_items; it += (int)gridDim.x) {
        if (threadIdx.x == 0 && it + (int)gridDim.x < n_items) {
            const int nx = it + (int)gridDim.x, ns = nx % nslots, nh = nx / nslots;
            long long ncs;
            int nLc;
            if (slot_chunk(cu_seqlens, T, num_seqs, ns, ncs, nLc)) {
                ptx::tma_prefetch_l2_3d(&tm_q, 0, nh, (int)ncs);
                ptx::tma_prefetch_l2_3d(&tm_k, 0, nh, (int)ncs);
                if constexpr (!GS) ptx::tma_prefetch_l2_3d(&tm_g, 0, nh, (int)ncs);
            }
        }
        const int slot = it % nslots, h = it / nslots;
        const int r = intra_chunk<DK, GS, PRO, false, BX>(slot, h, q, k, log_alpha, beta, cu_seqlens, T, H,
                                                          num_seqs, ws, sm, tmem, ph_mma);
        if (r == 1) {   // the chunk decays faster than tier A covers (uniform over the CTA)
            __syncthreads();
            intra_chunk_strong<DK, GS, PRO, BX>(slot, h, q, k, log_alpha, beta, cu_seqlens, T, H, num_seqs, ws, sm,
                                                tmem, &ph_mma);
        }
        if (r < 0) break;   // a wait timed out (flagged; uniform)
        // this item's shared memory and TMEM are free before the next item starts
        ptx::tc_fence_before();
        __syncthreads();
        ptx::tc_fence_after();
    }
    ptx::tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, INTRA_TMEM_COLS);
    }
}

// Grid of the persistent first pass: two CTAs per SM, at most one per item.
inline unsigned intra_grid(long long items) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess)
        sms = 148;
    return (unsigned)(items < 2LL * sms ? items : 2LL * sms);
}

// Tensor maps the first pass prefetches with (q, k and the per-channel gate rows).
inline bool intra_tmaps(CUtensorMap *tq, CUtensorMap *tk, CUtensorMap *tg, const void *q, const void *k,
                        const void *gate, bool gate_scalar, bool gate_bf16, long long tokens, int H, int dk) {
    memset(tg, 0, sizeof(*tg));
    if (!make_tmap(tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, dk, dk) ||
        !make_tmap(tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, dk, dk))
        return false;
    if (gate_scalar) return true;
    return gate_bf16 ? make_tmap(tg, gate, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, dk, dk)
                     : make_tmap(tg, gate, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, tokens, H, dk, dk);
}

// ------------------------------------------------------------------ pass 2

template <int DK, int DVT, int NBUF>
struct InterLayout {
    static constexpr int KA = DK / 64;
    static constexpr int REC = Rec<DK>::BYTES;
    static constexpr int SP = NBUF * REC;                 // bf16 S, MN-major (key rows = K, value columns = N)
    static constexpr int ZT = SP + KA * DVT * 128;        // bf16 Z, MN-major (tokens = K, value columns = N)
    static constexpr int VIN = ZT + DVT * 128;            // bf16 [NBUF][64][DVT]
    static constexpr int MISC = VIN + NBUF * C * DVT * 2; // mbarriers, TMEM base, flags
    static constexpr int BYTES = MISC + 64;
    static constexpr int ALLOC = BYTES + 1024;
    static_assert(REC % 1024 == 0 && SP % 1024 == 0 && ZT % 1024 == 0 && VIN % 128 == 0, "tile alignment");
};

constexpr uint32_t INTER_TMEM_COLS = 256;
constexpr uint32_t XCOL_XY = 0;       // [128 x DVT] rows 0-63 X, rows 64-127 Y, then O

// ---- pass 2: warp-specialised
//
// Eight compute warps and one issue warp.  Lane 0 of the issue warp loads the
// records and V tiles and issues every tcgen05.mma (each issue holds its thread
// for tens of cycles); the compute warps never wait on an issuing thread, only on
// the products they consume.  Per chunk c (buffer b = c % NBUF):
//
//   compute (all)      wait record b; e^{G_last} -> register; quads 2-3 then release b
//   issue              wait record b and S_c in bf16 (bar_s) -> [X; Y] = [K^; Q^] S_c
//                      into XY[c & 1], commit bar_x
//   compute (quads 0-1) wait bar_x -> Z = V - X in bf16 -> bar_z, release b
//   compute (quads 2-3) wait bar_o[(c-1) & 1] -> O of chunk c-1 -> o
//   issue              wait bar_z -> dS = Kt Z (commit bar_ds), O = Y + Pt Z onto
//                      XY[c & 1] (commit bar_o[c & 1]); then, once chunk c-1's
//                      buffer is released and its products are done, load chunk
//                      c-1+NBUF into it
//   compute (all)      wait bar_ds -> S <- Diag(e^{G_last}) S + dS -> S_{c+1} in bf16 -> bar_s
//
// so the serial path per chunk is the two dependent products and the two
// elementwise steps between them; the output product, the readout of O and the
// record loads overlap it.  Every wait is bounded: a thread whose wait runs out
// flags the device status and leaves its loop; the others then run out in turn.
//
// CK (the backward's forward state sweep, dv = 128): ws (and ckpt, the same bytes,
// writable) hold [slot][H] BwdUnit; only the Khat rows, the Kt rows and e^{G_last}
// of each record are loaded (the Qhat rows hold stale bytes whose products are
// never read); no output; instead the state at each chunk's start, bf16, goes to
// the unit's SC tile (a K-major operand S with K = value columns, MN-major for S^T).

constexpr int NT_WS = NT + 32;   // 8 compute warps + the issue warp

template <int DK, int DVT, int NBUF>
struct InterWsLayout {
    using B = InterLayout<DK, DVT, NBUF>;
    static constexpr int SP = B::SP, ZT = B::ZT, VIN = B::VIN, MISC = B::MISC;
    // MISC: bar_rec[NBUF], bar_free[NBUF], bar_s, bar_x, bar_z, bar_ds, bar_o[2], TMEM base
    static constexpr int BAR_REC = MISC, BAR_FREE = MISC + 32, BAR_S = MISC + 64, BAR_X = MISC + 72,
                         BAR_Z = MISC + 80, BAR_DS = MISC + 88, BAR_O = MISC + 96, TSLOT = MISC + 112;
    static constexpr int BYTES = MISC + 128;
    static constexpr int ALLOC = BYTES + 1024;
    static_assert(NBUF <= 4, "barrier slots");
};

// Three record buffers (two chunks of lead for each load) where they fit.
template <int DK, int DVT>
constexpr int inter_ws_nbuf() {
    return InterWsLayout<DK, DVT, 3>::ALLOC <= 232448 ? 3 : 2;
}

// TMEM: [X; Y] alternates by chunk parity between two buffers XY_STRIDE apart; Kt Z
// follows them.  256 columns up to 64-column value tiles, 512 for 128-column tiles.
template <int DVT>
struct InterWsCols {
    static constexpr uint32_t XY_STRIDE = DVT <= 64 ? 64u : 128u;
    static constexpr uint32_t DS = 2 * XY_STRIDE;
    static constexpr uint32_t ALLOC = DVT <= 64 ? 256u : 512u;
    static_assert(DS + DVT <= ALLOC, "TMEM columns");
};

template <int DK, int DVT, int NBUF, bool CK = false>
__device__ __forceinline__ void inter_ws_body(int tile, const CUtensorMap *tm_v, const uint8_t *__restrict__ ws,
                                              const float *__restrict__ init_state, __nv_bfloat16 *__restrict__ o,
                                              float *__restrict__ final_state,
                                              const int32_t *__restrict__ cu_seqlens, int T, int H, int DV,
                                              const int32_t *__restrict__ slots, int num_slots,
                                              uint8_t *__restrict__ ckpt = nullptr) {
    using L = InterWsLayout<DK, DVT, NBUF>;
    using R = Rec<DK>;
    using TC = InterWsCols<DVT>;
    using MN = MnOp<DVT>;
    static_assert(DVT % 32 == 0 && DVT >= 32 && DVT <= 128, "value tile");
    constexpr int CPT = DVT / 2;
    constexpr uint32_t REC_TX = CK ? (uint32_t)(DK / 64 * 64 * 128 + DK * 128 + DK * 4) : (uint32_t)R::BYTES;
    constexpr uint32_t TX = REC_TX + (uint32_t)(C * DVT * 2);
    constexpr size_t USTRIDE = CK ? (size_t)BwdUnit<DK>::BYTES : (size_t)R::BYTES;   // bytes per (slot, head)
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = ptx::smem_u32(sm);
    const uint32_t bar_rec = sb + L::BAR_REC, bar_free = sb + L::BAR_FREE, bar_s = sb + L::BAR_S,
                   bar_x = sb + L::BAR_X, bar_z = sb + L::BAR_Z, bar_ds = sb + L::BAR_DS, bar_o = sb + L::BAR_O;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::TSLOT);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = (warp >> 2) & 1;
    const int col_base = tile * DVT, h = blockIdx.y;
    const int n = seq_for_cta(cu_seqlens, T, (int)gridDim.z);

    long long t0, t1;
    seq_span(cu_seqlens, T, n, t0, t1);
    const int nck = (int)((t1 - t0 + C - 1) / C);
    const long long first = n + t0 / C;   // slot of chunk 0

    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), TC::ALLOC);
        ptx::tmem_relinquish();
    }
    if (tid == NT) {
        for (int b = 0; b < NBUF; ++b) {
            ptx::mbar_init(bar_rec + 8 * b, 1);
            ptx::mbar_init(bar_free + 8 * b, NT / 32);   // one arrival per compute warp
        }
        ptx::mbar_init(bar_s, NT / 32);
        ptx::mbar_init(bar_x, 1);
        ptx::mbar_init(bar_z, 4);                         // the four warps of quads 0-1
        ptx::mbar_init(bar_ds, 1);
        ptx::mbar_init(bar_o, 1);
        ptx::mbar_init(bar_o + 8, 1);
        ptx::fence_mbar_init();
        if (nck > 0) ptx::prefetch_tmap(tm_v);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == NT / 32) {
        // ---------------- issue warp (lane 0)
        if (lane == 0) {
            int n_issued = 0, n_mma = 0;   // chunks whose loads were issued; chunks with all products issued
            auto issue = [&](int ci) {     // record and V tile of chunk ci into buffer ci % NBUF
                const int b = ci % NBUF;
                const uint32_t bar = bar_rec + 8 * b;
                ptx::mbar_arrive_expect_tx(bar, TX);
                const uint8_t *src = ws + ((size_t)(first + ci) * H + h) * USTRIDE;
                if constexpr (CK) {
#pragma unroll
                    for (int a = 0; a < DK / 64; ++a)
                        ptx::bulk_load(sb + b * R::BYTES + R::KQ + a * 16384, src + R::KQ + a * 16384, 64 * 128, bar);
                    ptx::bulk_load(sb + b * R::BYTES + R::KP, src + R::KP, DK * 128, bar);
                    ptx::bulk_load(sb + b * R::BYTES + R::DCH, src + R::DCH, DK * 4, bar);
                } else {
                    ptx::bulk_load(sb + b * R::BYTES, src, (uint32_t)R::BYTES, bar);
                }
                ptx::tma_load_3d(sb + L::VIN + b * C * DVT * 2, tm_v, bar, col_base, h,
                                 (int)(t0 + (long long)ci * C));
                n_issued = ci + 1;
            };
            for (int ci = 0; ci < NBUF && ci < nck; ++ci) issue(ci);
            constexpr uint32_t idx = ptx::idesc_bf16_f32(128, DVT, false, true);
            for (int ci = 0; ci < nck && ok; ++ci) {
                const int b = ci % NBUF;
                const uint32_t rb = sb + b * R::BYTES;
                const uint32_t xy = XCOL_XY + (uint32_t)(ci & 1) * TC::XY_STRIDE;
                ok = ptx::mbar_wait_bounded(bar_rec + 8 * b, (uint32_t)((ci / NBUF) & 1), WAIT_LIMIT_CYCLES) &&
                     ptx::mbar_wait_bounded(bar_s, (uint32_t)(ci & 1), WAIT_LIMIT_CYCLES);
                if (!ok) break;
                ptx::tc_fence_after();
#pragma unroll
                for (int s = 0; s < DK / 16; ++s)
                    ptx::mma_bf16(tmem + xy, kdesc(rb + R::KQ, s, 128), MN::desc(sb + L::SP, s, DK), idx, s > 0);
                ptx::mma_commit(bar_x);
                // chunk ci-1's buffer: released by the compute warps, its products done
                if (ci >= 1 && ci - 1 + NBUF < nck) {
                    const int cp = ci - 1;
                    ok = ptx::mbar_wait_bounded(bar_free + 8 * (cp % NBUF), (uint32_t)((cp / NBUF) & 1),
                                                WAIT_LIMIT_CYCLES) &&
                         ptx::mbar_wait_bounded(bar_o + 8 * (cp & 1), (uint32_t)((cp >> 1) & 1), WAIT_LIMIT_CYCLES);
                    if (!ok) break;
                    issue(cp + NBUF);
                }
                ok = ptx::mbar_wait_bounded(bar_z, (uint32_t)(ci & 1), WAIT_LIMIT_CYCLES);
                if (!ok) break;
                ptx::tc_fence_after();
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    ptx::mma_bf16(tmem + TC::DS, kdesc(rb + R::KP, s, DK + 64), MN::desc(sb + L::ZT, s, C), idx,
                                  s > 0);
                ptx::mma_commit(bar_ds);
                if constexpr (!CK) {
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        ptx::mma_bf16(tmem + xy, kdesc(rb + R::KP, s, DK + 64, DK - 64), MN::desc(sb + L::ZT, s, C),
                                      idx, 1);
                }
                ptx::mma_commit(bar_o + 8 * (ci & 1));   // CK: marks chunk ci's products done, for the reload
                n_mma = ci + 1;
            }
            if (!ok) {
                flag_status(KDA_DEV_WAIT_TIMEOUT);
                // let the products and copies in flight land (bounded) before the CTA leaves
                if (n_mma > 0) {
                    const int cl = n_mma - 1;
                    ptx::mbar_wait_bounded(bar_o + 8 * (cl & 1), (uint32_t)((cl >> 1) & 1), WAIT_LIMIT_CYCLES);
                }
                for (int c = max(0, n_issued - NBUF); c < n_issued; ++c)
                    ptx::mbar_wait_bounded(bar_rec + 8 * (c % NBUF), (uint32_t)((c / NBUF) & 1), WAIT_LIMIT_CYCLES);
            }
        }
        __syncwarp();
    } else {
        // ---------------- compute warps: thread <-> key row srow, value columns scol..scol+CPT-1
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
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
        // S (the state at chunk c's start) -> bf16 B operand of chunk c's [X; Y] product
        // (CK: and the unit's checkpoint), then bar_s
        auto put_state = [&](int c) {
            if (has_row) {
                uint8_t *ck = CK ? ckpt + ((size_t)(first + c) * H + h) * USTRIDE + BwdUnit<DK>::SC : nullptr;
#pragma unroll
                for (int g = 0; g < CPT / 8; ++g) {
                    const uint4 w =
                        make_uint4(pack_bf16(S[8 * g], S[8 * g + 1]), pack_bf16(S[8 * g + 2], S[8 * g + 3]),
                                   pack_bf16(S[8 * g + 4], S[8 * g + 5]), pack_bf16(S[8 * g + 6], S[8 * g + 7]));
                    *reinterpret_cast<uint4 *>(sm + L::SP + MN::off(srow, scol + 8 * g, DK)) = w;
                    if constexpr (CK) *reinterpret_cast<uint4 *>(ck + sw128(srow, col_base + scol + 8 * g, DK)) = w;
                }
                ptx::fence_proxy_async_smem();
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar_s);
        };
        // quads 2-3 (TMEM lanes 64-127): O rows of chunk c -> o
        auto store_o = [&](int c) -> bool {
            if (!ptx::mbar_wait_bounded(bar_o + 8 * (c & 1), (uint32_t)((c >> 1) & 1), WAIT_LIMIT_CYCLES)) return false;
            ptx::tc_fence_after();
            const long long cs = t0 + (long long)c * C;
            const int Lc = (int)min((long long)C, t1 - cs);
            const int i = (quad - 2) * 32 + lane;
#pragma unroll 1
            for (int cc = 0; cc < CPT / 16; ++cc) {
                float o16[16];
                ptx::tmem_ld16(tl + XCOL_XY + (uint32_t)(c & 1) * TC::XY_STRIDE + scol + cc * 16, o16);
                ptx::tmem_wait_ld();
                if (i < Lc) {
                    __nv_bfloat16 *dst = o + ((cs + i) * H + h) * DV + col_base + scol + cc * 16;
                    reinterpret_cast<uint4 *>(dst)[0] =
                        make_uint4(pack_bf16(o16[0], o16[1]), pack_bf16(o16[2], o16[3]), pack_bf16(o16[4], o16[5]),
                                   pack_bf16(o16[6], o16[7]));
                    reinterpret_cast<uint4 *>(dst)[1] =
                        make_uint4(pack_bf16(o16[8], o16[9]), pack_bf16(o16[10], o16[11]),
                                   pack_bf16(o16[12], o16[13]), pack_bf16(o16[14], o16[15]));
                }
            }
            return true;
        };
        if (nck > 0) put_state(0);
        for (int ci = 0; ci < nck; ++ci) {
            const long long cs = t0 + (long long)ci * C;
            const int Lc = (int)min((long long)C, t1 - cs);
            const int b = ci % NBUF;
            const uint32_t xy = XCOL_XY + (uint32_t)(ci & 1) * TC::XY_STRIDE;
            if (!(ok = ptx::mbar_wait_bounded(bar_rec + 8 * b, (uint32_t)((ci / NBUF) & 1), WAIT_LIMIT_CYCLES))) break;
            const float dch = has_row ? reinterpret_cast<const float *>(sm + b * R::BYTES + R::DCH)[srow] : 0.f;
            if (quad < 2) {
                // ---- Z = V - X (X in TMEM lanes 0-63) -> Z^T, bf16
                if (!(ok = ptx::mbar_wait_bounded(bar_x, (uint32_t)(ci & 1), WAIT_LIMIT_CYCLES))) break;
                ptx::tc_fence_after();
                const int j = quad * 32 + lane;
                const uint8_t *vin = sm + L::VIN + b * C * DVT * 2;
#pragma unroll 1
                for (int cc = 0; cc < CPT / 16; ++cc) {
                    float x16[16], v16[16];
                    ptx::tmem_ld16(tl + xy + scol + cc * 16, x16);
                    if (j < Lc) {
                        unpack_bf16x8(*reinterpret_cast<const uint4 *>(vin + (j * DVT + scol + cc * 16) * 2), v16);
                        unpack_bf16x8(*reinterpret_cast<const uint4 *>(vin + (j * DVT + scol + cc * 16 + 8) * 2),
                                      v16 + 8);
                    } else {
#pragma unroll
                        for (int u = 0; u < 16; ++u) v16[u] = 0.f;
                    }
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int g = 0; g < 2; ++g)
                        *reinterpret_cast<uint4 *>(sm + L::ZT + MN::off(j, scol + cc * 16 + 8 * g, C)) = make_uint4(
                            pack_bf16(v16[8 * g] - x16[8 * g], v16[8 * g + 1] - x16[8 * g + 1]),
                            pack_bf16(v16[8 * g + 2] - x16[8 * g + 2], v16[8 * g + 3] - x16[8 * g + 3]),
                            pack_bf16(v16[8 * g + 4] - x16[8 * g + 4], v16[8 * g + 5] - x16[8 * g + 5]),
                            pack_bf16(v16[8 * g + 6] - x16[8 * g + 6], v16[8 * g + 7] - x16[8 * g + 7]));
                }
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(bar_z);
                    ptx::mbar_arrive(bar_free + 8 * b);   // V and e^{G_last} of buffer b read
                }
            } else {
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar_free + 8 * b);   // e^{G_last} read
                if (!CK && ci > 0 && !(ok = store_o(ci - 1))) break;
            }
            // ---- S <- Diag(e^{G_last}) S + Kt Z
            if (!(ok = ptx::mbar_wait_bounded(bar_ds, (uint32_t)(ci & 1), WAIT_LIMIT_CYCLES))) break;
            ptx::tc_fence_after();
            if (has_row) {
#pragma unroll
                for (int cc = 0; cc < CPT / 16; ++cc) {
                    float d16[16];
                    ptx::tmem_ld16(tl + TC::DS + scol + cc * 16, d16);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int u = 0; u < 16; ++u) S[cc * 16 + u] = fmaf(dch, S[cc * 16 + u], d16[u]);
                }
            }
            if (ci + 1 < nck) put_state(ci + 1);
        }
        if (!CK && ok && nck > 0 && quad >= 2) ok = store_o(nck - 1);   // O of the last chunk
        if (!ok) flag_status(KDA_DEV_WAIT_TIMEOUT);
        if (ok && final_state && has_row && row >= 0) {
#pragma unroll
            for (int j = 0; j < CPT; j += 4)
                store4(final_state + st_off + (long long)srow * DV + j,
                       make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]));
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, TC::ALLOC);
    }
}

template <int DK, int DVT, int NBUF>
__global__ void __launch_bounds__(NT_WS, 1)
chunk_inter_kernel(const __grid_constant__ CUtensorMap tm_v, const uint8_t *__restrict__ ws,
                   const float *__restrict__ init_state, __nv_bfloat16 *__restrict__ o,
                   float *__restrict__ final_state, const int32_t *__restrict__ cu_seqlens, int T, int H, int DV,
                   const int32_t *__restrict__ slots, int num_slots) {
    inter_ws_body<DK, DVT, NBUF>((int)blockIdx.x, &tm_v, ws, init_state, o, final_state, cu_seqlens, T, H, DV, slots,
                                 num_slots);
}

// ------------------------------------------------------------------ host side

template <int DK, int DVT, bool GS, bool PRO>
int launch_two_pass_t(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                      const float *init_state, void *o, float *final_state, const int32_t *cu_seqlens,
                      long long tokens, int T, int H, int dv, int num_seqs, const int32_t *slots, int num_slots,
                      void *workspace, cudaStream_t st, char *msg, size_t msg_len) {
    CUtensorMap tv;
    if (!make_tmap(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, dv, DVT)) {
        snprintf(msg, msg_len, "building TMA descriptors failed (driver entry point cuTensorMapEncodeTiled)");
        return KDA_ERR_CUDA;
    }
    const long long rec_slots = chunk_slots(tokens, num_seqs);   // workspace records per head
    if (rec_slots > 0x7fffffffLL) {
        snprintf(msg, msg_len, "%lld chunk slots exceed the grid limit", rec_slots);
        return KDA_ERR_UNSUPPORTED;
    }
    constexpr int smem1 = IntraLayout<DK>::ALLOC;
    auto k1 = chunk_intra_kernel<DK, GS, PRO>;
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1);
    if (e != cudaSuccess) {
        snprintf(msg, msg_len, "cudaFuncSetAttribute(chunk_intra): %s", cudaGetErrorString(e));
        return KDA_ERR_CUDA;
    }
    CUtensorMap tq, tk, tg;
    if (!intra_tmaps(&tq, &tk, &tg, q, k, log_alpha, GS, PRO, tokens, H, DK)) {
        snprintf(msg, msg_len, "building TMA descriptors failed (driver entry point cuTensorMapEncodeTiled)");
        return KDA_ERR_CUDA;
    }
    k1<<<intra_grid(rec_slots * H), NT, smem1, st>>>(tq, tk, tg, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k,
                                                  log_alpha, beta, cu_seqlens, T, H, num_seqs, (int)rec_slots,
                                                  (uint8_t *)workspace);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        snprintf(msg, msg_len, "chunk_intra launch: %s", cudaGetErrorString(e));
        return KDA_ERR_CUDA;
    }
    constexpr int NBUF = inter_ws_nbuf<DK, DVT>();
    constexpr int smem2 = InterWsLayout<DK, DVT, NBUF>::ALLOC;
    static_assert(smem2 <= 232448, "shared memory budget");
    auto k2 = chunk_inter_kernel<DK, DVT, NBUF>;
    e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2);
    if (e != cudaSuccess) {
        snprintf(msg, msg_len, "cudaFuncSetAttribute(chunk_inter): %s", cudaGetErrorString(e));
        return KDA_ERR_CUDA;
    }
    k2<<<dim3(dv / DVT, H, num_seqs), NT_WS, smem2, st>>>(tv, (const uint8_t *)workspace, init_state,
                                                           (__nv_bfloat16 *)o, final_state, cu_seqlens, T, H, dv,
                                                           slots, num_slots);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        snprintf(msg, msg_len, "chunk_inter launch: %s", cudaGetErrorString(e));
        return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

inline int launch_two_pass(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                           const float *init_state, void *o, float *final_state, const int32_t *cu_seqlens,
                           long long tokens, int T, int H, int dk, int dv, int num_seqs, const int32_t *slots,
                           int num_slots, bool gate_scalar, void *workspace, cudaStream_t st, char *msg,
                           size_t msg_len, bool prologue = false) {
    // value-tile width of the recurrence pass: the widest that still gives one CTA per SM
    const long long chains = (long long)num_seqs * H;
    int dvt = 32;
    for (int cand = dv; cand >= 32; cand /= 2)
        if (chains * (dv / cand) >= 148) { dvt = cand; break; }
#define KDA_2P_ARGS                                                                                                \
    (q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, tokens, T, H, dv, num_seqs, slots, num_slots, \
     workspace, st, msg, msg_len)
#define KDA_2P(DKv, DVTv)                                                              \
    return gate_scalar ? launch_two_pass_t<DKv, DVTv, true, false> KDA_2P_ARGS          \
           : prologue  ? launch_two_pass_t<DKv, DVTv, false, true> KDA_2P_ARGS          \
                       : launch_two_pass_t<DKv, DVTv, false, false> KDA_2P_ARGS
    if (dk == 128) {
        if (dvt == 128) KDA_2P(128, 128);
        if (dvt == 64) KDA_2P(128, 64);
        KDA_2P(128, 32);
    }
    if (dvt == 128) KDA_2P(64, 128);
    if (dvt == 64) KDA_2P(64, 64);
    KDA_2P(64, 32);
#undef KDA_2P
#undef KDA_2P_ARGS
}

}  // namespace tc
}  // namespace kda
