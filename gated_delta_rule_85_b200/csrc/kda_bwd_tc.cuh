// KDA backward on the tensor cores (tcgen05, bf16 operands, fp32 accumulators in
// TMEM) for bf16 inputs with dk = dv = 128.
//
// The chunk form of the forward ("Kimi Linear、独自の土俵でFull Attentionを上回る"
// (remio.ai), § "Kimi Linearがより賢いRecurrent Memoryを使う方法": chunkwise
// training on the diagonal-plus-low-rank transition), with per chunk (C = 64
// tokens) G the running sum of log_alpha, Khat = e^G K, Qhat = e^G Q,
// Kbar = e^{G_last - G} K, D = e^{G_last}, Akk (j < i), Aqk (j <= i),
// T = (I + Diag(beta) Akk)^{-1}, Tb = T Diag(beta), Kt = Kbar^T Tb, Pt = Aqk Tb:
//   W = V - Khat S,  U = Tb W,  S' = Diag(D) S + Kbar^T U,  O = Qhat S + Aqk U.
// Differentiated, with dO and dS' (the adjoint of the state after the chunk):
//   dU = Aqk^T dO + Kbar dS',  lam = T^T dU,  mu = Diag(beta) lam = Pt^T dO + Kt^T dS',
//   dV = mu,  dbeta_i = <lam_i, W_i - (Akk U)_i>,
//   dAqk = dO U^T (j <= i),  dAkk = -Diag(beta) lam U^T (j < i),
//   dQhat = dO S^T,  dKhat = -mu S^T,  dKbar = U dS'^T,
//   dS = Diag(D) dS' + Qhat^T dO - Khat^T mu,
// then the chain rule through the decay factors and a reverse running sum for
// dlog_alpha.  Three launches:
//   1. chunk_intra_kernel<BX>: the forward's first pass, plus Akk, Aqk and T;
//   2. bwd_sweeps_kernel: the two serial sweeps side by side, each warp-specialised
//      like the forward's second pass -- the forward's state sweep storing each
//      chunk's starting state (bf16) instead of the output (inter_ws_body<CK>), and
//      the adjoint sweep, chunks in reverse, storing each chunk's ending adjoint
//      (bf16) and dS_0 (adj_ws_body);
//   3. bwd_grad_kernel (per chunk, head): every product above that needs S or
//      dS', in a transposed form whose 128 rows are value or key channels
//      (W^T, U^T, dU^T, lam^T: M = dv; the sums over the value columns: M = dk),
//      then the pair terms of dAqk and dAkk through e^{G_i - G_j} and the chain
//      rule -> dq, dk, dv, dlog_alpha, dbeta.
#pragma once

#include <cstring>

#include "kda_chunk_2pass.cuh"

namespace kda {
namespace tc {

// ------------------------------------------------------------------ adjoint sweep

template <int DK, int DVT, int NBUF>
struct AdjLayout {
    static constexpr int KA = DK / 64;
    static constexpr int REC = Rec<DK>::BYTES;
    static constexpr int SP = NBUF * REC;                 // bf16 dS, MN-major (K = key rows, N = value columns)
    static constexpr int MU = SP + KA * DVT * 128;        // bf16 -mu, MN-major (K = tokens, N = value columns)
    static constexpr int DOT = MU + DVT * 128;            // bf16 [NBUF] dO tiles [64][DVT], MN-major (TMA swizzle)
    static constexpr int MISC = DOT + NBUF * C * DVT * 2; // mbarriers, TMEM base
    static constexpr int BYTES = MISC + 64;
    static constexpr int ALLOC = BYTES + 1024;
    static_assert(REC % 1024 == 0 && SP % 1024 == 0 && MU % 1024 == 0 && DOT % 1024 == 0, "tile alignment");
};

// Adjoint sweep: one CTA per (value tile, head, sequence), chunks from the last to
// the first, warp-specialised like the forward's second pass (8 compute warps + 1
// issue warp).  Per step t (chunk c = nck-1-t, buffer b = t % NBUF):
//
//   issue              wait record b -> the state-independent products first:
//                      MU = Pt^T dO (M = 128 over a 64-row operand: the A
//                      descriptor's second 64-row half reads neighbouring bytes,
//                      whose rows are ignored) and DS[t & 1] = Qhat^T dO; then wait
//                      dS' in bf16 (bar_s) -> MU += Kt^T dS', commit bar_mu
//   compute (quads 0-1) wait bar_mu -> -mu in bf16 -> bar_z
//   issue              wait bar_z -> DS[t & 1] += Khat^T (-mu) (M = dk), commit bar_ds;
//                      meanwhile, once step t-1's buffer is released and its
//                      products are done (bar_mu of step t), load step t-1+NBUF into it
//   compute (all)      wait bar_ds -> dS <- Diag(D) dS' + DS -> dS' of the next step in
//                      bf16 (and the unit's DSC checkpoint) -> bar_s
//
// so only Kt^T dS' (8 MMAs), the -mu conversion, Khat^T (-mu) (4 MMAs) and the update
// are on the serial path.  dS_0 goes to dinit_state.  Bounded waits as in the forward.
template <int DK, int DVT, int NBUF>
struct AdjWsLayout {
    using B = AdjLayout<DK, DVT, NBUF>;
    static constexpr int SP = B::SP, MU = B::MU, DOT = B::DOT, MISC = B::MISC;
    // MISC: bar_rec[NBUF], bar_free[NBUF], bar_s, bar_mu, bar_z, bar_ds, TMEM base
    static constexpr int BAR_REC = MISC, BAR_FREE = MISC + 32, BAR_S = MISC + 64, BAR_MU = MISC + 72,
                         BAR_Z = MISC + 80, BAR_DS = MISC + 88, TSLOT = MISC + 112;
    static constexpr int BYTES = MISC + 128;
    static constexpr int ALLOC = BYTES + 1024;
    static_assert(NBUF <= 4, "barrier slots");
};

constexpr uint32_t ACOL_MU = 0;     // [128 x DVT] mu (lanes 0-63; lanes 64-127 unused)
constexpr uint32_t ACOL_DS = 64;    // [128 x DVT] x 2 by step parity: Qhat^T dO - Khat^T mu
static_assert(ACOL_DS + 2 * 64 <= INTER_TMEM_COLS, "TMEM columns");

template <int DK, int DVT, int NBUF>
__device__ __forceinline__ void adj_ws_body(int tile, const CUtensorMap *tm_do, uint8_t *__restrict__ ws,
                                            const float *__restrict__ dfinal, float *__restrict__ dinit_state,
                                            const int32_t *__restrict__ cu_seqlens, int T, int H, int DV) {
    using L = AdjWsLayout<DK, DVT, NBUF>;
    using R = Rec<DK>;
    using U = BwdUnit<DK>;
    static_assert(DK == 128 && (DVT == 32 || DVT == 64), "tile shape");
    constexpr int CPT = DVT / 2;
    constexpr uint32_t TX = (uint32_t)(R::BYTES + C * DVT * 2);
    using MN = MnOp<DVT>;
    using M64 = MnOp<64>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = ptx::smem_u32(sm);
    const uint32_t bar_rec = sb + L::BAR_REC, bar_free = sb + L::BAR_FREE, bar_s = sb + L::BAR_S,
                   bar_mu = sb + L::BAR_MU, bar_z = sb + L::BAR_Z, bar_ds = sb + L::BAR_DS;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::TSLOT);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = (warp >> 2) & 1;
    const int col_base = tile * DVT, h = blockIdx.y;
    const int n = seq_for_cta(cu_seqlens, T, (int)gridDim.z);
    long long t0, t1;
    seq_span(cu_seqlens, T, n, t0, t1);
    const int nck = (int)((t1 - t0 + C - 1) / C);
    const long long first = n + t0 / C;

    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), INTER_TMEM_COLS);
        ptx::tmem_relinquish();
    }
    if (tid == NT) {
        for (int b = 0; b < NBUF; ++b) {
            ptx::mbar_init(bar_rec + 8 * b, 1);
            ptx::mbar_init(bar_free + 8 * b, NT / 32);
        }
        ptx::mbar_init(bar_s, NT / 32);
        ptx::mbar_init(bar_mu, 1);
        ptx::mbar_init(bar_z, 4);
        ptx::mbar_init(bar_ds, 1);
        ptx::fence_mbar_init();
        if (nck > 0) ptx::prefetch_tmap(tm_do);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == NT / 32) {
        // ---------------- issue warp (lane 0)
        if (lane == 0) {
            int n_issued = 0, n_done = 0;   // steps whose loads were issued; steps with all products issued
            auto issue = [&](int t) {      // record and dO tile of step t (chunk nck-1-t) into buffer t % NBUF
                const int b = t % NBUF, ci = nck - 1 - t;
                const uint32_t bar = bar_rec + 8 * b;
                ptx::mbar_arrive_expect_tx(bar, TX);
                ptx::bulk_load(sb + b * R::BYTES, ws + ((size_t)(first + ci) * H + h) * U::BYTES, (uint32_t)R::BYTES,
                               bar);
                ptx::tma_load_3d(sb + L::DOT + b * C * DVT * 2, tm_do, bar, col_base, h,
                                 (int)(t0 + (long long)ci * C));
                n_issued = t + 1;
            };
            for (int t = 0; t < NBUF && t < nck; ++t) issue(t);
            constexpr uint32_t im = ptx::idesc_bf16_f32(128, DVT, true, true);
            for (int t = 0; t < nck && ok; ++t) {
                const int b = t % NBUF;
                const uint32_t rb = sb + b * R::BYTES, dob = sb + L::DOT + b * C * DVT * 2, kp = rb + R::KP;
                const uint32_t ds = ACOL_DS + (uint32_t)(t & 1) * 64;
                if (!(ok = ptx::mbar_wait_bounded(bar_rec + 8 * b, (uint32_t)((t / NBUF) & 1), WAIT_LIMIT_CYCLES)))
                    break;
                ptx::tc_fence_after();
                // state-independent: MU = Pt^T dO, DS = Qhat^T dO (MU was read before the last bar_z;
                // DS[t & 1] before the bar_s of step t-1)
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    ptx::mma_bf16(tmem + ACOL_MU, ptx::desc_mnmajor_sw128(kp + (DK + 16 * s) * 128, 2048, 1024),
                                  MN::desc(dob, s, C), im, s > 0);
#pragma unroll
                for (int s = 4; s < 8; ++s)
                    ptx::mma_bf16(tmem + ds, M64::desc(rb + R::KQ, s, 128), MN::desc(dob, s - 4, C), im, s > 4);
                if (!(ok = ptx::mbar_wait_bounded(bar_s, (uint32_t)(t & 1), WAIT_LIMIT_CYCLES))) break;
                ptx::tc_fence_after();
#pragma unroll
                for (int s = 0; s < DK / 16; ++s)
                    ptx::mma_bf16(tmem + ACOL_MU, ptx::desc_mnmajor_sw128(kp + s * 2048, 2048, 1024),
                                  MN::desc(sb + L::SP, s, DK), im, 1);
                ptx::mma_commit(bar_mu);
                // step t-1's buffer: released by the compute warps, its products done (bar_mu of step t)
                if (t >= 1 && t - 1 + NBUF < nck) {
                    ok = ptx::mbar_wait_bounded(bar_free + 8 * ((t - 1) % NBUF), (uint32_t)(((t - 1) / NBUF) & 1),
                                                WAIT_LIMIT_CYCLES) &&
                         ptx::mbar_wait_bounded(bar_mu, (uint32_t)(t & 1), WAIT_LIMIT_CYCLES);
                    if (!ok) break;
                    issue(t - 1 + NBUF);
                }
                if (!(ok = ptx::mbar_wait_bounded(bar_z, (uint32_t)(t & 1), WAIT_LIMIT_CYCLES))) break;
                ptx::tc_fence_after();
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    ptx::mma_bf16(tmem + ds, M64::desc(rb + R::KQ, s, 128), MN::desc(sb + L::MU, s, C), im, 1);
                ptx::mma_commit(bar_ds);
                n_done = t + 1;
            }
            if (!ok) {
                flag_status(KDA_DEV_WAIT_TIMEOUT);
                // let the products and copies in flight land (bounded) before the CTA leaves
                if (n_done > 0) ptx::mbar_wait_bounded(bar_ds, (uint32_t)((n_done - 1) & 1), WAIT_LIMIT_CYCLES);
                for (int t = max(0, n_issued - NBUF); t < n_issued; ++t)
                    ptx::mbar_wait_bounded(bar_rec + 8 * (t % NBUF), (uint32_t)((t / NBUF) & 1), WAIT_LIMIT_CYCLES);
            }
        }
        __syncwarp();
    } else {
        // ---------------- compute warps: thread <-> key row srow, value columns scol..scol+CPT-1
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        const int srow = quad * 32 + lane;
        const int scol = half * CPT;
        const long long st_off = ((long long)n * H + h) * DK * DV + col_base + scol;
        float S[CPT];   // dS' (fp32), this thread's row and columns
#pragma unroll
        for (int j = 0; j < CPT; j += 4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (dfinal) x = load4(dfinal + st_off + (long long)srow * DV + j);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
        // dS' of step t (the end of chunk nck-1-t) -> bf16 B operand and the unit's checkpoint, then bar_s
        auto put_adj = [&](int t) {
            uint8_t *ck = ws + ((size_t)(first + nck - 1 - t) * H + h) * U::BYTES + U::DSC;
#pragma unroll
            for (int g = 0; g < CPT / 8; ++g) {
                const uint4 w = make_uint4(pack_bf16(S[8 * g], S[8 * g + 1]), pack_bf16(S[8 * g + 2], S[8 * g + 3]),
                                           pack_bf16(S[8 * g + 4], S[8 * g + 5]), pack_bf16(S[8 * g + 6], S[8 * g + 7]));
                *reinterpret_cast<uint4 *>(sm + L::SP + MN::off(srow, scol + 8 * g, DK)) = w;
                *reinterpret_cast<uint4 *>(ck + sw128(srow, col_base + scol + 8 * g, DK)) = w;
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar_s);
        };
        if (nck > 0) put_adj(0);
        for (int t = 0; t < nck; ++t) {
            const int b = t % NBUF;
            if (!(ok = ptx::mbar_wait_bounded(bar_rec + 8 * b, (uint32_t)((t / NBUF) & 1), WAIT_LIMIT_CYCLES))) break;
            const float dch = reinterpret_cast<const float *>(sm + b * R::BYTES + R::DCH)[srow];
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar_free + 8 * b);   // e^{G_last} read; the rest only feeds MMAs
            if (quad < 2) {
                // ---- -mu (TMEM lanes 0-63) -> bf16 B operand rows
                if (!(ok = ptx::mbar_wait_bounded(bar_mu, (uint32_t)(t & 1), WAIT_LIMIT_CYCLES))) break;
                ptx::tc_fence_after();
                const int j = quad * 32 + lane;
#pragma unroll 1
                for (int cc = 0; cc < CPT / 16; ++cc) {
                    float x16[16];
                    ptx::tmem_ld16(tl + ACOL_MU + scol + cc * 16, x16);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int g = 0; g < 2; ++g)
                        *reinterpret_cast<uint4 *>(sm + L::MU + MN::off(j, scol + cc * 16 + 8 * g, C)) = make_uint4(
                            pack_bf16(-x16[8 * g], -x16[8 * g + 1]), pack_bf16(-x16[8 * g + 2], -x16[8 * g + 3]),
                            pack_bf16(-x16[8 * g + 4], -x16[8 * g + 5]), pack_bf16(-x16[8 * g + 6], -x16[8 * g + 7]));
                }
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar_z);
            }
            // ---- dS <- Diag(D) dS' + Qhat^T dO - Khat^T mu
            if (!(ok = ptx::mbar_wait_bounded(bar_ds, (uint32_t)(t & 1), WAIT_LIMIT_CYCLES))) break;
            ptx::tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < CPT / 16; ++cc) {
                float d16[16];
                ptx::tmem_ld16(tl + ACOL_DS + (uint32_t)(t & 1) * 64 + scol + cc * 16, d16);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 16; ++u) S[cc * 16 + u] = fmaf(dch, S[cc * 16 + u], d16[u]);
            }
            if (t + 1 < nck) put_adj(t + 1);
        }
        if (!ok) flag_status(KDA_DEV_WAIT_TIMEOUT);
        if (ok && dinit_state) {
#pragma unroll
            for (int j = 0; j < CPT; j += 4)
                store4(dinit_state + st_off + (long long)srow * DV + j, make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]));
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, INTER_TMEM_COLS);
    }
}

// Both state sweeps in one launch (they are independent): CTAs with
// blockIdx.x < DV / DVT run the forward sweep (chunk-start states), the others the
// adjoint sweep, one per (value tile, head, sequence) each; 8 compute warps and
// one issue warp in either role.
template <int DK, int DVT, int NBUF>
__global__ void __launch_bounds__(NT_WS, 1)
bwd_sweeps_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  uint8_t *__restrict__ ws, const float *__restrict__ init_state, const float *__restrict__ dfinal,
                  float *__restrict__ dinit_state, const int32_t *__restrict__ cu_seqlens, int T, int H, int DV) {
    const int nt = DV / DVT;
    if ((int)blockIdx.x < nt)
        inter_ws_body<DK, DVT, NBUF, true>((int)blockIdx.x, &tm_v, ws, init_state, nullptr, nullptr, cu_seqlens, T,
                                           H, DV, nullptr, 0, ws);
    else
        adj_ws_body<DK, DVT, NBUF>((int)blockIdx.x - nt, &tm_do, ws, dfinal, dinit_state, cu_seqlens, T, H, DV);
}

template <int DK, int DVT, int NBUF>
constexpr int sweeps_smem() {
    return InterWsLayout<DK, DVT, NBUF>::ALLOC > AdjWsLayout<DK, DVT, NBUF>::ALLOC ? InterWsLayout<DK, DVT, NBUF>::ALLOC
                                                                                   : AdjWsLayout<DK, DVT, NBUF>::ALLOC;
}

// ------------------------------------------------------------------ per-chunk sums

// Running sum G of log_alpha over one chunk, per (token, channel), for the 8 tokens x
// 4 channels of this thread (tokens 8 seg.., channels 4 cg..; 256 threads): rows
// past Lc count as log_alpha = 0 and k = q = 0.  fSeg: [8][128] fp32 scratch.
// Returns the thread's G values, k (and q) rows as bf16 pairs, and G_last.  GS: one
// rate per (token, head) ([tokens, H]), the same for every channel.
template <bool WITH_Q, bool GS = false>
__device__ __forceinline__ void chunk_decay(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                                            const float *__restrict__ log_alpha, long long cs, int Lc, int H, int h,
                                            float *fSeg, float (&G)[8][4], uint2 (&kv)[8], uint2 (&qv)[8],
                                            float (&tot)[4]) {
    constexpr int DK = 128;
    const int tid = threadIdx.x, cg = tid & 31, seg = tid >> 5, c0 = 4 * cg, i0 = 8 * seg;
    float4 gv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const long long row = cs + min(i0 + u, Lc - 1), off = (row * H + h) * DK + c0;
        if constexpr (GS) {
            const float gs = __ldg(log_alpha + row * H + h);
            gv[u] = make_float4(gs, gs, gs, gs);
        } else {
            gv[u] = __ldg(reinterpret_cast<const float4 *>(log_alpha + off));
        }
        kv[u] = __ldg(reinterpret_cast<const uint2 *>(k + off));
        if constexpr (WITH_Q) qv[u] = __ldg(reinterpret_cast<const uint2 *>(q + off));
    }
    float run[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const bool in = i0 + u < Lc;
        const float g4[4] = {gv[u].x, gv[u].y, gv[u].z, gv[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            run[e] += in ? g4[e] : 0.f;
            G[u][e] = run[e];
        }
        if (!in) {
            kv[u] = make_uint2(0u, 0u);
            qv[u] = make_uint2(0u, 0u);
        }
    }
    *reinterpret_cast<float4 *>(fSeg + seg * DK + c0) = make_float4(run[0], run[1], run[2], run[3]);
    __syncthreads();
    float pre[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int e = 0; e < 4; ++e) tot[e] = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < 8; ++s2) {
        const float4 x = *reinterpret_cast<const float4 *>(fSeg + s2 * DK + c0);
        const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (s2 < seg) pre[e] += xv[e];
            tot[e] += xv[e];
        }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) G[u][e] += pre[e];
}

// Sum over the 32 lanes of a warp of x[j] for each j: lane l ends with the sum of
// element l (a butterfly that halves the vector at each step, 31 shuffles).
__device__ __forceinline__ float warp_transpose_sum32(float (&x)[32]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) {
        const bool up = (lane & w) != 0;
#pragma unroll
        for (int u = 0; u < w; ++u) {
            const float send = up ? x[u] : x[u + w];
            const float keep = up ? x[u + w] : x[u];
            x[u] = keep + __shfl_xor_sync(0xffffffffu, send, w);
        }
    }
    return x[0];
}

struct GradLayout {   // dk = dv = 128; bf16 tiles with a 128-byte swizzle unless noted
    // phases 1-3
    static constexpr int KH = 0;                // [2][64][128 B]   Khat rows (K-major B, N = tokens)
    static constexpr int EX = 16384;            // BwdX             Akk | Aqk | T
    static constexpr int SS = 40960;            // [2][128][128 B]  S at the chunk's start
    static constexpr int DS = 73728;            // [2][128][128 B]  dS' at its end
    static constexpr int DOL = 106496;          // [2][128][128 B]  dO rows 0-63 (TMA); rows 64-127 unused
    static constexpr int KBR = 139264;          // [2][64][128 B]   Kbar rows (K-major B, N = tokens), then lam^T
    static constexpr int VV = 155648;           // [64][128]        V, no swizzle
    static constexpr int AW = 172032;           // [128][128 B]     (Diag(beta) W)^T, then U^T
    static constexpr int ADU = 188416;          // [128][128 B]     dU^T, then -mu^T
    // the chain rule, over tiles that phase 3 has finished with
    static constexpr int DA = KH;               // [128][128 B]     dAkk rows 0-63, dAqk rows 64-127
    static constexpr int KE = SS;               // [2 parts][2][64][128 B]  e^{-G} K: bf16 high part, low part
    static constexpr int KQE = DS;              // [2 parts][2][128][128 B] e^{G - G_last} [K; Q], high, low
    static constexpr int FG = KBR;              // fp32 [64][128]   G
    static constexpr int QR = AW;               // bf16 [64][128]   q, no swizzle
    static constexpr int KR = ADU;              // bf16 [64][128]   k, no swizzle
    // output rows staged for 16-byte stores
    static constexpr int OV = KH;               // bf16 [64][128]   dv (readout 2, stored during phase 3)
    static constexpr int OQ = 0;                // bf16 [64][128]   dq  } over DA and EX, after phase 4
    static constexpr int OK = 16384;            // bf16 [64][128]   dk  }
    static constexpr int OG = FG;               // fp32 [64][128]   dlog_alpha, over G after the readout
    // fp32 scratch
    static constexpr int FB = 204800;           // [64]        beta
    static constexpr int FD = FB + 256;         // [128]       e^{G_last}
    static constexpr int FSEG = FD + 512;       // [8][128]    segment sums
    static constexpr int FDB = FSEG + 4096;     // [4][64]     <lam, W> per lane quadrant
    static constexpr int FDB2 = FDB + 1024;     // [2][64]     sum_j Akk L per column half
    static constexpr int FGC = FDB2 + 512;      // [2][128]    sum_v S dS' per column half
    static constexpr int FX = FGC + 1024;       // [2][2][128] per token half: sum_i k_i b_i, sum_i dG_i
    static constexpr int MISC = FX + 2048;      // mbarriers, TMEM base
    static constexpr int BYTES = MISC + 64;
    static constexpr int ALLOC = BYTES + 1024;
    static_assert(KE + 2 * 16384 <= KQE && KQE + 2 * 32768 <= FG && FG + 32768 <= QR && QR + 16384 <= KR &&
                      KR + 16384 <= FB,
                  "chain-rule tiles over the dead phase 1-3 tiles");
    static_assert(ALLOC <= 232448, "shared memory budget");
};

constexpr uint32_t GRAD_TMEM_COLS = 512;
// TMEM columns, 64 each.  Phase 1: S^T Khat^T, dU^T.  Phase 2: U^T, lam^T.  Phase 3:
// dAqk, S dO^T, -S mu^T, dS' U^T, L = lam U^T (dAqk and L in lanes 0-63).  Phase 4
// (tier A) adds the row terms onto S dO^T and -S mu^T (the same factor e^G scales
// both) and puts the column terms over dAqk, which has been read out.
constexpr uint32_t GC_0 = 0, GC_1 = 64, GC_2 = 128, GC_3 = 192, GC_4 = 256;

// bf16 element (r, j) of a one-atom (64-column) tile with a 128-byte swizzle.
__device__ __forceinline__ float ld_sw128(const uint8_t *tile, int r, int j) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(tile + r * 128 + ((((j >> 3) ^ (r & 7))) << 4) +
                                                                      ((j & 7) << 1)));
}

// Four values as a bf16 high part and the bf16 rounding of the remainder.
__device__ __forceinline__ void st_split_bf16x4(uint8_t *sm, uint32_t hi, uint32_t lo, const float (&x)[4]) {
    float h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        h[e] = __bfloat162float(__float2bfloat16_rn(x[e]));
        l[e] = x[e] - h[e];
    }
    st_bf16x4(sm, hi, h[0], h[1], h[2], h[3]);
    st_bf16x4(sm, lo, l[0], l[1], l[2], l[3]);
}

// Tier B of the chain rule (a chunk decaying faster than the tensor-core factors
// cover): the exact pair terms RQ, RK, CT of key channel c for tokens i0 .. i0+31,
// into fp32 [3][64][128] at out.  Kept out of line and not unrolled: it runs only
// for such chunks.
__device__ __noinline__ void chain_pairs_exact(const uint8_t *da, const float *fG, const __nv_bfloat16 *sq,
                                               const __nv_bfloat16 *sk, int c, int i0, float *out) {
    constexpr int DK = 128;
#pragma unroll 1
    for (int i = i0; i < i0 + 32; ++i) {
        const float Gi = fG[i * DK + c];
        float RQ = 0.f, RK = 0.f, CT = 0.f;
#pragma unroll 1
        for (int j = 0; j <= i; ++j) {
            const float f = __expf(Gi - fG[j * DK + c]) * __bfloat162float(sk[j * DK + c]);
            RQ = fmaf(ld_sw128(da, 64 + i, j), f, RQ);
            RK = fmaf(ld_sw128(da, i, j), f, RK);
        }
#pragma unroll 1
        for (int m = i; m < C; ++m) {
            const float f = __expf(fG[m * DK + c] - Gi);
            const float x = ld_sw128(da, 64 + m, i) * __bfloat162float(sq[m * DK + c]) +
                            ld_sw128(da, m, i) * __bfloat162float(sk[m * DK + c]);
            CT = fmaf(x, f, CT);
        }
        out[i * DK + c] = RQ;
        out[C * DK + i * DK + c] = RK;
        out[2 * C * DK + i * DK + c] = CT;
    }
}

// Persistent: each CTA (256 threads, one per SM) takes (chunk slot, head) items in
// turn, prefetching the next one's inputs into L2.  Warps w and w + 4 share TMEM lane
// quadrant w & 3 (value channel or key channel 32 (w & 3) + lane) and split the 64
// token columns in halves.
//   Phases 1-3: every product that needs S or dS' -> dV, dbeta, dAqk/dAkk and
//   dQhat^T, dKhat^T, dKbar^T (M = key channels), kept in TMEM.
//   Phase 4, the chain rule through the decay factors, with the pair terms of
//   channel c
//     RQ_i = sum_{j<=i} dAqk[i][j] e^{G_i-G_j} k_j,  RK_i = sum_{j<i} dAkk[i][j] e^{G_i-G_j} k_j,
//     CT_j = sum_{i>=j} (dAqk[i][j] q_i + dAkk[i][j] k_i) e^{G_i-G_j}.
//   Tier A (every channel's chunk decay >= -DECAY_LIM): RQ = e^{G_i} [(e^{-G} K)^T dAqk^T]_i,
//   RK likewise, CT = e^{G_last - G_j} [(e^{G - G_last} [K; Q])^T [dAkk; dAqk]]_j on the
//   tensor cores: every operand factor is >= 1 and <= e^DECAY_LIM and the products are
//   scaled down afterwards, so no gradient underflows on the way; the decay-scaled
//   operands are split into a bf16 high and low part (two products), because each
//   pair term enters dG_i and dG_j with opposite signs and cancels in the running
//   sum of dlog_alpha only as far as its two roundings agree.  Tier B: the exact
//   sums on the CUDA cores.  Then, with a = e^G dKhat + RK, b = e^{G_last - G} dKbar:
//     dq = e^G dQhat + RQ,  dk = a + b + CT,  dG = q dq + k (a - b - CT),
//     dlog_alpha_t = e^{G_last} sum_v S dS' + sum_i k_i b_i + sum_{i>=t} dG_i.
template <bool GS>
__global__ void __launch_bounds__(NT, 1)
bwd_grad_kernel(const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_g, const __nv_bfloat16 *__restrict__ q,
                const __nv_bfloat16 *__restrict__ k, const float *__restrict__ log_alpha,
                const float *__restrict__ beta, const int32_t *__restrict__ cu_seqlens, int T, int H, int num_seqs,
                int nslots, const uint8_t *__restrict__ ws,
                __nv_bfloat16 *__restrict__ dq, __nv_bfloat16 *__restrict__ dk_out, __nv_bfloat16 *__restrict__ dv_out,
                float *__restrict__ dlog_alpha, float *__restrict__ dbeta) {
    using L = GradLayout;
    using R = Rec<128>;
    using U = BwdUnit<128>;
    constexpr int DK = 128, DV = 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sb = ptx::smem_u32(sm);
    const uint32_t bar_ld = sb + L::MISC, bar_mma = sb + L::MISC + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::MISC + 16);
    float *fB = reinterpret_cast<float *>(sm + L::FB), *fD = reinterpret_cast<float *>(sm + L::FD);
    float *fSeg = reinterpret_cast<float *>(sm + L::FSEG), *fDB = reinterpret_cast<float *>(sm + L::FDB);
    float *fDB2 = reinterpret_cast<float *>(sm + L::FDB2), *fGC = reinterpret_cast<float *>(sm + L::FGC);
    float *fX = reinterpret_cast<float *>(sm + L::FX), *fG = reinterpret_cast<float *>(sm + L::FG);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, quad = warp & 3, half = warp >> 2;
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), GRAD_TMEM_COLS);
        ptx::tmem_relinquish();
    }
    if (tid == 0) {
        ptx::mbar_init(bar_ld, 1);
        ptx::mbar_init(bar_mma, 1);
        ptx::fence_mbar_init();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    uint32_t ph_ld = 0, ph_mma = 0;
    int n_commit = 0, n_ld = 0;
    bool ok = true;
    const int n_items = nslots * H;
    // thread 0: an item's inputs into L2 (nothing waits on it; the item's own copies find them there)
    auto prefetch = [&](int it) {
        const int ps = it % nslots, hp = it / nslots;
        long long pcs;
        int pLc;
        if (!slot_chunk(cu_seqlens, T, num_seqs, ps, pcs, pLc)) return;
        const uint8_t *pu = ws + ((size_t)ps * H + hp) * U::BYTES;
        ptx::bulk_prefetch_l2(pu + R::KQ, 8192u);
        ptx::bulk_prefetch_l2(pu + R::KQ + 16384, 8192u);
        ptx::bulk_prefetch_l2(pu + U::BXO, (uint32_t)(U::BYTES - U::BXO));
        ptx::tma_prefetch_l2_3d(&tm_do, 0, hp, (int)pcs);
        ptx::tma_prefetch_l2_3d(&tm_do, 64, hp, (int)pcs);
        ptx::tma_prefetch_l2_3d(&tm_v, 0, hp, (int)pcs);
        ptx::tma_prefetch_l2_3d(&tm_q, 0, hp, (int)pcs);
        ptx::tma_prefetch_l2_3d(&tm_k, 0, hp, (int)pcs);
        if constexpr (!GS) ptx::tma_prefetch_l2_3d(&tm_g, 0, hp, (int)pcs);
    };
    // persistent: items (slot, head), slot fastest, strided by the grid
    for (int it = (int)blockIdx.x; ok && it < n_items; it += (int)gridDim.x) {
        const int slot = it % nslots, h = it / nslots;
        long long cs;
        int Lc;
        if (!slot_chunk(cu_seqlens, T, num_seqs, slot, cs, Lc)) continue;   // uniform: a slot without a chunk
        const uint8_t *unit = ws + ((size_t)slot * H + h) * U::BYTES;
        if (tid == 0) {
            ptx::mbar_arrive_expect_tx(bar_ld, 16384u + (uint32_t)BwdX::BYTES + 2u * 32768u + 16384u + 16384u);
            ptx::bulk_load(sb + L::KH, unit + R::KQ, 8192u, bar_ld);                 // Khat rows of atom 0
            ptx::bulk_load(sb + L::KH + 8192, unit + R::KQ + 16384, 8192u, bar_ld);  // and of atom 1
            ptx::bulk_load(sb + L::EX, unit + U::BXO, (uint32_t)BwdX::BYTES, bar_ld);
            ptx::bulk_load(sb + L::SS, unit + U::SC, 32768u, bar_ld);
            ptx::bulk_load(sb + L::DS, unit + U::DSC, 32768u, bar_ld);
            ptx::tma_load_3d(sb + L::DOL, &tm_do, bar_ld, 0, h, (int)cs);
            ptx::tma_load_3d(sb + L::DOL + 16384, &tm_do, bar_ld, 64, h, (int)cs);
            ptx::tma_load_3d(sb + L::VV, &tm_v, bar_ld, 0, h, (int)cs);
            ++n_ld;
            if (it + (int)gridDim.x < n_items) prefetch(it + (int)gridDim.x);
        }
        if (tid < C) fB[tid] = tid < Lc ? beta[(cs + tid) * H + h] : 0.f;
        // G, k and q of this thread's 8 tokens x 4 channels, kept for phase 4
        float G[8][4], tot[4];
        uint2 kv[8], qv[8];
        chunk_decay<true, GS>(q, k, log_alpha, cs, Lc, H, h, fSeg, G, kv, qv, tot);
        const int c0 = 4 * (tid & 31), i0 = 8 * (tid >> 5);
        {   // Kbar = e^{G_last - G} K (factors <= 1) and e^{G_last}, while the copies fly
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float4 k4 = bf16x4_to_float4(kv[u]);
                st_bf16x4(sm, L::KBR + sw128(i0 + u, c0, 64), k4.x * __expf(tot[0] - G[u][0]),
                          k4.y * __expf(tot[1] - G[u][1]), k4.z * __expf(tot[2] - G[u][2]),
                          k4.w * __expf(tot[3] - G[u][3]));
            }
            if (tid < 32) *reinterpret_cast<float4 *>(fD + c0) = make_float4(__expf(tot[0]), __expf(tot[1]),
                                                                             __expf(tot[2]), __expf(tot[3]));
        }
        ptx::tc_fence_before();
        const bool strong = __syncthreads_or(tot[0] < -DECAY_LIM || tot[1] < -DECAY_LIM || tot[2] < -DECAY_LIM ||
                                             tot[3] < -DECAY_LIM) != 0;   // uniform: tier B
        ptx::tc_fence_after();
        ok = wait_all(bar_ld, ph_ld);
        if (ok && Lc < C) {   // rows past the chunk's end: zero dO and V (the copies read the next tokens)
            for (int idx = tid; idx < (C - Lc) * 16; idx += NT) {
                const int i = Lc + idx / 16, g = idx % 16;
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                *reinterpret_cast<uint4 *>(sm + L::DOL + (g >> 3) * 16384 + i * 128 + (g & 7) * 16) = z;
                *reinterpret_cast<uint4 *>(sm + L::VV + i * 256 + g * 16) = z;
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();

        // ---- phase 1: S^T Khat^T (-> W^T = V^T - that) ; dU^T = dO^T Aqk + dS'^T Kbar^T
        if (ok && tid == 0) {
            ptx::tc_fence_after();
            constexpr uint32_t i_mk = ptx::idesc_bf16_f32(128, 64, true, false);
            constexpr uint32_t i_mm = ptx::idesc_bf16_f32(128, 64, true, true);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                ptx::mma_bf16(tmem + GC_0, ptx::desc_mnmajor_sw128(sb + L::SS + s * 2048, 16384, 1024),
                              kdesc(sb + L::KH, s, 64), i_mk, s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                ptx::mma_bf16(tmem + GC_1, ptx::desc_mnmajor_sw128(sb + L::DOL + s * 2048, 16384, 1024),
                              ptx::desc_mnmajor_sw128(sb + L::EX + BwdX::AQK + s * 2048, 8192, 1024), i_mm, s > 0);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                ptx::mma_bf16(tmem + GC_1, ptx::desc_mnmajor_sw128(sb + L::DS + s * 2048, 16384, 1024),
                              kdesc(sb + L::KBR, s, 64), i_mk, 1);
            ptx::mma_commit(bar_mma);
            ++n_commit;
        }
        if (ok) ok = wait_all(bar_mma, ph_mma);
        const int vr = quad * 32 + lane;   // this lane's TMEM row: value channel (phases 1-2) or key channel
        if (ok) {   // W^T (scaled by beta_i) and dU^T -> bf16 K-major A operands, rows = value channels
            float x[32], y[32];
            ptx::tmem_ld32(tl + GC_0 + 32 * half, x);
            ptx::tmem_ld32(tl + GC_1 + 32 * half, y);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int i = 32 * half + u;
                const float vi = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(sm + L::VV)[i * DV + vr]);
                x[u] = fB[i] * (vi - x[u]);
            }
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                st_bf16x8(sm, L::AW + sw128_chunk(vr, 4 * half + gq), x + 8 * gq);
                st_bf16x8(sm, L::ADU + sw128_chunk(vr, 4 * half + gq), y + 8 * gq);
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();

        // ---- phase 2: U^T = (beta W)^T T^T ; lam^T = dU^T T
        if (ok && tid == 0) {
            ptx::tc_fence_after();
            constexpr uint32_t i_kk = ptx::idesc_bf16_f32(128, 64);
            constexpr uint32_t i_km = ptx::idesc_bf16_f32(128, 64, false, true);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                ptx::mma_bf16(tmem + GC_2, kdesc(sb + L::AW, s, 128), kdesc(sb + L::EX + BwdX::TI, s, 64), i_kk, s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                ptx::mma_bf16(tmem + GC_3, kdesc(sb + L::ADU, s, 128),
                              ptx::desc_mnmajor_sw128(sb + L::EX + BwdX::TI + s * 2048, 8192, 1024), i_km, s > 0);
            ptx::mma_commit(bar_mma);
            ++n_commit;
        }
        if (ok) ok = wait_all(bar_mma, ph_mma);
        if (ok) {
            float x[32];
            // U^T -> bf16 (rows = value channels): the MN-major B of [dO; lam] U^T and dS' U^T
            ptx::tmem_ld32(tl + GC_2 + 32 * half, x);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) st_bf16x8(sm, L::AW + sw128_chunk(vr, 4 * half + gq), x + 8 * gq);
            // <lam_j, W_j> summed over this warp's 32 value channels
            float lam[32], p[32];
            ptx::tmem_ld32(tl + GC_3 + 32 * half, lam);
            ptx::tmem_ld32(tl + GC_0 + 32 * half, x);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int j = 32 * half + u;
                const float vj = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(sm + L::VV)[j * DV + vr]);
                p[u] = lam[u] * (vj - x[u]);
            }
            fDB[quad * 64 + 32 * half + lane] = warp_transpose_sum32(p);
            // mu = beta lam: dV; lam^T and -mu^T (rows = value channels) for phase 3
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int j = 32 * half + u;
                const float mu = fB[j] * lam[u];
                reinterpret_cast<__nv_bfloat16 *>(sm + L::OV)[j * DV + vr] = __float2bfloat16_rn(mu);
                p[u] = -mu;
            }
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                st_bf16x8(sm, L::KBR + sw128_chunk(vr, 4 * half + gq), lam + 8 * gq);
                st_bf16x8(sm, L::ADU + sw128_chunk(vr, 4 * half + gq), p + 8 * gq);
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();

        // ---- phase 3: dAqk = dO U^T ; S dO^T ; S (-mu)^T ; dS' U^T ; L = lam U^T
        // (dAqk and L: M = 128 over 64-row operands, whose second halves read neighbouring
        // bytes; those rows are ignored)
        if (ok && tid == 0) {
            ptx::tc_fence_after();
            constexpr uint32_t i_kk = ptx::idesc_bf16_f32(128, 64);
            constexpr uint32_t i_km = ptx::idesc_bf16_f32(128, 64, false, true);
            constexpr uint32_t i_mm = ptx::idesc_bf16_f32(128, 64, true, true);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                ptx::mma_bf16(tmem + GC_0, kdesc(sb + L::DOL, s, 128),
                              ptx::desc_mnmajor_sw128(sb + L::AW + s * 2048, 8192, 1024), i_km, s > 0);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                ptx::mma_bf16(tmem + GC_4, ptx::desc_mnmajor_sw128(sb + L::KBR + s * 2048, 8192, 1024),
                              ptx::desc_mnmajor_sw128(sb + L::AW + s * 2048, 8192, 1024), i_mm, s > 0);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                ptx::mma_bf16(tmem + GC_1, kdesc(sb + L::SS, s, 128), kdesc(sb + L::DOL, s, 128), i_kk, s > 0);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                ptx::mma_bf16(tmem + GC_2, kdesc(sb + L::SS, s, 128),
                              ptx::desc_mnmajor_sw128(sb + L::ADU + s * 2048, 8192, 1024), i_km, s > 0);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                ptx::mma_bf16(tmem + GC_3, kdesc(sb + L::DS, s, 128),
                              ptx::desc_mnmajor_sw128(sb + L::AW + s * 2048, 8192, 1024), i_km, s > 0);
            ptx::mma_commit(bar_mma);
            ++n_commit;
        }
        if (ok) {   // meanwhile: the dv rows, and sum_v S dS' (this lane's key channel, the half's 64 columns)
            for (int idx = tid; idx < Lc * (DV / 8); idx += NT) {
                const int j = idx / (DV / 8), g = idx % (DV / 8);
                *reinterpret_cast<uint4 *>(dv_out + ((cs + j) * H + h) * DV + 8 * g) =
                    *reinterpret_cast<const uint4 *>(sm + L::OV + (j * DV + 8 * g) * 2);
            }
            float acc = 0.f;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                float a8[8], b8[8];
                unpack_bf16x8(*reinterpret_cast<const uint4 *>(sm + L::SS + half * 16384 + sw128_chunk(vr, g)), a8);
                unpack_bf16x8(*reinterpret_cast<const uint4 *>(sm + L::DS + half * 16384 + sw128_chunk(vr, g)), b8);
#pragma unroll
                for (int u = 0; u < 8; ++u) acc = fmaf(a8[u], b8[u], acc);
            }
            fGC[half * 128 + vr] = acc;
        }
        if (ok) ok = wait_all(bar_mma, ph_mma);   // phase 1-3 tiles are free from here on
        if (ok) {
            // dA -> the bf16 tile (masked), TMEM lanes 0-63: dAqk (j <= i) -> rows 64-127;
            // L = lam U^T -> dAkk = -beta_i L (j < i) -> rows 0-63, and sum_j Akk L for dbeta
            if (quad < 2) {
                const int i = vr;
                float x[32];
                ptx::tmem_ld32(tl + GC_0 + 32 * half, x);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 32; ++u) x[u] = (32 * half + u <= i) ? x[u] : 0.f;
#pragma unroll
                for (int gq = 0; gq < 4; ++gq) st_bf16x8(sm, L::DA + sw128_chunk(64 + i, 4 * half + gq), x + 8 * gq);
                ptx::tmem_ld32(tl + GC_4 + 32 * half, x);
                ptx::tmem_wait_ld();
                const float bi = fB[i];
                float dot = 0.f, a8[8];
#pragma unroll
                for (int gq = 0; gq < 4; ++gq) {
                    const uint32_t ao = L::EX + BwdX::AKK + sw128_chunk(i, 4 * half + gq);
                    unpack_bf16x8(*reinterpret_cast<const uint4 *>(sm + ao), a8);
#pragma unroll
                    for (int u = 0; u < 8; ++u) dot = fmaf(a8[u], x[8 * gq + u], dot);
                }
                fDB2[half * 64 + i] = dot;
#pragma unroll
                for (int u = 0; u < 32; ++u) x[u] = (32 * half + u < i) ? -bi * x[u] : 0.f;
#pragma unroll
                for (int gq = 0; gq < 4; ++gq) st_bf16x8(sm, L::DA + sw128_chunk(i, 4 * half + gq), x + 8 * gq);
            }
            // G, raw q and k (row-major), and in tier A the split decay-scaled operands
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + u;
                *reinterpret_cast<float4 *>(fG + i * DK + c0) = make_float4(G[u][0], G[u][1], G[u][2], G[u][3]);
                *reinterpret_cast<uint2 *>(sm + L::QR + (i * DK + c0) * 2) = qv[u];
                *reinterpret_cast<uint2 *>(sm + L::KR + (i * DK + c0) * 2) = kv[u];
                if (!strong) {
                    const float4 k4 = bf16x4_to_float4(kv[u]), q4 = bf16x4_to_float4(qv[u]);
                    const float kq[4] = {k4.x, k4.y, k4.z, k4.w}, qq[4] = {q4.x, q4.y, q4.z, q4.w};
                    float xe[4], xk[4], xq[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float en = __expf(-G[u][e]), er = __expf(G[u][e] - tot[e]);   // <= e^DECAY_LIM
                        xe[e] = kq[e] * en;
                        xk[e] = kq[e] * er;
                        xq[e] = qq[e] * er;
                    }
                    st_split_bf16x4(sm, L::KE + sw128(i, c0, 64), L::KE + 16384 + sw128(i, c0, 64), xe);
                    st_split_bf16x4(sm, L::KQE + sw128(i, c0, 128), L::KQE + 32768 + sw128(i, c0, 128), xk);
                    st_split_bf16x4(sm, L::KQE + sw128(64 + i, c0, 128), L::KQE + 32768 + sw128(64 + i, c0, 128), xq);
                }
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();

        // ---- phase 4 (tier A): row terms onto S dO^T and -S mu^T; column terms over dA
        if (ok && !strong) {
            if (tid == 0) {
                ptx::tc_fence_after();
                constexpr uint32_t i_mk = ptx::idesc_bf16_f32(128, 64, true, false);
                constexpr uint32_t i_mm = ptx::idesc_bf16_f32(128, 64, true, true);
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const uint32_t ke = sb + L::KE + part * 16384, kqe = sb + L::KQE + part * 32768;
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        ptx::mma_bf16(tmem + GC_1, ptx::desc_mnmajor_sw128(ke + s * 2048, 8192, 1024),
                                      kdesc(sb + L::DA + 8192, s, 64), i_mk, 1);
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        ptx::mma_bf16(tmem + GC_2, ptx::desc_mnmajor_sw128(ke + s * 2048, 8192, 1024),
                                      kdesc(sb + L::DA, s, 64), i_mk, 1);
#pragma unroll
                    for (int s = 0; s < 8; ++s)
                        ptx::mma_bf16(tmem + GC_0, ptx::desc_mnmajor_sw128(kqe + s * 2048, 16384, 1024),
                                      ptx::desc_mnmajor_sw128(sb + L::DA + s * 2048, 8192, 1024), i_mm,
                                      part > 0 || s > 0);
                }
                ptx::mma_commit(bar_mma);
                ++n_commit;
            }
            ok = wait_all(bar_mma, ph_mma);
        }

        // ---- readout: thread (key channel c, token half)
        const int c = vr;
        const float gl = fG[(C - 1) * DK + c];   // G_last (rows past Lc add nothing)
        const float *fP = reinterpret_cast<const float *>(sm + L::KE);   // tier B: exact RQ, RK, CT
        if (ok && strong)
            chain_pairs_exact(sm + L::DA, fG, reinterpret_cast<const __nv_bfloat16 *>(sm + L::QR),
                              reinterpret_cast<const __nv_bfloat16 *>(sm + L::KR), c, 32 * half,
                              reinterpret_cast<float *>(sm + L::KE));
        if (strong) __syncthreads();   // every thread is done with DA before dq and dk go over it
        __nv_bfloat16 *oq = reinterpret_cast<__nv_bfloat16 *>(sm + L::OQ);
        __nv_bfloat16 *okk = reinterpret_cast<__nv_bfloat16 *>(sm + L::OK);
        const __nv_bfloat16 *sq = reinterpret_cast<const __nv_bfloat16 *>(sm + L::QR);
        const __nv_bfloat16 *sk = reinterpret_cast<const __nv_bfloat16 *>(sm + L::KR);
        float dG[32], kb = 0.f, sdg = 0.f;
        if (ok) {
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                float t1[16], t2[16], t3[16], t0[16];
                const uint32_t col = 32 * half + 16 * cc;
                ptx::tmem_ld16(tl + GC_1 + col, t1);
                ptx::tmem_ld16(tl + GC_2 + col, t2);
                ptx::tmem_ld16(tl + GC_3 + col, t3);
                if (!strong) ptx::tmem_ld16(tl + GC_0 + col, t0);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int i = col + u;
                    const float Gi = fG[i * DK + c];
                    const float qi = __bfloat162float(sq[i * DK + c]), ki = __bfloat162float(sk[i * DK + c]);
                    const float eg = __expf(Gi), eb = __expf(gl - Gi);
                    float RQ = 0.f, RK = 0.f, CT;
                    if (!strong) {
                        CT = eb * t0[u];
                    } else {
                        RQ = fP[i * DK + c];
                        RK = fP[C * DK + i * DK + c];
                        CT = fP[2 * C * DK + i * DK + c];
                    }
                    const float dqi = fmaf(eg, t1[u], RQ);
                    const float a = fmaf(eg, t2[u], RK), b = eb * t3[u];
                    const float dki = a + b + CT;
                    const float g = qi * dqi + ki * (a - b - CT);
                    dG[16 * cc + u] = g;
                    sdg += g;
                    kb = fmaf(ki, b, kb);
                    oq[i * DK + c] = __float2bfloat16_rn(dqi);
                    okk[i * DK + c] = __float2bfloat16_rn(dki);
                }
            }
            fX[half * DK + c] = kb;
            fX[2 * DK + half * DK + c] = sdg;
        }
        __syncthreads();
        float *og = reinterpret_cast<float *>(sm + L::OG);   // over G, which nobody reads any more
        if (ok) {
            float run = fD[c] * (fGC[c] + fGC[128 + c]) + fX[c] + fX[DK + c];
            if (half == 0) run += fX[2 * DK + DK + c];   // all of the later half's dG
#pragma unroll
            for (int u = 31; u >= 0; --u) {
                run += dG[u];
                og[(32 * half + u) * DK + c] = run;
            }
            if (tid < C && tid < Lc) {
                const float db =
                    fDB[tid] + fDB[64 + tid] + fDB[128 + tid] + fDB[192 + tid] - fDB2[tid] - fDB2[64 + tid];
                dbeta[(cs + tid) * H + h] = db;
            }
        }
        __syncthreads();
        if (ok) {   // dq, dk, dlog_alpha rows as 16-byte stores
            for (int idx = tid; idx < Lc * (DK / 8); idx += NT) {
                const int i = idx / (DK / 8), g = idx % (DK / 8);
                const long long o = ((cs + i) * H + h) * DK + 8 * g;
                *reinterpret_cast<uint4 *>(dq + o) = *reinterpret_cast<const uint4 *>(oq + i * DK + 8 * g);
                *reinterpret_cast<uint4 *>(dk_out + o) = *reinterpret_cast<const uint4 *>(okk + i * DK + 8 * g);
            }
            if constexpr (GS) {   // the shared rate's gradient: the sum over the channels, one warp per row
                for (int i = warp; i < Lc; i += NT / 32) {
                    const float4 x = *reinterpret_cast<const float4 *>(og + i * DK + 4 * lane);
                    float t = (x.x + x.y) + (x.z + x.w);
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
                    if (lane == 0) dlog_alpha[(cs + i) * H + h] = t;
                }
            } else {
                for (int idx = tid; idx < Lc * (DK / 4); idx += NT) {
                    const int i = idx / (DK / 4), g = idx % (DK / 4);
                    *reinterpret_cast<float4 *>(dlog_alpha + ((cs + i) * H + h) * DK + 4 * g) =
                        *reinterpret_cast<const float4 *>(og + i * DK + 4 * g);
                }
            }
        }
        // this item's shared-memory reads complete before the next item's copies land
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();
        ptx::tc_fence_after();
    }
    if (!ok && tid == 0) {   // a wait timed out: let the copies and MMAs in flight land (bounded)
        if (n_ld > 0) ptx::mbar_wait_bounded(bar_ld, (uint32_t)((n_ld - 1) & 1), WAIT_LIMIT_CYCLES);
        if (n_commit > 0) ptx::mbar_wait_bounded(bar_mma, (uint32_t)((n_commit - 1) & 1), WAIT_LIMIT_CYCLES);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, GRAD_TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host side

// Workspace of the tensor-core backward: one BwdUnit per (chunk slot, head).
inline size_t backward_tc_workspace_bytes(long long tokens, int H, int num_seqs) {
    if (tokens <= 0) return 0;
    return (size_t)chunk_slots(tokens, num_seqs) * (size_t)H * (size_t)BwdUnit<128>::BYTES;
}

template <typename K>
inline int set_smem_tc(K kern, int bytes, const char *what, char *msg, size_t msg_len) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) return KDA_OK;
    snprintf(msg, msg_len, "cudaFuncSetAttribute(%s): %s", what, cudaGetErrorString(e));
    return KDA_ERR_CUDA;
}

inline int launch_ok(const char *what, char *msg, size_t msg_len) {
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) return KDA_OK;
    snprintf(msg, msg_len, "%s launch: %s", what, cudaGetErrorString(e));
    return KDA_ERR_CUDA;
}

// The three launches for bf16 inputs, dk = dv = 128; GS: one decay rate per
// (token, head) (Gated DeltaNet), log_alpha and dlog_alpha [tokens, H].
template <bool GS>
inline int launch_backward_tc(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                              const float *init_state, const void *d_o, const float *dfinal, void *dq, void *dk_out,
                              void *dv_out, float *dlog_alpha, float *dbeta, float *dinit_state,
                              const int32_t *cu_seqlens, long long tokens, int T, int H, int num_seqs,
                              void *workspace, cudaStream_t st, char *msg, size_t msg_len) {
    constexpr int DK = 128, DV = 128, DVT = 64, NBUF = 3;   // one wave of sweeps at 32 heads
    const long long slots = tokens > 0 ? chunk_slots(tokens, num_seqs) : 0;
    if (slots > 0x7fffffffLL) {
        snprintf(msg, msg_len, "%lld chunk slots exceed the grid limit", slots);
        return KDA_ERR_UNSUPPORTED;
    }
    uint8_t *ws = (uint8_t *)workspace;
    const auto *qb = (const __nv_bfloat16 *)q, *kb = (const __nv_bfloat16 *)k;
    static_assert(DVT == 64, "the sweeps' dO tile is the 128-byte-swizzled 64-column box");
    CUtensorMap t_v64, t_do64, t_v128, t_q, t_k, t_g;
    memset(&t_v64, 0, sizeof(t_v64));   // no tokens: the sweeps load nothing (the adjoint one copies dfinal)
    memset(&t_do64, 0, sizeof(t_do64));
    memset(&t_g, 0, sizeof(t_g));       // GS: log_alpha is not prefetched by tensor map
    if (slots > 0 && (!make_tmap(&t_v64, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, DV, DVT) ||
        !make_tmap(&t_do64, d_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, DV, 64,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap(&t_v128, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, DV, 128) ||
        !make_tmap(&t_q, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, DK, DK) ||
        !make_tmap(&t_k, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, DK, DK) ||
        (!GS && !make_tmap(&t_g, log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, tokens, H, DK, DK)))) {
        snprintf(msg, msg_len, "building TMA descriptors failed (driver entry point cuTensorMapEncodeTiled)");
        return KDA_ERR_CUDA;
    }
    int rc;
    auto k1 = chunk_intra_kernel<DK, GS, false, true>;
    auto k2 = bwd_sweeps_kernel<DK, DVT, NBUF>;
    auto k4 = bwd_grad_kernel<GS>;
    constexpr int s1 = IntraLayout<DK>::ALLOC, s2 = sweeps_smem<DK, DVT, NBUF>(), s4 = GradLayout::ALLOC;
    if ((rc = set_smem_tc(k1, s1, "chunk_intra", msg, msg_len)) ||
        (rc = set_smem_tc(k2, s2, "bwd_sweeps", msg, msg_len)) || (rc = set_smem_tc(k4, s4, "bwd_grad", msg, msg_len)))
        return rc;
    if (slots > 0) {
        CUtensorMap iq, ik, ig;
        if (!intra_tmaps(&iq, &ik, &ig, q, k, log_alpha, GS, false, tokens, H, DK)) {
            snprintf(msg, msg_len, "building TMA descriptors failed (driver entry point cuTensorMapEncodeTiled)");
            return KDA_ERR_CUDA;
        }
        k1<<<intra_grid(slots * H), NT, s1, st>>>(iq, ik, ig, qb, kb, log_alpha, beta, cu_seqlens, T, H, num_seqs,
                                                  (int)slots, ws);
        if ((rc = launch_ok("chunk_intra", msg, msg_len))) return rc;
    }
    // both sweeps; with no tokens only the adjoint half has work (dinit_state = dfinal)
    k2<<<dim3(2 * (DV / DVT), H, num_seqs), NT_WS, s2, st>>>(t_v64, t_do64, ws, init_state, dfinal, dinit_state,
                                                             cu_seqlens, T, H, DV);
    if ((rc = launch_ok("bwd_sweeps", msg, msg_len))) return rc;
    if (slots > 0) {
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                      cudaSuccess)
            sms = 148;
        const long long items = slots * H;
        const unsigned grid = (unsigned)(items < sms ? items : sms);
        k4<<<grid, NT, s4, st>>>(t_do64, t_v128, t_q, t_k, t_g, qb, kb, log_alpha, beta, cu_seqlens, T, H, num_seqs,
                                 (int)slots, ws, (__nv_bfloat16 *)dq, (__nv_bfloat16 *)dk_out, (__nv_bfloat16 *)dv_out,
                                 dlog_alpha, dbeta);
        if ((rc = launch_ok("bwd_grad", msg, msg_len))) return rc;
    }
    return KDA_OK;
}

}  // namespace tc
}  // namespace kda
