// KDA decode step: one token per (sequence, head), state updated in place.
//
// Per (n, h), with alpha = exp(log_alpha) on the key axis
// ("Kimi Delta Attention 徹底解説" (tech-tide.dev), § "Kimi Delta Attention の仕組み"):
//   S' = Diag(alpha) S;  r = S'^T k;  p = S'^T q;  u = beta (v - r)
//   S  = S' + k u^T;     o = S^T q = p + (k . q) u
// so the dk x dv fp32 state is read once and written once.
//
// Mapping: one 256-thread CTA per (n, h).  Warp w owns a 32-column stripe of the
// state and a group of rows; lane l owns 4 consecutive columns (8 lanes span
// 128 bytes of a row, the warp spans 4 rows per 128-bit access).  Reductions over
// the key axis run in registers, then across the warp's 4 row lanes by shuffles,
// then across the row groups through 2 KB of shared memory.
#pragma once

#include "kda_common.cuh"

namespace kda {

// GS: scalar gate, one log_alpha per (sequence, head) (Gated DeltaNet), else one per key channel.
// PRO: fused input prologue -- q and k raw (scaled here to unit norm), log_alpha
// points to the gate pre-activation x [N, H, DK] in Tin, alpha = exp(-softplus(x)).
template <int DK, int DV, typename Tin, bool GS, bool PRO>
__global__ void __launch_bounds__(256, 2)
decode_step_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                   const float *__restrict__ log_alpha, const float *__restrict__ beta,
                   float *__restrict__ state, Tin *__restrict__ o, const int32_t *__restrict__ slots,
                   int num_slots, int H) {
    constexpr int NSTRIPE = DV / 32;          // 32-column stripes
    constexpr int RG = 8 / NSTRIPE;           // row groups (warps per stripe)
    constexpr int ROWS_PER_GROUP = DK / RG;
    constexpr int RPT = ROWS_PER_GROUP / 4;   // rows held by one thread
    static_assert(NSTRIPE * RG == 8 && RPT >= 1, "decode tiling");

    const long long pair = blockIdx.x;        // n * H + h
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int stripe = warp % NSTRIPE, rg = warp / NSTRIPE;
    const int cg = lane & 7, rl = lane >> 3;
    const int col0 = stripe * 32 + cg * 4;
    const int row0 = rg * ROWS_PER_GROUP + rl;   // this thread's rows: row0 + 4 m

    __shared__ float s_a[DK], s_k[DK], s_ak[DK], s_aq[DK];
    __shared__ float s_red[RG][2][DV];
    __shared__ float s_qk[8];

    // state of this (sequence, head): row n, or its slot in a state pool
    const int row = state_row(slots, num_slots, (int)(pair / H));
    if (row < 0) {   // no state: a padding entry; its output row is zero
        if (rg == 0 && rl == 0) store4(o + pair * DV + col0, make_float4(0.f, 0.f, 0.f, 0.f));
        return;
    }
    float *S = state + ((long long)row * H + pair % H) * (long long)(DK * DV);

    // The state dominates the traffic: put all of this thread's loads in flight first.
    float4 s[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) s[m] = ld_stream(S + (row0 + 4 * m) * DV + col0);

    const long long kb = pair * DK;
    float qk = 0.f;
    if constexpr (!PRO) {
        for (int c = tid; c < DK; c += 256) {
            const float a = expf(GS ? log_alpha[pair] : log_alpha[kb + c]);
            const float kc = Elem<Tin>::load(k + kb + c);
            const float qc = Elem<Tin>::load(q + kb + c);
            s_a[c] = a;
            s_k[c] = kc;
            s_ak[c] = a * kc;
            s_aq[c] = a * qc;
            qk = fmaf(qc, kc, qk);
        }
    } else {
        // raw rows: one channel per thread (DK <= 256); the norms are block sums
        static_assert(DK <= 256, "one key channel per thread");
        __shared__ float s_nrm[8][2];
        const int c = tid;
        float qc = 0.f, kc = 0.f, a = 0.f;
        if (c < DK) {
            qc = Elem<Tin>::load(q + kb + c);
            kc = Elem<Tin>::load(k + kb + c);
            a = expf(neg_softplus(Elem<Tin>::load(reinterpret_cast<const Tin *>(log_alpha) + kb + c)));
        }
        float sq = qc * qc, sk = kc * kc;
#pragma unroll
        for (int off = 16; off; off >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
            sk += __shfl_xor_sync(0xffffffffu, sk, off);
        }
        if (lane == 0) {
            s_nrm[warp][0] = sq;
            s_nrm[warp][1] = sk;
        }
        __syncthreads();
        float tq = 0.f, tk = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            tq += s_nrm[w][0];
            tk += s_nrm[w][1];
        }
        qc *= inv_row_norm(tq);
        kc *= inv_row_norm(tk);
        if (c < DK) {
            s_a[c] = a;
            s_k[c] = kc;
            s_ak[c] = a * kc;
            s_aq[c] = a * qc;
        }
        qk = qc * kc;
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, off);
    if (lane == 0) s_qk[warp] = qk;
    const float4 vv = load4(v + pair * DV + col0);
    const float b = beta[pair];
    __syncthreads();

    // Partial r = (alpha k)^T S and p = (alpha q)^T S over this thread's rows.
    float r[4] = {0.f, 0.f, 0.f, 0.f}, p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int c = row0 + 4 * m;
        const float ak = s_ak[c], aq = s_aq[c];
        r[0] = fmaf(ak, s[m].x, r[0]); r[1] = fmaf(ak, s[m].y, r[1]);
        r[2] = fmaf(ak, s[m].z, r[2]); r[3] = fmaf(ak, s[m].w, r[3]);
        p[0] = fmaf(aq, s[m].x, p[0]); p[1] = fmaf(aq, s[m].y, p[1]);
        p[2] = fmaf(aq, s[m].z, p[2]); p[3] = fmaf(aq, s[m].w, p[3]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        r[j] += __shfl_xor_sync(0xffffffffu, r[j], 8);
        r[j] += __shfl_xor_sync(0xffffffffu, r[j], 16);
        p[j] += __shfl_xor_sync(0xffffffffu, p[j], 8);
        p[j] += __shfl_xor_sync(0xffffffffu, p[j], 16);
    }
    if (rl == 0) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            s_red[rg][0][col0 + j] = r[j];
            s_red[rg][1][col0 + j] = p[j];
        }
    }
    __syncthreads();
    float R[4] = {0.f, 0.f, 0.f, 0.f}, P[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int g = 0; g < RG; ++g)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            R[j] += s_red[g][0][col0 + j];
            P[j] += s_red[g][1][col0 + j];
        }
    float qk_all = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) qk_all += s_qk[w];

    const float u0 = b * (vv.x - R[0]), u1 = b * (vv.y - R[1]);
    const float u2 = b * (vv.z - R[2]), u3 = b * (vv.w - R[3]);
    if (rg == 0 && rl == 0) {
        store4(o + pair * DV + col0, make_float4(fmaf(qk_all, u0, P[0]), fmaf(qk_all, u1, P[1]),
                                                 fmaf(qk_all, u2, P[2]), fmaf(qk_all, u3, P[3])));
    }
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int c = row0 + 4 * m;
        const float a = s_a[c], kc = s_k[c];
        float4 w;
        w.x = fmaf(a, s[m].x, kc * u0);
        w.y = fmaf(a, s[m].y, kc * u1);
        w.z = fmaf(a, s[m].z, kc * u2);
        w.w = fmaf(a, s[m].w, kc * u3);
        st_stream(S + c * DV + col0, w);
    }
}

}  // namespace kda
