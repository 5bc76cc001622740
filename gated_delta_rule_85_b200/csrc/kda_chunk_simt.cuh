// KDA chunked prefill on CUDA cores, fp32 throughout.
//
// The token recurrence ("Kimi Delta Attention 徹底解説" (tech-tide.dev),
// § "Kimi Delta Attention の仕組み") regrouped into 64-token chunks (the page's
// prefill mode; "Kimi Linear、独自の土俵でFull Attentionを上回る" (remio.ai),
// § "Kimi Linearがより賢いRecurrent Memoryを使う方法": chunkwise processing).
// For a chunk starting from state S, with G_i = sum_{s<=i} log_alpha_s per channel:
//   Akk[i][j] = sum_c k_ic k_jc e^{G_ic - G_jc}   (j < i)
//   Aqk[i][j] = sum_c q_ic k_jc e^{G_ic - G_jc}   (j <= i)
//   Z = V - (e^G * K) S
//   U_i = beta_i (Z_i - sum_{j<i} Akk[i][j] U_j)          (forward substitution)
//   O = (e^G * Q) S + Aqk U
//   S <- Diag(e^{G_last}) S + (e^{G_last - G} * K)^T U
// Every decay factor is an exponent of a non-positive number, so nothing
// overflows whatever the gate values.  One 256-thread CTA per
// (32-column value tile, head, sequence); it walks the sequence's chunks in
// order with the fp32 state tile resident in shared memory.
#pragma once

#include "kda_common.cuh"

namespace kda {

namespace simt {
constexpr int C = 64;      // chunk length
constexpr int DVT = 32;    // value columns per CTA
constexpr int NT = 256;    // threads per CTA

template <int DK>
struct Smem {
    static constexpr int DKP = DK + 1;   // padded row stride (conflict-free column walks)
    static constexpr int CP = C + 1;
    static constexpr int q = 0;                       // [C][DKP] q, then e^G * q
    static constexpr int k = q + C * DKP;             // [C][DKP] k, then e^G * k
    static constexpr int g = k + C * DKP;             // [C][DKP] G, then e^{G_last-G} * k
    static constexpr int S = g + C * DKP;             // [DK][DVT] state tile
    static constexpr int akk = S + DK * DVT;          // [C][CP]
    static constexpr int aqk = akk + C * CP;          // [C][CP]
    static constexpr int vz = aqk + C * CP;           // [C][DVT] v, then Z
    static constexpr int y = vz + C * DVT;            // [C][DVT]
    static constexpr int u = y + C * DVT;             // [C][DVT]
    static constexpr int b = u + C * DVT;             // [C]
    static constexpr int d = b + C;                   // [DK]
    static constexpr int total = d + DK;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};
}  // namespace simt

// GS: scalar gate, log_alpha [tokens, H] (Gated DeltaNet), else [tokens, H, DK].
// PRO: fused input prologue -- q and k raw (scaled here to unit norm over the key
// axis), log_alpha points to the gate pre-activation x [tokens, H, DK] in Tin,
// log_alpha = -softplus(x).
template <int DK, typename Tin, bool GS, bool PRO>
__global__ void __launch_bounds__(simt::NT, 1)
chunk_simt_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                  const float *__restrict__ log_alpha, const float *__restrict__ beta,
                  const float *__restrict__ init_state, Tin *__restrict__ o,
                  float *__restrict__ final_state, const int32_t *__restrict__ cu_seqlens, int T, int H,
                  int DV, const int32_t *__restrict__ slots, int num_slots) {
    using namespace simt;
    using L = Smem<DK>;
    constexpr int DKP = L::DKP, CP = L::CP;
    extern __shared__ float sm[];
    float *sQ = sm + L::q, *sK = sm + L::k, *sG = sm + L::g, *sS = sm + L::S;
    float *sAkk = sm + L::akk, *sAqk = sm + L::aqk, *sV = sm + L::vz, *sY = sm + L::y;
    float *sU = sm + L::u, *sB = sm + L::b, *sD = sm + L::d;

    const int tid = threadIdx.x;
    const int col_base = blockIdx.x * DVT, h = blockIdx.y;
    const int n = seq_for_cta(cu_seqlens, T, (int)gridDim.z);
    long long t0, t1;
    seq_span(cu_seqlens, T, n, t0, t1);
    const int row = state_row(slots, num_slots, n);
    const long long state_off = ((long long)(row < 0 ? 0 : row) * H + h) * DK * DV + col_base;

    for (int idx = tid; idx < DK * DVT; idx += NT) {
        const int c = idx / DVT, j = idx % DVT;
        sS[idx] = (init_state && row >= 0) ? init_state[state_off + (long long)c * DV + j] : 0.f;
    }

    for (long long cs = t0; cs < t1; cs += C) {
        const int Lc = (int)min((long long)C, t1 - cs);
        __syncthreads();   // previous chunk finished with every buffer
        for (int idx = tid; idx < C * DK; idx += NT) {
            const int i = idx / DK, c = idx % DK;
            float qv = 0.f, kv = 0.f, gv = 0.f;
            if (i < Lc) {
                const long long off = ((cs + i) * H + h) * DK + c;
                qv = Elem<Tin>::load(q + off);
                kv = Elem<Tin>::load(k + off);
                if constexpr (PRO) gv = neg_softplus(Elem<Tin>::load(reinterpret_cast<const Tin *>(log_alpha) + off));
                else gv = GS ? log_alpha[(cs + i) * H + h] : log_alpha[off];
            }
            sQ[i * DKP + c] = qv;
            sK[i * DKP + c] = kv;
            sG[i * DKP + c] = gv;
        }
        for (int idx = tid; idx < C * DVT; idx += NT) {
            const int i = idx / DVT, j = idx % DVT;
            sV[idx] = i < Lc ? Elem<Tin>::load(v + ((cs + i) * H + h) * DV + col_base + j) : 0.f;
        }
        for (int i = tid; i < C; i += NT) sB[i] = i < Lc ? beta[(cs + i) * H + h] : 0.f;
        __syncthreads();
        if constexpr (PRO) {   // q, k rows to unit norm: 4 lanes per row
            static_assert(NT == 4 * C, "4 threads per chunk row");
            const int i = tid >> 2, l4 = tid & 3;
            float sq = 0.f, sk = 0.f;
            for (int c = l4; c < DK; c += 4) {
                sq = fmaf(sQ[i * DKP + c], sQ[i * DKP + c], sq);
                sk = fmaf(sK[i * DKP + c], sK[i * DKP + c], sk);
            }
            sq += __shfl_xor_sync(0xffffffffu, sq, 1);
            sq += __shfl_xor_sync(0xffffffffu, sq, 2);
            sk += __shfl_xor_sync(0xffffffffu, sk, 1);
            sk += __shfl_xor_sync(0xffffffffu, sk, 2);
            const float iq = inv_row_norm(sq), ik = inv_row_norm(sk);
            for (int c = l4; c < DK; c += 4) {
                sQ[i * DKP + c] *= iq;
                sK[i * DKP + c] *= ik;
            }
            __syncthreads();
        }

        // G: running sum of log-decay over the chunk, one channel per thread.
        for (int c = tid; c < DK; c += NT) {
            float acc = 0.f;
            for (int i = 0; i < C; ++i) {
                acc += sG[i * DKP + c];
                sG[i * DKP + c] = acc;
            }
        }
        __syncthreads();

        // Akk, Aqk with the exact pairwise decay.  Thread pairs row i with row 63-i
        // so every thread handles ~65/8 (i, j) pairs.
        {
            const int l8 = tid & 7, ip = tid >> 3;
            for (int half = 0; half < 2; ++half) {
                const int i = half ? (C - 1 - ip) : ip;
                for (int j = l8; j <= i; j += 8) {
                    float akk = 0.f, aqk = 0.f;
                    for (int c = 0; c < DK; ++c) {
                        const float kj = sK[j * DKP + c] * expf(sG[i * DKP + c] - sG[j * DKP + c]);
                        akk = fmaf(sK[i * DKP + c], kj, akk);
                        aqk = fmaf(sQ[i * DKP + c], kj, aqk);
                    }
                    sAkk[i * CP + j] = (j < i) ? akk : 0.f;
                    sAqk[i * CP + j] = aqk;
                }
            }
        }
        __syncthreads();

        // Per-channel factors: q <- e^G q, k <- e^G k, G <- e^{G_last - G} k; d = e^{G_last}.
        for (int c = tid; c < DK; c += NT) {
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

        // Z = V - Khat S, Y = Qhat S.
        for (int idx = tid; idx < C * DVT; idx += NT) {
            const int i = idx / DVT, j = idx % DVT;
            float x = 0.f, y = 0.f;
            for (int c = 0; c < DK; ++c) {
                const float s = sS[c * DVT + j];
                x = fmaf(sK[i * DKP + c], s, x);
                y = fmaf(sQ[i * DKP + c], s, y);
            }
            sV[idx] -= x;
            sY[idx] = y;
        }
        __syncthreads();

        // U by forward substitution: 8 lanes of one warp per value column.
        {
            const int col = tid >> 3, l8 = tid & 7;
            for (int i = 0; i < C; ++i) {
                float part = 0.f;
                for (int j = l8; j < i; j += 8) part = fmaf(sAkk[i * CP + j], sU[j * DVT + col], part);
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                part += __shfl_xor_sync(0xffffffffu, part, 2);
                part += __shfl_xor_sync(0xffffffffu, part, 4);
                if (l8 == 0) sU[i * DVT + col] = sB[i] * (sV[i * DVT + col] - part);
                __syncwarp();
            }
        }
        __syncthreads();

        // O = Y + Aqk U for the chunk's valid rows.
        for (int idx = tid; idx < C * DVT; idx += NT) {
            const int i = idx / DVT, j = idx % DVT;
            if (i >= Lc) continue;
            float acc = sY[idx];
            for (int jj = 0; jj <= i; ++jj) acc = fmaf(sAqk[i * CP + jj], sU[jj * DVT + j], acc);
            Elem<Tin>::store(o + ((cs + i) * H + h) * DV + col_base + j, acc);
        }
        // S <- Diag(e^{G_last}) S + Kbar^T U.
        for (int idx = tid; idx < DK * DVT; idx += NT) {
            const int c = idx / DVT, j = idx % DVT;
            float acc = sD[c] * sS[idx];
            for (int i = 0; i < C; ++i) acc = fmaf(sG[i * DKP + c], sU[i * DVT + j], acc);
            sS[idx] = acc;
        }
    }
    __syncthreads();
    if (final_state && row >= 0) {
        for (int idx = tid; idx < DK * DVT; idx += NT) {
            const int c = idx / DVT, j = idx % DVT;
            final_state[state_off + (long long)c * DV + j] = sS[idx];
        }
    }
}

}  // namespace kda
