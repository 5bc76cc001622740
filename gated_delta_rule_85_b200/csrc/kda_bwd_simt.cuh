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
//   Qh = e^G q, Kh = e^G k, Kb = e^{G_C - G} k
//   W = V - Kh S;  U_i = beta_i R_i,  R_i = W_i - sum_{j<i} Akk[i][j] U_j
//   O = Qh S + Aqk U;  S_next = Diag(e^{G_C}) S + Kb^T U
// Backward of the chunk, given dO and dS (the adjoint of S_next):
//   dU = Aqk^T dO + Kb dS
//   lam: (I + Diag(beta) Akk)^T lam = dU   (back substitution)
//   mu = beta lam;  dV = mu;  dbeta_i = <lam_i, R_i>
//   dAkk[i][j] = -<mu_i, U_j> (j < i);  dAqk[i][j] = <dO_i, U_j> (j <= i)
//   dQh = dO S^T;  dKh = -mu S^T;  dKb = U dS^T
//   dS_prev = Diag(e^{G_C}) dS + Qh^T dO - Kh^T mu
// and through the decay factors (a = e^G dKh, b = e^{G_C - G} dKb):
//   dq  = e^G dQh + sum_j dAqk[i][j] k_j e^{G_i - G_j}
//   dk  = a + b + sum_j dAkk[i][j] k_j e^{G_i-G_j}
//             + sum_{i>=j} (dAqk[i][j] q_i + dAkk[i][j] k_i) e^{G_i - G_j}   (column j)
//   dG_i = q_i (dq_i) + k_i (dk_i row terms) - k_i (column terms) + k_i (a_i - b_i) ...
//   dG_C += e^{G_C} sum_j S[:, j] dS[:, j] + sum_i k_i b_i;   dlog_alpha_s = sum_{i>=s} dG_i
//
// Kernels:
//   bwd_sweep_kernel, one CTA per (32-column value tile, head, sequence):
//     forward over the chunks storing each chunk's starting state tile, then
//     backward over them carrying dS; writes dV, dS_0 and, per (chunk, tile),
//     the partial sums over its columns of dQh, dKh, dKb, dAqk, dAkk, dbeta and
//     sum_j S dS.
//   bwd_chunk_kernel, one CTA per (chunk slot, head): sums the tiles' partials
//     and applies the decay-factor chain rule; writes dq, dk, dlog_alpha, dbeta.
// Chunk slots as in the two-pass forward: chunk c of sequence n (tokens
// [t0, t1)) is slot n + floor(t0 / 64) + c.
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace bwd {

constexpr int C = 64;      // chunk length
constexpr int DVT = 32;    // value columns per sweep CTA
constexpr int NT = 256;    // threads per CTA
constexpr int TP = DVT + 1;   // padded row stride of [*][DVT] tiles

inline long long chunk_slots(long long tokens, int num_seqs) { return (tokens + C - 1) / C + num_seqs; }

// Per (chunk slot, head, value tile) partial sums, in floats.
template <int DK>
struct Part {
    static constexpr int DQ = 0;                 // [C][DK]  dO S^T
    static constexpr int DKH = DQ + C * DK;      // [C][DK]  -mu S^T
    static constexpr int DKB = DKH + C * DK;     // [C][DK]  U dS^T
    static constexpr int AQK = DKB + C * DK;     // [C][C]   <dO_i, U_j>, j <= i
    static constexpr int AKK = AQK + C * C;      // [C][C]   -<mu_i, U_j>, j < i
    static constexpr int DB = AKK + C * C;       // [C]      <lam_i, R_i>
    static constexpr int DGC = DB + C;           // [DK]     sum_j S[c][j] dS[c][j]
    static constexpr int FLOATS = DGC + DK;
};

// Workspace: chunk-start states [slots][H][DK][DV], then partials
// [slots][H][DV / DVT][Part::FLOATS], all fp32.
inline size_t backward_workspace_bytes(long long tokens, int H, int dk, int dv, int num_seqs) {
    if (tokens <= 0) return 0;
    const size_t slots = (size_t)chunk_slots(tokens, num_seqs);
    const size_t part = dk == 64 ? (size_t)Part<64>::FLOATS : (size_t)Part<128>::FLOATS;
    return slots * (size_t)H * ((size_t)dk * dv + (size_t)(dv / DVT) * part) * sizeof(float);
}

template <int DK>
struct SweepSmem {
    static constexpr int DKP = DK + 1;
    static constexpr int CP = C + 1;
    static constexpr int q = 0;                  // [C][DKP] q, then Qh
    static constexpr int k = q + C * DKP;        // [C][DKP] k, then Kh
    static constexpr int g = k + C * DKP;        // [C][DKP] G, then Kb
    static constexpr int S = g + C * DKP;        // [DK][TP] state tile
    static constexpr int dS = S + DK * TP;       // [DK][TP] adjoint tile
    static constexpr int akk = dS + DK * TP;     // [C][CP]
    static constexpr int aqk = akk + C * CP;     // [C][CP]
    static constexpr int w = aqk + C * CP;       // [C][TP] v, W, then R
    static constexpr int u = w + C * TP;         // [C][TP] U
    static constexpr int dout = u + C * TP;      // [C][TP] dO
    static constexpr int lam = dout + C * TP;    // [C][TP] dU, lam, then mu
    static constexpr int b = lam + C * TP;       // [C]
    static constexpr int d = b + C;              // [DK] e^{G_C}
    static constexpr int total = d + DK;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

// Loads one chunk's q (optional), k and log_alpha rows (zero past Lc) and
// beta, then turns log_alpha into the running sum G (per channel).
template <int DK, typename Tin>
__device__ __forceinline__ void load_chunk_qkg(const Tin *__restrict__ q, const Tin *__restrict__ k,
                                               const float *__restrict__ log_alpha, const float *__restrict__ beta,
                                               long long cs, int Lc, int H, int h, float *sQ, float *sK, float *sG,
                                               float *sB) {
    constexpr int DKP = DK + 1;
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

// Akk (strictly lower) and, if sAqk, Aqk (lower with the diagonal), with the
// exact pairwise decay.  Row i is paired with row 63 - i for balance.
template <int DK>
__device__ __forceinline__ void chunk_grams(const float *sQ, const float *sK, const float *sG, float *sAkk,
                                            float *sAqk) {
    constexpr int DKP = DK + 1, CP = C + 1;
    const int tid = threadIdx.x, l8 = tid & 7, ip = tid >> 3;
    for (int half = 0; half < 2; ++half) {
        const int i = half ? (C - 1 - ip) : ip;
        for (int j = l8; j <= i; j += 8) {
            float akk = 0.f, aqk = 0.f;
            for (int c = 0; c < DK; ++c) {
                const float kj = sK[j * DKP + c] * expf(sG[i * DKP + c] - sG[j * DKP + c]);
                akk = fmaf(sK[i * DKP + c], kj, akk);
                if (sAqk) aqk = fmaf(sQ[i * DKP + c], kj, aqk);
            }
            sAkk[i * CP + j] = (j < i) ? akk : 0.f;
            if (sAqk) sAqk[i * CP + j] = aqk;
        }
    }
    __syncthreads();
}

// q <- e^G q (if sQ), k -> e^G k and G -> e^{G_C - G} k; d = e^{G_C}.
template <int DK>
__device__ __forceinline__ void chunk_factors(float *sQ, float *sK, float *sG, float *sD) {
    constexpr int DKP = DK + 1;
    for (int c = threadIdx.x; c < DK; c += NT) {
        const float gl = sG[(C - 1) * DKP + c];
        sD[c] = expf(gl);
        for (int i = 0; i < C; ++i) {
            const float gi = sG[i * DKP + c];
            const float e = expf(gi);
            const float kc = sK[i * DKP + c];
            if (sQ) sQ[i * DKP + c] *= e;
            sK[i * DKP + c] = kc * e;
            sG[i * DKP + c] = kc * expf(gl - gi);
        }
    }
    __syncthreads();
}

// W <- W - Kh S, then forward substitution U_i = beta_i R_i,
// R_i = W_i - sum_{j<i} Akk[i][j] U_j (R replaces W when keep_r).
template <int DK>
__device__ __forceinline__ void chunk_solve_u(const float *sKh, const float *sS, const float *sAkk, const float *sB,
                                              float *sW, float *sU, bool keep_r) {
    constexpr int DKP = DK + 1, CP = C + 1;
    const int tid = threadIdx.x;
    for (int idx = tid; idx < C * DVT; idx += NT) {
        const int i = idx / DVT, j = idx % DVT;
        float x = 0.f;
        for (int c = 0; c < DK; ++c) x = fmaf(sKh[i * DKP + c], sS[c * TP + j], x);
        sW[i * TP + j] -= x;
    }
    __syncthreads();
    const int col = tid >> 3, l8 = tid & 7;
    for (int i = 0; i < C; ++i) {
        float part = 0.f;
        for (int j = l8; j < i; j += 8) part = fmaf(sAkk[i * CP + j], sU[j * TP + col], part);
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        part += __shfl_xor_sync(0xffffffffu, part, 4);
        if (l8 == 0) {
            const float r = sW[i * TP + col] - part;
            sU[i * TP + col] = sB[i] * r;
            if (keep_r) sW[i * TP + col] = r;
        }
        __syncwarp();
    }
    __syncthreads();
}

template <int DK, typename Tin>
__global__ void __launch_bounds__(NT, 1)
bwd_sweep_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                 const float *__restrict__ log_alpha, const float *__restrict__ beta,
                 const float *__restrict__ init_state, const Tin *__restrict__ d_o,
                 const float *__restrict__ dfinal, Tin *__restrict__ dv_out, float *__restrict__ dinit_state,
                 const int32_t *__restrict__ cu_seqlens, int T, int H, int DV, float *__restrict__ hs,
                 float *__restrict__ part) {
    using L = SweepSmem<DK>;
    using P = Part<DK>;
    constexpr int DKP = L::DKP, CP = L::CP;
    extern __shared__ float sm[];
    float *sQ = sm + L::q, *sK = sm + L::k, *sG = sm + L::g, *sS = sm + L::S, *sdS = sm + L::dS;
    float *sAkk = sm + L::akk, *sAqk = sm + L::aqk, *sW = sm + L::w, *sU = sm + L::u;
    float *sDO = sm + L::dout, *sL = sm + L::lam, *sB = sm + L::b, *sD = sm + L::d;

    const int tid = threadIdx.x;
    const int tile = blockIdx.x, col_base = tile * DVT, h = blockIdx.y;
    const int ntile = DV / DVT;
    const int n = seq_for_cta(cu_seqlens, T, (int)gridDim.z);
    long long t0, t1;
    seq_span(cu_seqlens, T, n, t0, t1);
    const long long first = n + t0 / C;
    const int nch = (int)((t1 - t0 + C - 1) / C);
    const long long st_off = ((long long)n * H + h) * DK * DV + col_base;

    for (int idx = tid; idx < DK * DVT; idx += NT) {
        const int c = idx / DVT, j = idx % DVT;
        sS[c * TP + j] = init_state ? init_state[st_off + (long long)c * DV + j] : 0.f;
    }

    // ---- forward: the state at the start of every chunk
    for (int ci = 0; ci < nch; ++ci) {
        const long long cs = t0 + (long long)ci * C;
        const int Lc = (int)min((long long)C, t1 - cs);
        __syncthreads();
        float *hsp = hs + ((first + ci) * H + h) * (long long)DK * DV + col_base;
        for (int idx = tid; idx < DK * DVT; idx += NT) {
            const int c = idx / DVT, j = idx % DVT;
            hsp[(long long)c * DV + j] = sS[c * TP + j];
        }
        for (int idx = tid; idx < C * DVT; idx += NT) {
            const int i = idx / DVT, j = idx % DVT;
            sW[i * TP + j] = i < Lc ? Elem<Tin>::load(v + ((cs + i) * H + h) * DV + col_base + j) : 0.f;
        }
        load_chunk_qkg<DK, Tin>(q, k, log_alpha, beta, cs, Lc, H, h, nullptr, sK, sG, sB);
        chunk_grams<DK>(nullptr, sK, sG, sAkk, nullptr);
        chunk_factors<DK>(nullptr, sK, sG, sD);
        chunk_solve_u<DK>(sK, sS, sAkk, sB, sW, sU, false);
        for (int idx = tid; idx < DK * DVT; idx += NT) {
            const int c = idx / DVT, j = idx % DVT;
            float acc = sD[c] * sS[c * TP + j];
            for (int i = 0; i < C; ++i) acc = fmaf(sG[i * DKP + c], sU[i * TP + j], acc);
            sS[c * TP + j] = acc;
        }
    }

    // ---- backward
    __syncthreads();
    for (int idx = tid; idx < DK * DVT; idx += NT) {
        const int c = idx / DVT, j = idx % DVT;
        sdS[c * TP + j] = dfinal ? dfinal[st_off + (long long)c * DV + j] : 0.f;
    }
    for (int ci = nch - 1; ci >= 0; --ci) {
        const long long cs = t0 + (long long)ci * C;
        const int Lc = (int)min((long long)C, t1 - cs);
        __syncthreads();
        // Each thread reads back exactly the state entries it stored above.
        const float *hsp = hs + ((first + ci) * H + h) * (long long)DK * DV + col_base;
        for (int idx = tid; idx < DK * DVT; idx += NT) {
            const int c = idx / DVT, j = idx % DVT;
            sS[c * TP + j] = hsp[(long long)c * DV + j];
        }
        for (int idx = tid; idx < C * DVT; idx += NT) {
            const int i = idx / DVT, j = idx % DVT;
            const long long off = ((cs + i) * H + h) * DV + col_base + j;
            sW[i * TP + j] = i < Lc ? Elem<Tin>::load(v + off) : 0.f;
            sDO[i * TP + j] = i < Lc ? Elem<Tin>::load(d_o + off) : 0.f;
        }
        load_chunk_qkg<DK, Tin>(q, k, log_alpha, beta, cs, Lc, H, h, sQ, sK, sG, sB);
        chunk_grams<DK>(sQ, sK, sG, sAkk, sAqk);
        chunk_factors<DK>(sQ, sK, sG, sD);
        chunk_solve_u<DK>(sK, sS, sAkk, sB, sW, sU, true);

        // dU = Aqk^T dO + Kb dS
        for (int idx = tid; idx < C * DVT; idx += NT) {
            const int j = idx / DVT, col = idx % DVT;
            float acc = 0.f;
            for (int i = j; i < C; ++i) acc = fmaf(sAqk[i * CP + j], sDO[i * TP + col], acc);
            for (int c = 0; c < DK; ++c) acc = fmaf(sG[j * DKP + c], sdS[c * TP + col], acc);
            sL[j * TP + col] = acc;
        }
        __syncthreads();
        // back substitution: lam_j = dU_j - sum_{i>j} beta_i Akk[i][j] lam_i
        {
            const int col = tid >> 3, l8 = tid & 7;
            for (int j = C - 1; j >= 0; --j) {
                float acc = 0.f;
                for (int i = j + 1 + l8; i < C; i += 8)
                    acc = fmaf(sB[i] * sAkk[i * CP + j], sL[i * TP + col], acc);
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                acc += __shfl_xor_sync(0xffffffffu, acc, 4);
                if (l8 == 0) sL[j * TP + col] -= acc;
                __syncwarp();
            }
        }
        __syncthreads();

        float *pp = part + (((first + ci) * H + h) * (long long)ntile + tile) * P::FLOATS;
        // dbeta partial: <lam_i, R_i> over this tile's columns (one warp per 8 rows)
        {
            const int warp = tid >> 5, lane = tid & 31;
            for (int i = warp * (C / 8); i < (warp + 1) * (C / 8); ++i) {
                float x = sL[i * TP + lane] * sW[i * TP + lane];
                for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                if (lane == 0) pp[P::DB + i] = x;
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
        // [C][DK] partials: dO S^T, -mu S^T, U dS^T
        for (int idx = tid; idx < C * DK; idx += NT) {
            const int i = idx / DK, c = idx % DK;
            float a0 = 0.f, a1 = 0.f, a2 = 0.f;
            for (int j = 0; j < DVT; ++j) {
                const float s = sS[c * TP + j];
                a0 = fmaf(sDO[i * TP + j], s, a0);
                a1 = fmaf(sL[i * TP + j], s, a1);
                a2 = fmaf(sU[i * TP + j], sdS[c * TP + j], a2);
            }
            pp[P::DQ + idx] = a0;
            pp[P::DKH + idx] = -a1;
            pp[P::DKB + idx] = a2;
        }
        // [C][C] partials over the lower triangle
        for (int idx = tid; idx < C * C; idx += NT) {
            const int i = idx / C, j = idx % C;
            if (j > i) continue;
            float aq = 0.f, ak = 0.f;
            for (int col = 0; col < DVT; ++col) {
                const float uj = sU[j * TP + col];
                aq = fmaf(sDO[i * TP + col], uj, aq);
                ak = fmaf(sL[i * TP + col], uj, ak);
            }
            pp[P::AQK + idx] = aq;
            pp[P::AKK + idx] = j < i ? -ak : 0.f;
        }
        for (int c = tid; c < DK; c += NT) {
            float acc = 0.f;
            for (int j = 0; j < DVT; ++j) acc = fmaf(sS[c * TP + j], sdS[c * TP + j], acc);
            pp[P::DGC + c] = acc;
        }
        __syncthreads();
        // dS <- Diag(e^{G_C}) dS + Qh^T dO - Kh^T mu
        for (int idx = tid; idx < DK * DVT; idx += NT) {
            const int c = idx / DVT, j = idx % DVT;
            float acc = sD[c] * sdS[c * TP + j];
            for (int i = 0; i < C; ++i) {
                acc = fmaf(sQ[i * DKP + c], sDO[i * TP + j], acc);
                acc = fmaf(-sK[i * DKP + c], sL[i * TP + j], acc);
            }
            sdS[c * TP + j] = acc;
        }
    }
    __syncthreads();
    if (dinit_state) {
        for (int idx = tid; idx < DK * DVT; idx += NT) {
            const int c = idx / DVT, j = idx % DVT;
            dinit_state[st_off + (long long)c * DV + j] = sdS[c * TP + j];
        }
    }
}

template <int DK>
struct ChunkSmem {
    static constexpr int CP = C + 1;
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
                 const float *__restrict__ beta, const int32_t *__restrict__ cu_seqlens, int T, int H, int DV,
                 int num_seqs, const float *__restrict__ part, Tin *__restrict__ dq, Tin *__restrict__ dk_out,
                 float *__restrict__ dlog_alpha, float *__restrict__ dbeta) {
    using L = ChunkSmem<DK>;
    using P = Part<DK>;
    constexpr int CP = L::CP;
    extern __shared__ float sm[];
    float *sQ = sm + L::q, *sK = sm + L::k, *sG = sm + L::g, *sDk = sm + L::dk, *sDg = sm + L::dg;
    float *sCk = sm + L::ck, *sDA = sm + L::da, *sGC = sm + L::gc;
    const int tid = threadIdx.x;
    const int slot = blockIdx.x, h = blockIdx.y;
    const int ntile = DV / DVT;

    // the sequence owning this slot: the last n whose first slot n + floor(t0_n / 64) is <= slot
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
    const long long cs = t0 + (long long)(slot - (lo + t0 / C)) * C;
    if (cs < t0 || cs >= t1) return;   // slot without a chunk (the whole CTA leaves)
    const int Lc = (int)min((long long)C, t1 - cs);
    const float *pp = part + ((long long)slot * H + h) * ntile * P::FLOATS;

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
    // tile sums of the [C][C] partials: dAqk on and below the diagonal, dAkk transposed above it
    for (int idx = tid; idx < C * C; idx += NT) {
        const int i = idx / C, j = idx % C;
        if (j > i) continue;
        float aq = 0.f, ak = 0.f;
        for (int t = 0; t < ntile; ++t) {
            aq += pp[t * P::FLOATS + P::AQK + idx];
            ak += pp[t * P::FLOATS + P::AKK + idx];
        }
        sDA[i * CP + j] = aq;
        if (j < i) sDA[j * CP + i] = ak;
    }
    for (int i = tid; i < Lc; i += NT) {
        float acc = 0.f;
        for (int t = 0; t < ntile; ++t) acc += pp[t * P::FLOATS + P::DB + i];
        dbeta[(cs + i) * H + h] = acc;
    }
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
            float rq = 0.f, rk = 0.f, rh = 0.f, rb = 0.f;
            for (int t = 0; t < ntile; ++t) {
                const float *pt = pp + t * P::FLOATS + i * DK + c;
                rq += pt[P::DQ];
                rh += pt[P::DKH];
                rb += pt[P::DKB];
            }
            const float eg = expf(gi);
            const float dqh = eg * rq, a = eg * rh, b = expf(gC - gi) * rb;
            float pq = 0.f, pk = 0.f;
            for (int j = 0; j <= i; ++j) {
                const float kj = sK[j * DK + c] * expf(gi - sG[j * DK + c]);
                pq = fmaf(sDA[i * CP + j], kj, pq);
                if (j < i) pk = fmaf(sDA[j * CP + i], kj, pk);
            }
            rk = a + b + pk;
            if (i < Lc) Elem<Tin>::store(dq + ((cs + i) * H + h) * DK + c, dqh + pq);
            sDk[i * DK + c] = rk;
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
        float dgc = 0.f;
        for (int t = 0; t < ntile; ++t) dgc += pp[t * P::FLOATS + P::DGC + cc];
        float acc = expf(sG[(C - 1) * DK + cc]) * dgc;
        for (int p2 = 0; p2 < NPART; ++p2) acc += sGC[p2 * DK + cc];
        for (int i = C - 1; i >= 0; --i) {
            acc += sDg[i * DK + cc];
            if (i < Lc) dlog_alpha[((cs + i) * H + h) * DK + cc] = acc;
        }
    }
}

}  // namespace bwd
}  // namespace kda
