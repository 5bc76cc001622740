// Shared device helpers for the KDA kernels (one translation unit: kda_lib.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

// Per-device status word; kernels OR KDA_DEV_* flags into it.
__device__ unsigned int g_status;

__device__ __forceinline__ void flag_status(unsigned int bits) { atomicOr(&g_status, bits); }

// ----------------------------------------------------------------- input access

template <typename T>
struct Elem;

template <>
struct Elem<float> {
    static __device__ __forceinline__ float load(const float *p) { return *p; }
    static __device__ __forceinline__ void store(float *p, float x) { *p = x; }
};

template <>
struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
};

// Load 4 consecutive elements (16-byte aligned for float, 8-byte for bf16) as floats.
__device__ __forceinline__ float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    uint2 raw = *reinterpret_cast<const uint2 *>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&raw.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&raw.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
}

__device__ __forceinline__ void store4(float *p, float4 x) { *reinterpret_cast<float4 *>(p) = x; }
__device__ __forceinline__ void store4(__nv_bfloat16 *p, float4 x) {
    __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(x.z, x.w);
    uint2 raw;
    raw.x = *reinterpret_cast<uint32_t *>(&a);
    raw.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = raw;
}

// Streaming (evict-first) 128-bit global access for data touched exactly once.
__device__ __forceinline__ float4 ld_stream(const float *p) {
    float4 r;
    asm volatile("ld.global.cs.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "l"(p));
    return r;
}
__device__ __forceinline__ void st_stream(float *p, float4 v) {
    asm volatile("st.global.cs.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w)
                 : "memory");
}

// Input prologue: log_alpha = -softplus(x) from the gate pre-activation x,
// evaluated as -(max(x, 0) + log(1 + exp(-|x|))) so no term overflows; the
// fast exponential and logarithm keep the absolute error near 1e-7.
__device__ __forceinline__ float neg_softplus(float x) { return -(fmaxf(x, 0.f) + __logf(1.f + __expf(-fabsf(x)))); }
// 1 / max(|x|_2, 1e-6): the prologue's scale of a q or k row from its squared norm.
__device__ __forceinline__ float inv_row_norm(float sumsq) { return 1.f / fmaxf(sqrtf(sumsq), 1e-6f); }

// Token range of sequence n in the flattened [B*T] token axis.  Packed offsets
// are clamped to [0, T] (B == 1 there) so a malformed cu_seqlens can never
// address memory outside the caller's tensors.
__device__ __forceinline__ void seq_span(const int32_t *cu_seqlens, int T, int n, long long &t0,
                                         long long &t1) {
    if (cu_seqlens) {
        t0 = min(max(cu_seqlens[n], 0), T);
        t1 = min(max(cu_seqlens[n + 1], (int)t0), T);
    } else {
        t0 = (long long)n * T;
        t1 = t0 + T;
    }
}

// State row of sequence n: slots[n] when a slot table is given, n otherwise.
// -1 means "no state": start from zeros and write nothing back.  Entries outside
// [-1, num_slots) flag KDA_DEV_BAD_SLOT and count as -1.  Uniform over the CTA.
__device__ __forceinline__ int state_row(const int32_t *slots, int num_slots, int n) {
    if (!slots) return n;
    const int s = slots[n];
    if (s < -1 || s >= num_slots) {
        if (threadIdx.x == 0) flag_status(KDA_DEV_BAD_SLOT);
        return -1;
    }
    return s;
}

// Sequence handled by this CTA (grid index z).  Packed inputs of up to 256
// sequences are taken longest first (z-th longest, ties by index): the hardware
// starts CTAs roughly in grid order, and starting the longest chains first keeps
// one long sequence from finishing alone at the end (longest-processing-time-first
// list scheduling).  Dense batches (equal lengths) and larger counts keep z.
// Clamped lengths make the ranks a permutation for any cu_seqlens contents.
// Every thread of the CTA must call it (it synchronises).
__device__ __forceinline__ int seq_for_cta(const int32_t *cu_seqlens, int T, int num_seqs) {
    const int z = blockIdx.z;
    if (!cu_seqlens || num_seqs <= 1 || num_seqs > 256) return z;
    __shared__ int s_len[256];
    __shared__ int s_pick;
    for (int i = threadIdx.x; i < num_seqs; i += blockDim.x) {
        long long a, b;
        seq_span(cu_seqlens, T, i, a, b);
        s_len[i] = (int)(b - a);
    }
    if (threadIdx.x == 0) s_pick = z;
    __syncthreads();
    for (int n = threadIdx.x; n < num_seqs; n += blockDim.x) {
        const int ln = s_len[n];
        int rank = 0;
        for (int m = 0; m < num_seqs; ++m) {
            const int lm = s_len[m];
            rank += (lm > ln) || (lm == ln && m < n);
        }
        if (rank == z) s_pick = n;
    }
    __syncthreads();
    return s_pick;
}

}  // namespace kda
