// libkda: the C ABI declared in include/kda.h.  One translation unit holds every
// kernel so the device status word is a single symbol per device.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "kda_common.cuh"
#include "kda_decode.cuh"
#include "kda_chunk_simt.cuh"
#include "kda_chunk_tc.cuh"
#include "kda_chunk_2pass.cuh"
#include "kda_bwd_simt.cuh"
#include "kda_bwd_tc.cuh"

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return code;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int cuda_fail(cudaError_t e, const char *what) {
    return fail(KDA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

// Validation shared by both prefill entry points.
int check_prefill(const void *q, const void *k, const void *v, const float *log_alpha,
                  const float *beta, const float *init_state, const void *o, const float *final_state,
                  const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv, int num_seqs,
                  int dtype, int chunk, bool gate_scalar = false) {
    if (B < 1 || T < 0 || H < 1 || num_seqs < 0)
        return fail(KDA_ERR_INVALID_ARG, "bad sizes B=%d T=%d H=%d num_seqs=%d", B, T, H, num_seqs);
    // With no tokens the per-token tensors are empty and may be NULL.
    if (T > 0 && (!q || !k || !v || !log_alpha || !beta || !o))
        return fail(KDA_ERR_INVALID_ARG, "q, k, v, log_alpha, beta and o are required");
    if (H > 65535) return fail(KDA_ERR_UNSUPPORTED, "H=%d above 65535", H);
    if (cu_seqlens) {
        if (B != 1) return fail(KDA_ERR_INVALID_ARG, "packed (cu_seqlens) input needs B == 1, got %d", B);
        if (num_seqs < 1) return fail(KDA_ERR_INVALID_ARG, "packed input needs num_seqs >= 1");
    } else if (num_seqs != B) {
        return fail(KDA_ERR_INVALID_ARG, "num_seqs (%d) must equal B (%d) without cu_seqlens", num_seqs, B);
    }
    if (num_seqs > 65535) return fail(KDA_ERR_UNSUPPORTED, "num_seqs=%d above 65535", num_seqs);
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128))
        return fail(KDA_ERR_UNSUPPORTED, "dk=%d dv=%d: each must be 64 or 128", dk, dv);
    if (chunk != 64) return fail(KDA_ERR_UNSUPPORTED, "chunk=%d: only 64 is supported", chunk);
    if (dtype != KDA_BF16 && dtype != KDA_F32) return fail(KDA_ERR_UNSUPPORTED, "dtype=%d", dtype);
    const void *p16[] = {q, k, v, gate_scalar ? nullptr : log_alpha, o, init_state, final_state};
    const char *n16[] = {"q", "k", "v", "log_alpha", "o", "init_state", "final_state"};
    for (int i = 0; i < 7; ++i)
        if (p16[i] && !aligned(p16[i], 16)) return fail(KDA_ERR_MISALIGNED, "%s is not 16-byte aligned", n16[i]);
    if (gate_scalar && log_alpha && !aligned(log_alpha, 4))
        return fail(KDA_ERR_MISALIGNED, "log_alpha is not 4-byte aligned");
    if (beta && !aligned(beta, 4)) return fail(KDA_ERR_MISALIGNED, "beta is not 4-byte aligned");
    if (cu_seqlens && !aligned(cu_seqlens, 4)) return fail(KDA_ERR_MISALIGNED, "cu_seqlens is not 4-byte aligned");
    return KDA_OK;
}

// Which tensor-core schedule runs, the workspace it needs, and (two-pass on one
// sequence longer than the budget allows) the window of tokens per launch pair.
struct Plan {
    int algo;
    size_t ws;
    long long window;   // 0: the whole input in one launch pair
};

constexpr size_t kAutoTwoPassDefault = (size_t)1 << 30;  // AUTO's workspace budget unless set
constexpr long long kAutoChainLimit = 2 * 148;           // AUTO takes TWO_PASS below this many chains
static std::atomic<size_t> g_auto_ws_limit{kAutoTwoPassDefault};

// The state carried between windows: two fp32 [H][dk][dv] buffers at the
// workspace's start (window w reads one and writes the other).
size_t window_carry_bytes(int H, int dk, int dv) {
    return ((size_t)2 * H * dk * dv * sizeof(float) + 1023) / 1024 * 1024;
}

// Longest window (a multiple of the chunk) whose records and carry fit in `limit`; 0 if none.
long long window_tokens(int H, int dk, int dv, size_t limit) {
    const size_t carry = window_carry_bytes(H, dk, dv);
    const size_t per_chunk = kda::tc::two_pass_workspace_bytes(1, H, dk, 0);   // records of one chunk slot
    if (limit <= carry + per_chunk) return 0;
    const long long chunks = (long long)((limit - carry) / per_chunk) - 1;     // one slot of slack per sequence
    return chunks > 0 ? chunks * kda::tc::C : 0;
}

Plan plan_prefill(int B, long long tokens, int H, int dk, int dv, int num_seqs, int algo) {
    const size_t ws2 = kda::tc::two_pass_workspace_bytes(tokens, H, dk, num_seqs);
    if (algo == KDA_ALGO_AUTO) {
        const size_t limit = g_auto_ws_limit.load(std::memory_order_relaxed);
        algo = KDA_ALGO_FUSED;
        if ((long long)num_seqs * H < kAutoChainLimit) {
            if (ws2 <= limit) {
                algo = KDA_ALGO_TWO_PASS;
            } else if (B == 1 && num_seqs == 1) {
                const long long w = window_tokens(H, dk, dv, limit);
                if (w > 0)
                    return Plan{KDA_ALGO_TWO_PASS,
                                window_carry_bytes(H, dk, dv) + kda::tc::two_pass_workspace_bytes(w, H, dk, 1), w};
            }
        }
    }
    return Plan{algo, algo == KDA_ALGO_TWO_PASS ? ws2 : 0, 0};
}

// One sequence (B = 1, no cu_seqlens) through the two-pass schedule in windows of
// `window` tokens: each window is a first-pass/second-pass launch pair on its own
// slice of the inputs and outputs, reusing the records' space; the state passes
// from one window to the next in fp32 through the carry buffers, so the result is
// the one-pair result.
int two_pass_windows(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                     const float *init_state, void *o, float *final_state, int T, int H, int dk, int dv,
                     long long window, bool gate_scalar, void *workspace, cudaStream_t st, char *msg,
                     size_t msg_len) {
    float *carry = (float *)workspace;
    const size_t state_elems = (size_t)H * dk * dv;
    void *rec = (uint8_t *)workspace + window_carry_bytes(H, dk, dv);
    const size_t gate_elems = gate_scalar ? 1 : (size_t)dk;   // log_alpha values per (token, head)
    int w = 0;
    for (long long t0 = 0; t0 < T; t0 += window, ++w) {
        const int tw = (int)std::min(window, (long long)T - t0);
        const bool last = t0 + tw >= T;
        const size_t th = (size_t)t0 * H;
        const float *s_in = w == 0 ? init_state : carry + (size_t)((w - 1) & 1) * state_elems;
        float *s_out = last ? final_state : carry + (size_t)(w & 1) * state_elems;
        const int rc = kda::tc::launch_two_pass(
            (const __nv_bfloat16 *)q + th * dk, (const __nv_bfloat16 *)k + th * dk,
            (const __nv_bfloat16 *)v + th * dv, log_alpha + th * gate_elems, beta + th, s_in,
            (__nv_bfloat16 *)o + th * dv, s_out, nullptr, tw, tw, H, dk, dv, 1, nullptr, 0, gate_scalar, rec, st,
            msg, msg_len);
        if (rc) return rc;
    }
    return KDA_OK;
}

// Scratch of kda_chunk_forward_static_ws: file scope, reserved on each device
// with the module.  Its device address is looked up per device and kept with the
// identity of the context it was taken in: after cudaDeviceReset (or any other
// teardown of the primary context) the module is loaded again and the array may
// move, so a changed context identity triggers a new lookup.
static __device__ __align__(256) uint8_t g_static_ws[KDA_STATIC_WS_BYTES];

constexpr int kMaxDevices = 64;

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Unique identity of the calling thread's current context (0 when there is none
// or the driver cannot tell; 0 is never cached as valid).
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of g_static_ws on the current device (nullptr on failure, with
// the CUDA error in *err).  The symbol is looked up again whenever the current
// context is not the one of the cached address.
void *static_ws_address(cudaError_t *err) {
    static std::mutex mu;
    static void *addr[kMaxDevices] = {};
    static unsigned long long ctx_of[kMaxDevices] = {};
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= kMaxDevices) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    const unsigned long long ctx = current_context_id();
    if (!addr[dev] || ctx == 0 || ctx != ctx_of[dev]) {
        void *p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_static_ws);
        if (*err != cudaSuccess) return nullptr;
        addr[dev] = p;
        ctx_of[dev] = current_context_id();   // the lookup may have created the context
    }
    return addr[dev];
}

template <int DK, typename Tin, bool GS, bool PRO = false>
int launch_simt(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                const float *init_state, void *o, float *final_state, const int32_t *cu_seqlens, int T,
                int H, int dv, int num_seqs, const int32_t *slots, int num_slots, cudaStream_t st) {
    constexpr size_t smem = kda::simt::Smem<DK>::bytes;
    auto kern = kda::chunk_simt_kernel<DK, Tin, GS, PRO>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(chunk_simt)");
    dim3 grid(dv / kda::simt::DVT, H, num_seqs);
    kern<<<grid, kda::simt::NT, smem, st>>>((const Tin *)q, (const Tin *)k, (const Tin *)v, log_alpha, beta,
                                             init_state, (Tin *)o, final_state, cu_seqlens, T, H, dv, slots,
                                             num_slots);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "chunk_simt launch");
    return KDA_OK;
}

template <int DK, int DV, typename Tin, bool GS, bool PRO = false>
int launch_decode(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                  float *state, void *o, long long pairs, const int32_t *slots, int num_slots, int H,
                  cudaStream_t st) {
    kda::decode_step_kernel<DK, DV, Tin, GS, PRO><<<(unsigned)pairs, 256, 0, st>>>(
        (const Tin *)q, (const Tin *)k, (const Tin *)v, log_alpha, beta, state, (Tin *)o, slots, num_slots, H);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "decode_step launch");
    return KDA_OK;
}

// The fp32 CUDA-core prefill after argument checks; `slots` (or NULL) maps
// sequences to state rows.
int simt_impl(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
              const float *init_state, void *o, float *final_state, const int32_t *cu_seqlens, int T, int H,
              int dk, int dv, int num_seqs, int dtype, const int32_t *slots, int num_slots, bool gate_scalar,
              cudaStream_t st, bool prologue = false) {
    if (num_seqs == 0) return KDA_OK;
#define KDA_SIMT(DKv, TT, GSv)                                                                                  \
    return launch_simt<DKv, TT, GSv>(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, T, H, dv, \
                                     num_seqs, slots, num_slots, st)
#define KDA_SIMT_PRO(DKv, TT)                                                                                         \
    return launch_simt<DKv, TT, false, true>(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, T, H, \
                                             dv, num_seqs, slots, num_slots, st)
    if (prologue) {
        if (dtype == KDA_BF16) {
            if (dk == 64) KDA_SIMT_PRO(64, __nv_bfloat16);
            KDA_SIMT_PRO(128, __nv_bfloat16);
        }
        if (dk == 64) KDA_SIMT_PRO(64, float);
        KDA_SIMT_PRO(128, float);
    }
#undef KDA_SIMT_PRO
    if (dtype == KDA_BF16) {
        if (dk == 64) {
            if (gate_scalar) KDA_SIMT(64, __nv_bfloat16, true);
            KDA_SIMT(64, __nv_bfloat16, false);
        }
        if (gate_scalar) KDA_SIMT(128, __nv_bfloat16, true);
        KDA_SIMT(128, __nv_bfloat16, false);
    }
    if (dk == 64) {
        if (gate_scalar) KDA_SIMT(64, float, true);
        KDA_SIMT(64, float, false);
    }
    if (gate_scalar) KDA_SIMT(128, float, true);
    KDA_SIMT(128, float, false);
#undef KDA_SIMT
}

// The tensor-core prefill after argument checks (dtype KDA_BF16, algo valid).
int prefill_impl(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                 const float *init_state, void *o, float *final_state, const int32_t *cu_seqlens, int B, int T,
                 int H, int dk, int dv, int num_seqs, int algo, const int32_t *slots, int num_slots,
                 bool gate_scalar, void *workspace, size_t ws_bytes, cudaStream_t st) {
    const long long tokens = (long long)B * T;
    Plan plan = plan_prefill(B, tokens, H, dk, dv, num_seqs, algo);
    // windows slice one plain sequence; with cu_seqlens or state slots AUTO takes the fused schedule
    if (plan.window && (cu_seqlens || slots)) plan = Plan{KDA_ALGO_FUSED, 0, 0};
    if (plan.ws && (!workspace || ws_bytes < plan.ws))
        return fail(KDA_ERR_WORKSPACE, "workspace of %zu bytes required, got %zu", plan.ws, ws_bytes);
    if (workspace && !aligned(workspace, 256)) return fail(KDA_ERR_MISALIGNED, "workspace is not 256-byte aligned");
    if (num_seqs == 0) return KDA_OK;
    if (tokens > 0x7fffffffLL)
        return fail(KDA_ERR_UNSUPPORTED, "B*T=%lld exceeds the 2^31 token limit of the TMA coordinates", tokens);
    char msg[256] = "";
    int rc;
    if (tokens == 0)
        rc = slots ? KDA_OK   // states stay in their slots
                   : kda::tc::state_passthrough(init_state, final_state, num_seqs, H, dk, dv, st, msg, sizeof(msg));
    else if (plan.window)
        rc = two_pass_windows(q, k, v, log_alpha, beta, init_state, o, final_state, T, H, dk, dv, plan.window,
                              gate_scalar, workspace, st, msg, sizeof(msg));
    else if (plan.algo == KDA_ALGO_TWO_PASS)
        rc = kda::tc::launch_two_pass(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, tokens, T,
                                      H, dk, dv, num_seqs, slots, num_slots, gate_scalar, workspace, st, msg,
                                      sizeof(msg));
    else
        rc = kda::tc::launch_fused(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, tokens, T, H,
                                   dk, dv, num_seqs, slots, num_slots, gate_scalar, st, msg, sizeof(msg));
    if (rc) return fail(rc, "%s", msg);
    return KDA_OK;
}

// Decode argument checks shared by both decode entry points.
int check_decode(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                 const float *state, const void *o, int N, int H, int dk, int dv, int dtype,
                 bool gate_scalar = false) {
    if (N < 0 || H < 1) return fail(KDA_ERR_INVALID_ARG, "bad sizes N=%d H=%d", N, H);
    if (N == 0) return KDA_OK;   // nothing to do; empty tensors may carry NULL pointers
    if (!q || !k || !v || !log_alpha || !beta || !state || !o)
        return fail(KDA_ERR_INVALID_ARG, "q, k, v, log_alpha, beta, state and o are required");
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128))
        return fail(KDA_ERR_UNSUPPORTED, "dk=%d dv=%d: each must be 64 or 128", dk, dv);
    if (dtype != KDA_BF16 && dtype != KDA_F32) return fail(KDA_ERR_UNSUPPORTED, "dtype=%d", dtype);
    const void *p16[] = {q, k, v, log_alpha, o, state};
    const char *n16[] = {"q", "k", "v", "log_alpha", "o", "state"};
    for (int i = 0; i < 6; ++i)
        if (!aligned(p16[i], (i == 3 && gate_scalar) ? 4 : 16))
            return fail(KDA_ERR_MISALIGNED, "%s is not %d-byte aligned", n16[i], (i == 3 && gate_scalar) ? 4 : 16);
    if (!aligned(beta, 4)) return fail(KDA_ERR_MISALIGNED, "beta is not 4-byte aligned");
    if ((long long)N * H > 0x7fffffffLL) return fail(KDA_ERR_UNSUPPORTED, "N*H=%lld too large", (long long)N * H);
    return KDA_OK;
}

int decode_impl(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                float *state, void *o, int N, int H, int dk, int dv, int dtype, const int32_t *slots,
                int num_slots, bool gate_scalar, cudaStream_t st, bool prologue = false) {
    const long long pairs = (long long)N * H;
    if (pairs == 0) return KDA_OK;
#define KDA_DEC_ARGS (q, k, v, log_alpha, beta, state, o, pairs, slots, num_slots, H, st)
#define KDA_DEC1(DKv, DVv, TT)                                                      \
    return gate_scalar ? launch_decode<DKv, DVv, TT, true, false> KDA_DEC_ARGS       \
           : prologue  ? launch_decode<DKv, DVv, TT, false, true> KDA_DEC_ARGS       \
                       : launch_decode<DKv, DVv, TT, false, false> KDA_DEC_ARGS;
#define KDA_DEC(DKv, DVv)                             \
    if (dk == DKv && dv == DVv) {                     \
        if (dtype == KDA_BF16) KDA_DEC1(DKv, DVv, __nv_bfloat16) \
        KDA_DEC1(DKv, DVv, float)                     \
    }
    KDA_DEC(64, 64)
    KDA_DEC(64, 128)
    KDA_DEC(128, 64)
    KDA_DEC(128, 128)
#undef KDA_DEC
#undef KDA_DEC1
#undef KDA_DEC_ARGS
    return fail(KDA_ERR_UNSUPPORTED, "dk=%d dv=%d", dk, dv);
}

template <typename K>
int set_smem(K kern, size_t bytes, const char *what) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    return e == cudaSuccess ? KDA_OK : cuda_fail(e, what);
}

template <int DK, typename Tin, bool GS>
int launch_backward(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                    const float *init_state, const void *d_o, const float *dfinal, void *dq, void *dk_out,
                    void *dv_out, float *dlog_alpha, float *dbeta, float *dinit_state, const int32_t *cu_seqlens,
                    long long tokens, int T, int H, int dv, int num_seqs, void *workspace, cudaStream_t st) {
    namespace b = kda::bwd;
    auto k_prep = b::bwd_prep_kernel<DK, Tin, GS>;
    auto k_state = b::bwd_state_kernel<DK, Tin>;
    auto k_part = b::bwd_part_kernel<DK, Tin>;
    auto k_chunk = b::bwd_chunk_kernel<DK, Tin, GS>;
    int rc;
    if ((rc = set_smem(k_prep, b::PrepSmem<DK>::bytes, "cudaFuncSetAttribute(bwd_prep)"))) return rc;
    if ((rc = set_smem(k_state, b::StateSmem<DK>::bytes, "cudaFuncSetAttribute(bwd_state)"))) return rc;
    if ((rc = set_smem(k_part, b::PartSmem<DK>::bytes, "cudaFuncSetAttribute(bwd_part)"))) return rc;
    if ((rc = set_smem(k_chunk, b::ChunkSmem<DK>::bytes, "cudaFuncSetAttribute(bwd_chunk)"))) return rc;
    const long long slots = tokens > 0 ? b::chunk_slots(tokens, num_seqs) : 0;
    const size_t sh = (size_t)slots * H;
    float *rec = (float *)workspace;
    float *ckpt = tokens > 0 ? rec + sh * b::Rec<DK>::FLOATS : nullptr;
    float *dckpt = tokens > 0 ? ckpt + sh * DK * dv : nullptr;
    float *part = tokens > 0 ? dckpt + sh * DK * dv : nullptr;
    const dim3 per_chunk((unsigned)slots, H);
    cudaError_t e;
    if (tokens > 0) {
        k_prep<<<per_chunk, b::PREP_NT, b::PrepSmem<DK>::bytes, st>>>((const Tin *)q, (const Tin *)k, log_alpha, beta,
                                                                  cu_seqlens, T, H, num_seqs, rec);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "bwd_prep launch");
    }
    k_state<<<dim3(2 * (dv / b::SV), H, num_seqs), b::NT, b::StateSmem<DK>::bytes, st>>>(
        (const Tin *)v, init_state, (const Tin *)d_o, dfinal, dinit_state, cu_seqlens, T, H, dv, rec, ckpt, dckpt);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "bwd_state launch");
    if (tokens > 0) {
        k_part<<<per_chunk, b::PartThreads<Tin>::value, b::PartSmem<DK>::bytes, st>>>((const Tin *)v, beta, (const Tin *)d_o,
                                                                  (Tin *)dv_out, cu_seqlens, T, H, dv, num_seqs,
                                                                  rec, ckpt, dckpt, part);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "bwd_part launch");
        k_chunk<<<per_chunk, b::CHUNK_NT, b::ChunkSmem<DK>::bytes, st>>>((const Tin *)q, (const Tin *)k, log_alpha,
                                                                    beta, cu_seqlens, T, H, num_seqs, part,
                                                                    (Tin *)dq, (Tin *)dk_out, dlog_alpha, dbeta);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "bwd_chunk launch");
    }
    return KDA_OK;
}

// The tensor-core backward covers bf16 inputs with dk = dv = 128 (either gate).
bool backward_tc_eligible(int dtype, int dk, int dv, bool gate_scalar) {
    (void)gate_scalar;
    return dtype == KDA_BF16 && dk == 128 && dv == 128;
}

// Workspace bytes of the backward path that `algo` selects (0 for an unusable choice).
size_t backward_ws(long long tokens, int H, int dk, int dv, int num_seqs, int dtype, bool gate_scalar, int algo) {
    const bool tc = backward_tc_eligible(dtype, dk, dv, gate_scalar);
    if (algo == KDA_BWD_TENSOR && !tc) return 0;
    if (tc && algo != KDA_BWD_SIMT) return kda::tc::backward_tc_workspace_bytes(tokens, H, num_seqs);
    return kda::bwd::backward_workspace_bytes(tokens, H, dk, dv, num_seqs);
}

// Every backward entry point after the shared checks; gate_scalar: Gated DeltaNet.
int backward_impl(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                  const float *init_state, const void *d_o, const float *dfinal_state, void *dq, void *dk_out,
                  void *dv_out, float *dlog_alpha, float *dbeta, float *dinit_state, const int32_t *cu_seqlens,
                  int B, int T, int H, int dk, int dv, int num_seqs, int dtype, int chunk, void *workspace,
                  size_t ws_bytes, void *stream, bool gate_scalar, int algo = KDA_BWD_AUTO) {
    if (algo != KDA_BWD_AUTO && algo != KDA_BWD_TENSOR && algo != KDA_BWD_SIMT)
        return fail(KDA_ERR_INVALID_ARG, "unknown backward algo %d", algo);
    // The forward checks cover the inputs (o stands in for d_o).
    int rc = check_prefill(q, k, v, log_alpha, beta, init_state, d_o, dfinal_state, cu_seqlens, B, T, H, dk, dv,
                           num_seqs, dtype, chunk, gate_scalar);
    if (rc) return rc;
    if (T > 0 && (!dq || !dk_out || !dv_out || !dlog_alpha || !dbeta))
        return fail(KDA_ERR_INVALID_ARG, "dq, dk, dv, dlog_alpha and dbeta are required");
    const void *p16[] = {dq, dk_out, dv_out, gate_scalar ? nullptr : dlog_alpha, dinit_state};
    const char *n16[] = {"dq", "dk", "dv", "dlog_alpha", "dinit_state"};
    for (int i = 0; i < 5; ++i)
        if (p16[i] && !aligned(p16[i], 16)) return fail(KDA_ERR_MISALIGNED, "%s is not 16-byte aligned", n16[i]);
    if (dbeta && !aligned(dbeta, 4)) return fail(KDA_ERR_MISALIGNED, "dbeta is not 4-byte aligned");
    if (gate_scalar && dlog_alpha && !aligned(dlog_alpha, 4))
        return fail(KDA_ERR_MISALIGNED, "dlog_alpha is not 4-byte aligned");
    const long long tokens = (long long)B * T;
    const bool use_tc = backward_tc_eligible(dtype, dk, dv, gate_scalar) && algo != KDA_BWD_SIMT;
    if (algo == KDA_BWD_TENSOR && !use_tc)
        return fail(KDA_ERR_UNSUPPORTED, "the tensor-core backward takes bf16 inputs with dk = dv = 128");
    const size_t need = backward_ws(tokens, H, dk, dv, num_seqs, dtype, gate_scalar, algo);
    if (need > 0 && (!workspace || ws_bytes < need))
        return fail(KDA_ERR_WORKSPACE, "backward workspace of %zu bytes needed, %zu given%s", need, ws_bytes,
                    workspace ? "" : " (NULL)");
    if (workspace && !aligned(workspace, 16)) return fail(KDA_ERR_MISALIGNED, "workspace is not 16-byte aligned");
    if (kda::bwd::chunk_slots(tokens, num_seqs) > 0x7fffffffLL)
        return fail(KDA_ERR_UNSUPPORTED, "too many chunk slots for one grid");
    if (num_seqs == 0) return KDA_OK;
    cudaStream_t st = (cudaStream_t)stream;
    if (use_tc) {
        char msg[256] = "";
        const int rc2 =
            gate_scalar
                ? kda::tc::launch_backward_tc<true>(q, k, v, log_alpha, beta, init_state, d_o, dfinal_state, dq, dk_out,
                                                    dv_out, dlog_alpha, dbeta, dinit_state, cu_seqlens, tokens, T, H,
                                                    num_seqs, workspace, st, msg, sizeof(msg))
                : kda::tc::launch_backward_tc<false>(q, k, v, log_alpha, beta, init_state, d_o, dfinal_state, dq,
                                                     dk_out, dv_out, dlog_alpha, dbeta, dinit_state, cu_seqlens,
                                                     tokens, T, H, num_seqs, workspace, st, msg, sizeof(msg));
        return rc2 ? fail(rc2, "%s", msg) : KDA_OK;
    }
#define KDA_BWD_ARGS                                                                                      \
    (q, k, v, log_alpha, beta, init_state, d_o, dfinal_state, dq, dk_out, dv_out, dlog_alpha, dbeta, dinit_state, \
     cu_seqlens, tokens, T, H, dv, num_seqs, workspace, st)
#define KDA_BWD(DKv, TT) \
    return gate_scalar ? launch_backward<DKv, TT, true> KDA_BWD_ARGS : launch_backward<DKv, TT, false> KDA_BWD_ARGS
    if (dtype == KDA_BF16) {
        if (dk == 64) KDA_BWD(64, __nv_bfloat16);
        KDA_BWD(128, __nv_bfloat16);
    }
    if (dk == 64) KDA_BWD(64, float);
    KDA_BWD(128, float);
#undef KDA_BWD
#undef KDA_BWD_ARGS
}

}  // namespace

namespace kda {
// An mbarrier that expects one arrival nobody makes: every thread's bounded wait
// runs out after limit_cycles and the CTA flags the timeout like a real kernel.
__global__ void wait_timeout_kernel(long long limit_cycles) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t addr = ptx::smem_u32(&bar);
    if (threadIdx.x == 0) {
        ptx::mbar_init(addr, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    const bool ok = ptx::mbar_wait_bounded(addr, 0u, limit_cycles);
    if (__syncthreads_or(!ok) && threadIdx.x == 0) flag_status(KDA_DEV_WAIT_TIMEOUT);
}
}  // namespace kda

extern "C" {

int kda_api_version(void) { return KDA_API_VERSION; }

const char *kda_last_error(void) { return g_err; }

size_t kda_chunk_forward_workspace_size_ex(int B, int T, int H, int dk, int dv, int num_seqs, int dtype,
                                           int chunk, int algo) {
    (void)dv; (void)chunk;
    if (dtype != KDA_BF16 || B < 1 || T < 0 || H < 1 || num_seqs < 0 || (dk != 64 && dk != 128)) return 0;
    return plan_prefill(B, (long long)B * T, H, dk, dv, num_seqs, algo).ws;
}

size_t kda_set_auto_workspace_limit(size_t bytes) {
    return g_auto_ws_limit.exchange(bytes ? bytes : kAutoTwoPassDefault);
}

size_t kda_chunk_forward_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs, int dtype,
                                        int chunk) {
    return kda_chunk_forward_workspace_size_ex(B, T, H, dk, dv, num_seqs, dtype, chunk, KDA_ALGO_AUTO);
}

int kda_chunk_forward_simt(const void *q, const void *k, const void *v, const float *log_alpha,
                           const float *beta, const float *init_state, void *o, float *final_state,
                           const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv, int num_seqs,
                           int dtype, int chunk, void *stream) {
    int rc = check_prefill(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, B, T, H, dk,
                           dv, num_seqs, dtype, chunk);
    if (rc) return rc;
    return simt_impl(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, T, H, dk, dv, num_seqs,
                     dtype, nullptr, 0, false, (cudaStream_t)stream);
}

int kda_chunk_forward_ex(const void *q, const void *k, const void *v, const float *log_alpha,
                         const float *beta, const float *init_state, void *o, float *final_state,
                         const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv, int num_seqs,
                         int dtype, int chunk, int algo, void *workspace, size_t ws_bytes, void *stream) {
    int rc = check_prefill(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, B, T, H, dk,
                           dv, num_seqs, dtype, chunk);
    if (rc) return rc;
    if (algo != KDA_ALGO_AUTO && algo != KDA_ALGO_FUSED && algo != KDA_ALGO_TWO_PASS)
        return fail(KDA_ERR_INVALID_ARG, "algo=%d is not a KDA_ALGO_* value", algo);
    if (dtype == KDA_F32)
        return simt_impl(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, T, H, dk, dv,
                         num_seqs, dtype, nullptr, 0, false, (cudaStream_t)stream);
    return prefill_impl(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, B, T, H, dk, dv,
                        num_seqs, algo, nullptr, 0, false, workspace, ws_bytes, (cudaStream_t)stream);
}

int kda_chunk_forward_slots(const void *q, const void *k, const void *v, const float *log_alpha,
                            const float *beta, float *state_pool, const int32_t *slots, void *o,
                            const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv, int num_seqs,
                            int num_slots, int dtype, int chunk, int algo, void *workspace, size_t ws_bytes,
                            void *stream) {
    int rc = check_prefill(q, k, v, log_alpha, beta, state_pool, o, state_pool, cu_seqlens, B, T, H, dk, dv,
                           num_seqs, dtype, chunk);
    if (rc) return rc;
    if (num_seqs > 0 && (!state_pool || !slots))
        return fail(KDA_ERR_INVALID_ARG, "state_pool and slots are required");
    if (num_slots < 1) return fail(KDA_ERR_INVALID_ARG, "num_slots=%d must be at least 1", num_slots);
    if (slots && !aligned(slots, 4)) return fail(KDA_ERR_MISALIGNED, "slots is not 4-byte aligned");
    if (algo != KDA_ALGO_AUTO && algo != KDA_ALGO_FUSED && algo != KDA_ALGO_TWO_PASS)
        return fail(KDA_ERR_INVALID_ARG, "algo=%d is not a KDA_ALGO_* value", algo);
    if (dtype == KDA_F32)
        return simt_impl(q, k, v, log_alpha, beta, state_pool, o, state_pool, cu_seqlens, T, H, dk, dv,
                         num_seqs, dtype, slots, num_slots, false, (cudaStream_t)stream);
    return prefill_impl(q, k, v, log_alpha, beta, state_pool, o, state_pool, cu_seqlens, B, T, H, dk, dv,
                        num_seqs, algo, slots, num_slots, false, workspace, ws_bytes, (cudaStream_t)stream);
}

int kda_chunk_forward(const void *q, const void *k, const void *v, const float *log_alpha,
                      const float *beta, const float *init_state, void *o, float *final_state,
                      const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv, int num_seqs,
                      int dtype, int chunk, void *workspace, size_t ws_bytes, void *stream) {
    return kda_chunk_forward_ex(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, B, T, H, dk,
                                dv, num_seqs, dtype, chunk, KDA_ALGO_AUTO, workspace, ws_bytes, stream);
}

int kda_chunk_forward_static_ws(const void *q, const void *k, const void *v, const float *log_alpha,
                                const float *beta, const float *init_state, void *o, float *final_state,
                                const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv, int num_seqs,
                                int dtype, int chunk, void *stream) {
    int rc = check_prefill(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, B, T, H, dk,
                           dv, num_seqs, dtype, chunk);
    if (rc) return rc;
    if (dtype == KDA_F32)
        return kda_chunk_forward_simt(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, B,
                                      T, H, dk, dv, num_seqs, dtype, chunk, stream);
    const size_t need = plan_prefill(B, (long long)B * T, H, dk, dv, num_seqs, KDA_ALGO_TWO_PASS).ws;
    // Too large for the built-in scratch: the fused schedule, which needs no scratch at all.
    if (need > KDA_STATIC_WS_BYTES)
        return kda_chunk_forward_ex(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, B, T, H, dk,
                                    dv, num_seqs, dtype, chunk, KDA_ALGO_FUSED, nullptr, 0, stream);
    if (num_seqs == 0) return KDA_OK;
    void *ws = nullptr;
    if (need) {
        cudaError_t e = cudaSuccess;
        ws = static_ws_address(&e);
        if (!ws) return cuda_fail(e, "looking up the built-in scratch (cudaGetSymbolAddress)");
    }
    return kda_chunk_forward_ex(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, B, T, H, dk,
                                dv, num_seqs, dtype, chunk, KDA_ALGO_TWO_PASS, ws, need, stream);
}

int kda_recurrent_step(const void *q, const void *k, const void *v, const float *log_alpha,
                       const float *beta, float *state, void *o, int N, int H, int dk, int dv, int dtype,
                       void *stream) {
    int rc = check_decode(q, k, v, log_alpha, beta, state, o, N, H, dk, dv, dtype);
    if (rc || N == 0) return rc;
    return decode_impl(q, k, v, log_alpha, beta, state, o, N, H, dk, dv, dtype, nullptr, 0, false,
                       (cudaStream_t)stream);
}

int kda_recurrent_step_slots(const void *q, const void *k, const void *v, const float *log_alpha,
                             const float *beta, float *state_pool, const int32_t *slots, void *o, int N, int H,
                             int dk, int dv, int num_slots, int dtype, void *stream) {
    int rc = check_decode(q, k, v, log_alpha, beta, state_pool, o, N, H, dk, dv, dtype);
    if (rc || N == 0) return rc;
    if (!slots) return fail(KDA_ERR_INVALID_ARG, "slots is required");
    if (!aligned(slots, 4)) return fail(KDA_ERR_MISALIGNED, "slots is not 4-byte aligned");
    if (num_slots < 1) return fail(KDA_ERR_INVALID_ARG, "num_slots=%d must be at least 1", num_slots);
    return decode_impl(q, k, v, log_alpha, beta, state_pool, o, N, H, dk, dv, dtype, slots, num_slots, false,
                       (cudaStream_t)stream);
}

int kda_gdn_chunk_forward(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, const float *init_state, void *o, float *final_state,
                          const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv, int num_seqs, int dtype,
                          int chunk, int algo, void *workspace, size_t ws_bytes, void *stream) {
    int rc = check_prefill(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, B, T, H, dk,
                           dv, num_seqs, dtype, chunk, true);
    if (rc) return rc;
    if (algo != KDA_ALGO_AUTO && algo != KDA_ALGO_FUSED && algo != KDA_ALGO_TWO_PASS)
        return fail(KDA_ERR_INVALID_ARG, "algo=%d is not a KDA_ALGO_* value", algo);
    if (dtype == KDA_F32)
        return simt_impl(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, T, H, dk, dv,
                         num_seqs, dtype, nullptr, 0, true, (cudaStream_t)stream);
    return prefill_impl(q, k, v, log_alpha, beta, init_state, o, final_state, cu_seqlens, B, T, H, dk, dv,
                        num_seqs, algo, nullptr, 0, true, workspace, ws_bytes, (cudaStream_t)stream);
}

int kda_gdn_recurrent_step(const void *q, const void *k, const void *v, const float *log_alpha,
                           const float *beta, float *state, void *o, int N, int H, int dk, int dv, int dtype,
                           void *stream) {
    int rc = check_decode(q, k, v, log_alpha, beta, state, o, N, H, dk, dv, dtype, true);
    if (rc || N == 0) return rc;
    return decode_impl(q, k, v, log_alpha, beta, state, o, N, H, dk, dv, dtype, nullptr, 0, true,
                       (cudaStream_t)stream);
}

int kda_chunk_forward_prologue(const void *q_raw, const void *k_raw, const void *v, const void *gate_x,
                               const float *beta, const float *init_state, void *o, float *final_state,
                               const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv, int num_seqs,
                               int dtype, int chunk, int algo, void *workspace, size_t ws_bytes, void *stream) {
    int rc = check_prefill(q_raw, k_raw, v, (const float *)gate_x, beta, init_state, o, final_state, cu_seqlens, B,
                           T, H, dk, dv, num_seqs, dtype, chunk);
    if (rc) return rc;
    if (algo != KDA_ALGO_AUTO && algo != KDA_ALGO_FUSED && algo != KDA_ALGO_TWO_PASS)
        return fail(KDA_ERR_INVALID_ARG, "algo=%d is not a KDA_ALGO_* value", algo);
    if (dtype == KDA_F32)
        return simt_impl(q_raw, k_raw, v, (const float *)gate_x, beta, init_state, o, final_state, cu_seqlens, T, H,
                         dk, dv, num_seqs, dtype, nullptr, 0, false, (cudaStream_t)stream, true);
    if (algo == KDA_ALGO_FUSED)
        return fail(KDA_ERR_UNSUPPORTED, "the fused schedule reads prepared inputs; use KDA_ALGO_TWO_PASS or AUTO");
    const long long tokens = (long long)B * T;
    const size_t need = kda::tc::two_pass_workspace_bytes(tokens, H, dk, num_seqs);
    if (need && (!workspace || ws_bytes < need))
        return fail(KDA_ERR_WORKSPACE, "workspace of %zu bytes required, got %zu", need, ws_bytes);
    if (workspace && !aligned(workspace, 256)) return fail(KDA_ERR_MISALIGNED, "workspace is not 256-byte aligned");
    if (num_seqs == 0) return KDA_OK;
    if (tokens > 0x7fffffffLL)
        return fail(KDA_ERR_UNSUPPORTED, "B*T=%lld exceeds the 2^31 token limit of the TMA coordinates", tokens);
    char msg[256] = "";
    cudaStream_t st = (cudaStream_t)stream;
    if (tokens == 0)
        rc = kda::tc::state_passthrough(init_state, final_state, num_seqs, H, dk, dv, st, msg, sizeof(msg));
    else
        rc = kda::tc::launch_two_pass(q_raw, k_raw, v, (const float *)gate_x, beta, init_state, o, final_state,
                                      cu_seqlens, tokens, T, H, dk, dv, num_seqs, nullptr, 0, false, workspace, st,
                                      msg, sizeof(msg), true);
    if (rc) return fail(rc, "%s", msg);
    return KDA_OK;
}

int kda_recurrent_step_prologue(const void *q_raw, const void *k_raw, const void *v, const void *gate_x,
                                const float *beta, float *state, void *o, int N, int H, int dk, int dv, int dtype,
                                void *stream) {
    int rc = check_decode(q_raw, k_raw, v, (const float *)gate_x, beta, state, o, N, H, dk, dv, dtype);
    if (rc) return rc;
    return decode_impl(q_raw, k_raw, v, (const float *)gate_x, beta, state, o, N, H, dk, dv, dtype, nullptr, 0, false,
                       (cudaStream_t)stream, true);
}

size_t kda_chunk_backward_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs) {
    if (B < 1 || T < 0 || H < 1 || num_seqs < 0 || (dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return 0;
    return kda::bwd::backward_workspace_bytes((long long)B * T, H, dk, dv, num_seqs);
}

size_t kda_chunk_backward_workspace_size_ex(int B, int T, int H, int dk, int dv, int num_seqs, int dtype, int algo) {
    if (B < 1 || T < 0 || H < 1 || num_seqs < 0 || (dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return 0;
    if (dtype != KDA_BF16 && dtype != KDA_F32) return 0;
    return backward_ws((long long)B * T, H, dk, dv, num_seqs, dtype, false, algo);
}

int kda_chunk_backward_ex(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                          const float *init_state, const void *d_o, const float *dfinal_state, void *dq, void *dk_out,
                          void *dv_out, float *dlog_alpha, float *dbeta, float *dinit_state,
                          const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv, int num_seqs, int dtype,
                          int chunk, void *workspace, size_t ws_bytes, void *stream, int algo) {
    return backward_impl(q, k, v, log_alpha, beta, init_state, d_o, dfinal_state, dq, dk_out, dv_out, dlog_alpha,
                         dbeta, dinit_state, cu_seqlens, B, T, H, dk, dv, num_seqs, dtype, chunk, workspace, ws_bytes,
                         stream, false, algo);
}

int kda_chunk_backward(const void *q, const void *k, const void *v, const float *log_alpha,
                       const float *beta, const float *init_state, const void *d_o,
                       const float *dfinal_state, void *dq, void *dk_out, void *dv_out, float *dlog_alpha,
                       float *dbeta, float *dinit_state, const int32_t *cu_seqlens, int B, int T, int H,
                       int dk, int dv, int num_seqs, int dtype, int chunk, void *workspace, size_t ws_bytes,
                       void *stream) {
    return backward_impl(q, k, v, log_alpha, beta, init_state, d_o, dfinal_state, dq, dk_out, dv_out, dlog_alpha,
                         dbeta, dinit_state, cu_seqlens, B, T, H, dk, dv, num_seqs, dtype, chunk, workspace, ws_bytes,
                         stream, false);
}

int kda_gdn_chunk_backward_ex(const void *q, const void *k, const void *v, const float *log_alpha,
                              const float *beta, const float *init_state, const void *d_o, const float *dfinal_state,
                              void *dq, void *dk_out, void *dv_out, float *dlog_alpha, float *dbeta,
                              float *dinit_state, const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv,
                              int num_seqs, int dtype, int chunk, void *workspace, size_t ws_bytes, void *stream,
                              int algo) {
    return backward_impl(q, k, v, log_alpha, beta, init_state, d_o, dfinal_state, dq, dk_out, dv_out, dlog_alpha,
                         dbeta, dinit_state, cu_seqlens, B, T, H, dk, dv, num_seqs, dtype, chunk, workspace, ws_bytes,
                         stream, true, algo);
}

int kda_gdn_chunk_backward(const void *q, const void *k, const void *v, const float *log_alpha,
                           const float *beta, const float *init_state, const void *d_o,
                           const float *dfinal_state, void *dq, void *dk_out, void *dv_out, float *dlog_alpha,
                           float *dbeta, float *dinit_state, const int32_t *cu_seqlens, int B, int T, int H,
                           int dk, int dv, int num_seqs, int dtype, int chunk, void *workspace, size_t ws_bytes,
                           void *stream) {
    return backward_impl(q, k, v, log_alpha, beta, init_state, d_o, dfinal_state, dq, dk_out, dv_out, dlog_alpha,
                         dbeta, dinit_state, cu_seqlens, B, T, H, dk, dv, num_seqs, dtype, chunk, workspace, ws_bytes,
                         stream, true);
}

int kda_debug_wait_timeout(long long limit_cycles, void *stream) {
    if (limit_cycles < 1 || limit_cycles > 2000000000ll)
        return fail(KDA_ERR_INVALID_ARG, "limit_cycles must lie in [1, 2e9], got %lld", limit_cycles);
    kda::wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(limit_cycles);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "wait_timeout_kernel launch");
    return KDA_OK;
}

int kda_get_device_status(unsigned int *bits, int clear, void *stream) {
    if (!bits) return fail(KDA_ERR_INVALID_ARG, "bits is required");
    cudaStream_t st = (cudaStream_t)stream;
    unsigned int host = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&host, kda::g_status, sizeof(host), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
    if (clear && host) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbolAsync(kda::g_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cuda_fail(e, "clearing the device status word");
    }
    *bits = host;
    if (host) return fail(KDA_ERR_DEVICE, "device status flags 0x%x", host);
    return KDA_OK;
}

}  // extern "C"
