/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention (KDA) operator.
 *
 * What the operator computes ("Kimi Delta Attention 徹底解説" (tech-tide.dev),
 * § "なぜ今「線形アテンション」なのか" and § "Kimi Delta Attention の仕組み";
 * "Kimi Linear、独自の土俵でFull Attentionを上回る" (remio.ai),
 * § "Kimi Linearがより賢いRecurrent Memoryを使う方法"): each (sequence, head)
 * keeps a fixed-size state S (dk x dv, fp32).  For every token t, in order,
 *
 *     S'  = Diag(alpha_t) S          alpha_t = exp(log_alpha_t), one rate per key channel
 *     S   = S' + beta_t k_t (v_t - S'^T k_t)^T
 *     o_t = S^T q_t
 *
 * Decode runs this token by token; prefill regroups the same computation into
 * 64-token chunks (same result up to rounding).  No normalisation of q or k and
 * no 1/sqrt(d) scale is applied inside the operator.
 *
 * Layouts (row-major, last index contiguous; every tensor dense, no strides):
 *   q, k        [B, T, H, dk]   dtype (bf16 or fp32)
 *   v, o        [B, T, H, dv]   dtype
 *   log_alpha   [B, T, H, dk]   fp32, must be <= 0 and finite
 *   beta        [B, T, H]       fp32
 *   states      [N, H, dk, dv]  fp32 (dv contiguous); the same layout for
 *                               prefill's init/final state and decode's state,
 *                               so a prefill's final_state is directly a valid
 *                               decode state (a state-layout mismatch between
 *                               chunked prefill and decode is the failure the
 *                               remio.ai page reports in § "オープンコードにより
 *                               主張は検証可能になる一方、ソフトウェアスタックは
 *                               リスクを加える").
 *   packed (varlen) prefill: B == 1, T = total tokens, cu_seqlens [N+1] int32 on
 *   the device, non-decreasing, cu_seqlens[0] == 0, cu_seqlens[N] == T;
 *   sequence n is tokens [cu_seqlens[n], cu_seqlens[n+1]) and the state never
 *   crosses a sequence boundary.  Without cu_seqlens, N == B and each batch row
 *   is one sequence of T tokens.
 *
 * Ownership and execution: the caller allocates and owns every buffer (device
 * memory unless stated).  The library never allocates, frees or synchronises
 * in these calls; work is enqueued on `stream` (a cudaStream_t passed as
 * void*, NULL = the legacy default stream) and the call returns immediately.
 * Pointers to tensors must be 16-byte aligned (beta and cu_seqlens: 4-byte).
 * Inputs must not alias outputs, except decode's in-place state.
 *
 * Errors: every call returns KDA_OK (0) or a negative kda_status.  Argument
 * errors are detected on the host before anything is enqueued (nothing runs).
 * A failed launch returns KDA_ERR_CUDA.  Conditions found on the device are
 * accumulated in a per-device status word read by kda_get_device_status().
 * kda_last_error() gives a message for the calling thread's last failure.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KDA_API_VERSION 1

typedef enum kda_status {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = -1,   /* NULL required pointer, bad shape or count */
    KDA_ERR_UNSUPPORTED = -2,   /* dk/dv not in {64, 128}, chunk != 64, bad dtype */
    KDA_ERR_MISALIGNED = -3,    /* pointer alignment below the requirement */
    KDA_ERR_CUDA = -4,          /* a CUDA runtime call or kernel launch failed */
    KDA_ERR_WORKSPACE = -5,     /* workspace missing or smaller than required */
    KDA_ERR_DEVICE = -6         /* kda_get_device_status() found a device-side flag */
} kda_status;

typedef enum kda_dtype {
    KDA_BF16 = 0,
    KDA_F32 = 1
} kda_dtype;

/* Device status word bits (kda_get_device_status). */
#define KDA_DEV_WAIT_TIMEOUT 0x1u    /* a bounded on-chip wait gave up; that CTA's output is invalid */
#define KDA_DEV_DECAY_RANGE 0x2u     /* reserved: no longer raised (the tensor-core prefill is exact
                                        for any log_alpha <= 0; see kda_chunk_forward) */
#define KDA_DEV_BAD_SLOT 0x4u        /* a state-slot table entry was outside [-1, num_slots); that
                                        sequence was treated as having no slot (see *_slots) */

/*
 * Chunked prefill, 64-token chunks.
 *
 * Source: the KDA recurrence above; the chunked regrouping is the prefill mode of
 * "Kimi Delta Attention 徹底解説" § "Kimi Delta Attention の仕組み" and the
 * chunkwise, diagonal-plus-low-rank form of "Kimi Linear、独自の土俵でFull Attention
 * を上回る" § "Kimi Linearがより賢いRecurrent Memoryを使う方法".
 *
 *   q, k, v       inputs in `dtype`, layouts above (required when T > 0)
 *   log_alpha     fp32 [B,T,H,dk]; beta fp32 [B,T,H] (required when T > 0)
 *   init_state    fp32 [N,H,dk,dv] or NULL (zeros)
 *   o             output [B,T,H,dv] in `dtype` (required when T > 0); rounded to nearest-even
 *   final_state   fp32 [N,H,dk,dv] or NULL (not written)
 *   cu_seqlens    int32 [N+1] device array or NULL (dense batch)
 *   B, T, H       batch, tokens per row, heads (T may be 0)
 *   dk, dv        64 or 128 each
 *   num_seqs      N; must equal B when cu_seqlens is NULL
 *   dtype         KDA_BF16: tensor-core (tcgen05) path, bf16 operands with fp32
 *                 accumulation; KDA_F32: fp32 CUDA-core path
 *   chunk         must be 64
 *   workspace     device scratch of at least kda_chunk_forward_workspace_size()
 *                 bytes, 256-byte aligned (may be NULL when that size is 0)
 *
 * Decay range: both paths are exact for every finite log_alpha <= 0, however
 * strong (a channel may forget everything in one token).  The tensor-core path
 * splits the pairwise decay e^{G_i - G_j} of a chunk into two bf16 operands whose
 * factors stay within e^{+-80}: against the chunk start when every channel's
 * decay summed over the chunk is >= -80, else against 16-token block starts, with
 * the diagonal 16 x 16 terms of any block that decays by more than e^80 added in
 * fp32.  Chunks of strong decay cost more (about four times the Gram products).
 */
size_t kda_chunk_forward_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs,
                                        int dtype, int chunk);

int kda_chunk_forward(const void *q, const void *k, const void *v, const float *log_alpha,
                      const float *beta, const float *init_state, void *o, float *final_state,
                      const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv, int num_seqs,
                      int dtype, int chunk, void *workspace, size_t ws_bytes, void *stream);

/*
 * Schedules of the tensor-core prefill.  Both compute the same chunk algebra in
 * the same precision; they differ in where the state-independent part of each
 * chunk (decay factors, Gram matrix, UT transform, Kt = Kbar^T T Diag(beta),
 * Pt = Aqk T Diag(beta)) is built.
 *
 *   KDA_ALGO_FUSED     one kernel; each CTA (value-column tile, head, sequence)
 *                      builds it inside its serial walk over the chunks.  No
 *                      workspace.  Best when there are many (sequence, head)
 *                      chains.
 *   KDA_ALGO_TWO_PASS  a first kernel builds it for every (chunk, head) at once
 *                      into the workspace (about 57 KB per chunk and head at
 *                      dk = 128, 33 KB at dk = 64); a second kernel walks the
 *                      chunks with only the state-dependent products left.
 *                      Best when there are few chains.
 *   KDA_ALGO_AUTO      TWO_PASS when num_seqs * H < 296 and its workspace fits
 *                      AUTO's budget (1 GiB unless kda_set_auto_workspace_limit
 *                      says otherwise).  A single sequence (B = 1, num_seqs = 1)
 *                      whose workspace would not fit runs TWO_PASS in windows:
 *                      consecutive slices of the tokens, each one launch pair
 *                      on the same records, the state handed from one window to
 *                      the next in fp32 (the result is the one-pair result), so
 *                      its workspace stays within the budget at any length.
 *                      Everything else runs FUSED.  A windowed plan called with
 *                      cu_seqlens or state slots runs FUSED instead.
 *                      kda_chunk_forward uses AUTO.
 */
#define KDA_ALGO_AUTO 0
#define KDA_ALGO_FUSED 1
#define KDA_ALGO_TWO_PASS 2

/* Sets AUTO's workspace budget in bytes (0 restores the default of 1 GiB) and
 * returns the previous one.  Process-wide; the workspace size a call needs is the
 * one kda_chunk_forward_workspace_size_ex reports under the budget in force at
 * that call, so change it between calls, not between a size query and its call
 * (a smaller workspace than the plan needs is KDA_ERR_WORKSPACE). */
size_t kda_set_auto_workspace_limit(size_t bytes);

/* Workspace bytes kda_chunk_forward_ex needs for these sizes and `algo` (0 when none). */
size_t kda_chunk_forward_workspace_size_ex(int B, int T, int H, int dk, int dv, int num_seqs,
                                           int dtype, int chunk, int algo);

/* kda_chunk_forward with an explicit schedule (KDA_ALGO_*; ignored for KDA_F32, which
 * always takes the fp32 CUDA-core path).  An unknown `algo` is KDA_ERR_INVALID_ARG. */
int kda_chunk_forward_ex(const void *q, const void *k, const void *v, const float *log_alpha,
                         const float *beta, const float *init_state, void *o, float *final_state,
                         const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv, int num_seqs,
                         int dtype, int chunk, int algo, void *workspace, size_t ws_bytes, void *stream);

/*
 * kda_chunk_forward_static_ws: the two-pass prefill (KDA_ALGO_TWO_PASS) without a
 * caller workspace.  It allocates nothing: its scratch is one file-scope device
 * array of KDA_STATIC_WS_BYTES inside libkda, reserved on each device when the
 * library's device code is loaded there.  The pages have no counterpart of this
 * call; it exists for callers that cannot allocate device memory at call time:
 * code inside a region that forbids allocation (a latency-critical serving loop
 * that must not enter an allocator, or a stream-ordered section whose allocator
 * would synchronise), plain-C hosts with no device allocator of their own, and
 * callers already at their memory limit.
 *
 *   arguments     as kda_chunk_forward, without workspace / ws_bytes
 *   capacity      when the two-pass workspace for these sizes
 *                 (kda_chunk_forward_workspace_size_ex(..., KDA_ALGO_TWO_PASS))
 *                 fits in KDA_STATIC_WS_BYTES the two-pass schedule runs on the
 *                 built-in scratch; larger sizes run the fused schedule
 *                 (KDA_ALGO_FUSED), which needs no scratch at all, so no size is
 *                 refused for lack of room
 *   KDA_F32       takes the fp32 CUDA-core path, which needs no scratch
 *   zeroing       nothing in the scratch has to start at zero: the first pass
 *                 writes every record the second pass reads
 *   first call    on each device the scratch address is looked up with
 *                 cudaGetSymbolAddress and kept with the identity of the current
 *                 context; after cudaDeviceReset (or any new primary context) the
 *                 next call looks it up again.  Make the first call on a device,
 *                 and the first after a reset, outside stream capture
 *   concurrency   all calls on one device share the one scratch array: calls
 *                 that can overlap in time (different streams, or host threads
 *                 without ordering) race and corrupt each other's results;
 *                 order them on one stream
 */
#define KDA_STATIC_WS_BYTES ((size_t)64 << 20)

int kda_chunk_forward_static_ws(const void *q, const void *k, const void *v, const float *log_alpha,
                                const float *beta, const float *init_state, void *o, float *final_state,
                                const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv,
                                int num_seqs, int dtype, int chunk, void *stream);

/*
 * Same contract as kda_chunk_forward, computed entirely on CUDA cores in fp32
 * (inputs in either dtype are widened exactly).  The accuracy reference for the
 * tensor-core path and the path taken for KDA_F32.  Needs no workspace.
 */
int kda_chunk_forward_simt(const void *q, const void *k, const void *v, const float *log_alpha,
                           const float *beta, const float *init_state, void *o, float *final_state,
                           const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv,
                           int num_seqs, int dtype, int chunk, void *stream);

/*
 * One decode step for N sequences: the token recurrence with T = 1, state
 * updated in place.  Source: the recurrence above ("Kimi Delta Attention 徹底解説"
 * § "Kimi Delta Attention の仕組み": decode is the token-by-token recurrence).
 *
 *   q, k     [N, H, dk] in dtype;  v, o [N, H, dv] in dtype
 *   log_alpha fp32 [N, H, dk];     beta fp32 [N, H]
 *   state    fp32 [N, H, dk, dv], read once and written once (in place)
 * N == 0 is a no-op (pointers may then be NULL).
 * Each state is streamed once from HBM and written back once.
 */
int kda_recurrent_step(const void *q, const void *k, const void *v, const float *log_alpha,
                       const float *beta, float *state, void *o, int N, int H, int dk, int dv,
                       int dtype, void *stream);

/*
 * State slots: the states live in a pool and each sequence names its slot, the
 * layout serving stacks use for batched decode with continuous batching and for
 * prefix caching (a prefill that resumes from a cached prefix state).  Sources:
 * "Kimi Linear、独自の土俵でFull Attentionを上回る" (remio.ai), § "オープンコードに
 * より主張は検証可能になる一方、ソフトウェアスタックはリスクを加える" (batched
 * decode, prefix caching and state across chunk boundaries as the behaviour to
 * test) and § "Kimi Linearリリース後に注目すべき点" (prefix reuse, continuous
 * batching); "Kimi Linearは広がりつつある…" (orcarouter.ai), § "既に起こった採用は
 * サービングスタックの中にあります" (KDA prefix caching in serving stacks).
 *
 *   state_pool   fp32 [num_slots, H, dk, dv] (dv contiguous), updated in place
 *   slots        int32 [N] device array: slot of sequence n, or -1 for "no state"
 *                (prefill: start from zeros and write nothing back; decode: a
 *                padding row whose output is zero).  Entries outside
 *                [-1, num_slots) set KDA_DEV_BAD_SLOT and count as -1.  Two
 *                sequences must not name the same slot in one call (their
 *                updates would race).
 * Everything else is as in kda_chunk_forward_ex / kda_recurrent_step; the
 * workspace is kda_chunk_forward_workspace_size_ex's for the same sizes and algo.
 */
int kda_chunk_forward_slots(const void *q, const void *k, const void *v, const float *log_alpha,
                            const float *beta, float *state_pool, const int32_t *slots, void *o,
                            const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv, int num_seqs,
                            int num_slots, int dtype, int chunk, int algo, void *workspace, size_t ws_bytes,
                            void *stream);

int kda_recurrent_step_slots(const void *q, const void *k, const void *v, const float *log_alpha,
                             const float *beta, float *state_pool, const int32_t *slots, void *o, int N, int H,
                             int dk, int dv, int num_slots, int dtype, void *stream);

/*
 * Gated DeltaNet: the same recurrence with one decay rate per (token, head)
 * instead of one per key channel, S' = alpha_t S with a scalar alpha_t
 * ("Kimi Delta Attention 徹底解説" (tech-tide.dev), § "Kimi Delta Attention の仕組み":
 * Gated DeltaNet decays the whole state by one scalar, KDA makes it a diagonal
 * matrix; "Kimi Linearは広がりつつある…" (orcarouter.ai): serving stacks ship fused
 * KDA and Gated DeltaNet kernels).  The same kernels run with the gate read as a
 * scalar, so the gate stream is 4 instead of 4 dk bytes per token-head.
 *
 *   log_alpha   fp32 [B, T, H] (prefill) or [N, H] (decode), 4-byte aligned;
 *               every other argument, the workspace (kda_chunk_forward_workspace_size_ex
 *               with the same sizes and algo) and the error behaviour are as in
 *               kda_chunk_forward_ex / kda_recurrent_step.
 */
int kda_gdn_chunk_forward(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, const float *init_state, void *o, float *final_state,
                          const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv, int num_seqs, int dtype,
                          int chunk, int algo, void *workspace, size_t ws_bytes, void *stream);

int kda_gdn_recurrent_step(const void *q, const void *k, const void *v, const float *log_alpha,
                           const float *beta, float *state, void *o, int N, int H, int dk, int dv, int dtype,
                           void *stream);

/*
 * Fused input prologue: the operator on raw inputs, with the two input steps
 * that precede it done inside the kernels instead of as separate passes over
 * memory -- q and k scaled to unit L2 norm over the key axis (row / max(|row|_2,
 * 1e-6)), and the per-channel decay from the gate pre-activation x,
 * log_alpha = -softplus(x), i.e. alpha = 1 / (1 + e^x).  "Kimi Linear、独自の土俵で
 * Full Attentionを上回る" (remio.ai), § "Kimi Linearがより賢いRecurrent Memoryを使う
 * 方法" computes the decay per channel from the current token; the pages leave
 * the parametrisation open, and this is its plainest form with alpha in (0, 1).
 * The gate stream is x in the input dtype (2 dk bytes per token-head for bf16
 * instead of 4 dk for fp32 log_alpha).
 *
 *   q_raw, k_raw  [B, T, H, dk] in dtype, any scale (zero rows stay zero).
 *   gate_x        [B, T, H, dk] (prefill) or [N, H, dk] (decode) in dtype,
 *                 16-byte aligned.
 * Every other argument and the error behaviour are as in kda_chunk_forward_ex /
 * kda_recurrent_step.  dtype KDA_BF16 runs the two-pass tensor-core schedule
 * (AUTO means TWO_PASS here; its workspace is
 * kda_chunk_forward_workspace_size_ex(..., KDA_ALGO_TWO_PASS); KDA_ALGO_FUSED is
 * KDA_ERR_UNSUPPORTED), KDA_F32 the fp32 CUDA-core path.
 */
int kda_chunk_forward_prologue(const void *q_raw, const void *k_raw, const void *v, const void *gate_x,
                               const float *beta, const float *init_state, void *o, float *final_state,
                               const int32_t *cu_seqlens, int B, int T, int H, int dk, int dv, int num_seqs,
                               int dtype, int chunk, int algo, void *workspace, size_t ws_bytes, void *stream);

int kda_recurrent_step_prologue(const void *q_raw, const void *k_raw, const void *v, const void *gate_x,
                                const float *beta, float *state, void *o, int N, int H, int dk, int dv, int dtype,
                                void *stream);

/*
 * Backward of the chunked prefill: the gradients of
 *     L = sum_t <d_o_t, o_t> + <dfinal_state, final_state>
 * with respect to every input of kda_chunk_forward -- what the chunkwise
 * training algorithm needs ("Kimi Linear、独自の土俵でFull Attentionを上回る"
 * (remio.ai), § "Kimi Linearがより賢いRecurrent Memoryを使う方法"), for the
 * recurrence of "Kimi Delta Attention 徹底解説" (tech-tide.dev),
 * § "Kimi Delta Attention の仕組み".  Tensor-core products with fp32
 * accumulation (split tf32 for KDA_F32, keeping fp32 accuracy; bf16 and tf32
 * operands for KDA_BF16), and no decay-range precondition: decay factors pass
 * through 16-token block boundaries with both factors <= 1, and within a block
 * take the exact pairwise exponent unless every channel's in-block decay is
 * small enough to factor too.  For dtype KDA_BF16 and KDA_F32.
 *
 *   q, k, v, log_alpha, beta, init_state, cu_seqlens, B, T, H, dk, dv,
 *   num_seqs, dtype, chunk
 *                 the forward call's inputs, layouts and rules as in
 *                 kda_chunk_forward (init_state NULL = zeros).
 *   d_o           [B, T, H, dv] in dtype: dL/do.
 *   dfinal_state  fp32 [N, H, dk, dv] or NULL (zero): dL/dfinal_state.
 *   dq, dk_out    [B, T, H, dk] in dtype;  dv_out [B, T, H, dv] in dtype.
 *   dlog_alpha    fp32 [B, T, H, dk];  dbeta fp32 [B, T, H].
 *   dinit_state   fp32 [N, H, dk, dv], or NULL (not computed): dL/dinit_state,
 *                 the gradient at the given initial state (at zero when
 *                 init_state is NULL).
 *   workspace     device memory of at least kda_chunk_backward_workspace_size()
 *                 bytes for the same sizes (enough for either schedule; the
 *                 schedule this call takes needs kda_chunk_backward_workspace_size_ex
 *                 with KDA_BWD_AUTO), 16-byte aligned; no contents are required.
 *                 It holds per (64-token chunk slot, head) what the schedules
 *                 below keep between their launches: about 145 KB for the
 *                 tensor-core schedule, 570 KB for the SIMT one (dk = dv = 128).
 *                 Calls that can overlap in time need separate workspaces.  A
 *                 long input can be taken in pieces from its end, each piece's
 *                 dinit_state passed as the previous piece's dfinal_state and its
 *                 init_state the forward state at the piece's start -- exact by
 *                 the chain rule.
 * The caller owns every buffer; all pointers except cu_seqlens and beta are
 * 16-byte aligned.  Every gradient is overwritten, not accumulated; tokens
 * outside every sequence (packed input with cu_seqlens[N] < T) are not written.
 * Errors: as kda_chunk_forward, plus KDA_ERR_WORKSPACE for a missing or small
 * workspace; nothing is launched on an error.
 */
size_t kda_chunk_backward_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs);

int kda_chunk_backward(const void *q, const void *k, const void *v, const float *log_alpha,
                       const float *beta, const float *init_state, const void *d_o,
                       const float *dfinal_state, void *dq, void *dk_out, void *dv_out, float *dlog_alpha,
                       float *dbeta, float *dinit_state, const int32_t *cu_seqlens, int B, int T, int H,
                       int dk, int dv, int num_seqs, int dtype, int chunk, void *workspace, size_t ws_bytes,
                       void *stream);

/*
 * Backward schedules (kda_chunk_backward_ex):
 *   KDA_BWD_TENSOR  bf16 inputs with dk = dv = 128 (per-channel decay, or one rate
 *                   per token-head through kda_gdn_chunk_backward_ex): three
 *                   launches on the tensor cores (tcgen05) -- the forward's first
 *                   pass keeping the chunk's Akk, Aqk and T; the state sweep
 *                   storing each chunk's starting state and the adjoint sweep
 *                   storing each chunk's ending adjoint (bf16), side by side; and
 *                   per (chunk, head) the products that need them and the chain
 *                   rule through the decay factors.
 *                   Workspace: one 145 KB unit per (64-token chunk slot, head)
 *                   (0.61 GB for 8192 tokens x 32 heads).  Operands are bf16
 *                   with fp32 accumulation, like the forward's tensor-core path.
 *   KDA_BWD_SIMT    the fp32-record schedule on warp-level MMAs (any supported
 *                   dtype and size; the workspace described above).
 *   KDA_BWD_AUTO    TENSOR where it applies, else SIMT (what kda_chunk_backward does).
 */
#define KDA_BWD_AUTO 0
#define KDA_BWD_TENSOR 1
#define KDA_BWD_SIMT 2

/* Workspace bytes kda_chunk_backward_ex needs with this dtype and algo (0 when the
 * sizes are unsupported or KDA_BWD_TENSOR does not apply).  Never more than
 * kda_chunk_backward_workspace_size for the same sizes. */
size_t kda_chunk_backward_workspace_size_ex(int B, int T, int H, int dk, int dv, int num_seqs, int dtype,
                                            int algo);

/* kda_chunk_backward with an explicit schedule (KDA_BWD_*).  KDA_ERR_UNSUPPORTED
 * when KDA_BWD_TENSOR is asked for inputs it does not cover; KDA_ERR_INVALID_ARG
 * for an unknown algo; otherwise as kda_chunk_backward.  The workspace is
 * kda_chunk_backward_workspace_size_ex's for the same sizes, dtype and algo. */
int kda_chunk_backward_ex(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, const float *init_state, const void *d_o,
                          const float *dfinal_state, void *dq, void *dk_out, void *dv_out, float *dlog_alpha,
                          float *dbeta, float *dinit_state, const int32_t *cu_seqlens, int B, int T, int H,
                          int dk, int dv, int num_seqs, int dtype, int chunk, void *workspace, size_t ws_bytes,
                          void *stream, int algo);

/*
 * Backward of the Gated DeltaNet prefill (kda_gdn_chunk_forward): the same
 * gradients as kda_chunk_backward with the decay rate shared by the key
 * channels -- log_alpha and dlog_alpha are fp32 [B, T, H] (4-byte aligned), and
 * dlog_alpha is the sum over the channels of the per-channel gradient (the
 * gradient of a value broadcast over them).  Everything else, the workspace
 * (kda_chunk_backward_workspace_size) and the error behaviour are as in
 * kda_chunk_backward.
 */
int kda_gdn_chunk_backward(const void *q, const void *k, const void *v, const float *log_alpha,
                           const float *beta, const float *init_state, const void *d_o,
                           const float *dfinal_state, void *dq, void *dk_out, void *dv_out, float *dlog_alpha,
                           float *dbeta, float *dinit_state, const int32_t *cu_seqlens, int B, int T, int H,
                           int dk, int dv, int num_seqs, int dtype, int chunk, void *workspace, size_t ws_bytes,
                           void *stream);

/* kda_gdn_chunk_backward with an explicit schedule (KDA_BWD_*), as
 * kda_chunk_backward_ex (the same workspace sizes). */
int kda_gdn_chunk_backward_ex(const void *q, const void *k, const void *v, const float *log_alpha,
                              const float *beta, const float *init_state, const void *d_o,
                              const float *dfinal_state, void *dq, void *dk_out, void *dv_out, float *dlog_alpha,
                              float *dbeta, float *dinit_state, const int32_t *cu_seqlens, int B, int T, int H,
                              int dk, int dv, int num_seqs, int dtype, int chunk, void *workspace, size_t ws_bytes,
                              void *stream, int algo);

/* Message for the calling thread's last non-OK return ("" if none). */
const char *kda_last_error(void);

/*
 * Reads (and, if `clear` is non-zero, resets) the current device's status word
 * after synchronising `stream`.  *bits receives KDA_DEV_* flags.  Returns KDA_OK
 * when no flag is set, KDA_ERR_DEVICE when some flag is set, KDA_ERR_CUDA when
 * the read failed.  This call synchronises; use it off the hot path.
 */
int kda_get_device_status(unsigned int *bits, int clear, void *stream);

/*
 * Test hook for the bounded waits every tensor-core kernel uses.  Launches one
 * 32-thread CTA on `stream` that waits on a shared-memory mbarrier which no copy
 * or arrival will ever complete, giving up after `limit_cycles` SM clock cycles
 * (1 .. 2e9; 2e6 is about a millisecond); the wait runs out, the CTA flags
 * KDA_DEV_WAIT_TIMEOUT in the status word and returns, and the context stays
 * usable.  Returns KDA_OK once launched (read the flag with
 * kda_get_device_status), KDA_ERR_INVALID_ARG for a limit outside the range,
 * KDA_ERR_CUDA for a launch failure.
 */
int kda_debug_wait_timeout(long long limit_cycles, void *stream);

/* KDA_API_VERSION of the loaded library. */
int kda_api_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
