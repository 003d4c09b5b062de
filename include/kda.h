/*
 * kda.h -- C ABI of the KDA / gated-DeltaNet layer for NVIDIA B200 (sm_100a).
 *
 * The layer keeps, per (sequence, head), a d_k x d_v fp32 state S and for each
 * token t applies
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *     o_t = S_t^T q_t,                 alpha_t = exp(log_alpha_t)  (per channel)
 *
 * ("Hybrid Linear Attention Architecture: Making LLM Training and Inference
 * More Efficient", section 3.3: decay per channel first, then the delta
 * rule's erase and write; the output is read after the write as in the
 * inference loop of "Demystifying Hybrid LLM Architectures", section 2.3.)
 * No query scaling is applied.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor pointer is a DEVICE pointer owned by the caller.  The
 *    library allocates no device memory and keeps no pointer after the call
 *    returns.  The tensor-core chunk forward needs scratch memory (per-chunk
 *    operand records and a few index arrays): the caller passes it as
 *    `workspace` / `workspace_bytes`, sized by kda_chunk_fwd_workspace_size() or
 *    kda_varlen_fwd_workspace_size() for the same arguments.  The workspace is
 *    used asynchronously on `stream` (it must stay allocated until the work
 *    queued there has run) and its contents need no initialisation.  The one
 *    exception is kda_chunk_fwd_noalloc(), which keeps its scratch in a fixed
 *    library-owned area (see there).
 *  - Layouts are dense, row-major, token-major ("[B, T, H, d]": d fastest).
 *  - q, k and v have the element type `dtype` (KDA_BF16 or KDA_F32); the
 *    output o has the element type `o_dtype` (either, independently; KDA_F32
 *    keeps the fp32 accumulation, KDA_BF16 rounds it to nearest even);
 *    beta, log_alpha and all states are always fp32.  log_alpha must be <= 0
 *    (alpha in (0, 1]); it is not checked on the device.
 *  - Every tensor pointer must be 16-byte aligned, except beta and
 *    cu_seqlens (4-byte aligned).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *    asynchronous on that stream and never synchronise.
 *  - Argument errors are reported synchronously (nothing is launched).  A
 *    launch failure returns KDA_ERR_CUDA.  Device-side failures (a bounded
 *    wait that ran out) are recorded in a per-device status word and reported
 *    by kda_check().
 *  - Supported: d_k, d_v in {64, 128}, chunk == 64.  Other sizes return
 *    KDA_ERR_UNSUPPORTED.  No C++ exception crosses this interface.
 *  - Numerical domain: the tensor-core chunk forward, the backward and the
 *    DPLR forward factor the per-channel decay inside one 64-token chunk
 *    around the chunk's middle token; that requires the decay of any 32
 *    consecutive tokens of one channel to stay below about 80 nats (average
 *    alpha above ~0.08).  Stronger gates lose accuracy in the intra-chunk
 *    terms (results stay finite); those kernels detect it per (chunk,
 *    channel) and kda_check() then reports KDA_WARN_DOMAIN.  The CUDA-core
 *    chunk forward (fp32 inputs, or KDA_MODE_CUDA_CORES) splits the decay
 *    by 16-token blocks with every factor at most 1 and has no such limit;
 *    neither has the decode step.  The tensor-core path rounds
 *    its operands to fp16: entries of e^G q, e^G k, the state, beta (v - k S)
 *    and of the intra-chunk inverse (I + A)^-1 must stay below 65504 in
 *    magnitude.  With keys of norm at most 1 and beta <= 1 the inverse's
 *    entries are at most 1 in magnitude.
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, bad size          */
    KDA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (d, chunk, dtype)  */
    KDA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed         */
    KDA_ERR_TIMEOUT = 4,      /* a device-side bounded wait ran out           */
    KDA_WARN_DOMAIN = 5       /* a chunk's gate decay left the factorisation
                                 range: results are finite but inexact      */
} kda_status;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;

/*
 * Chunkwise-parallel forward over B equal-length sequences (training and
 * prefill).  The chunk recurrence is the one given in "Hybrid Linear Attention
 * Architecture: Making LLM Training and Inference More Efficient", section IV,
 * "... Technical Deep Dive ...", section 4 and "Linear Attention Architecture
 * Deep Dive", section 5 (state carried between chunks, WY residual
 * correction U - W S, lower-triangular intra-chunk term).
 *
 *   q, k        [B, T, H, dk]  dtype
 *   v           [B, T, H, dv]  dtype
 *   beta        [B, T, H]      fp32, write strength in (0, 1)
 *   log_alpha   [B, T, H, dk]  fp32, per-channel log forget gate (<= 0)
 *   initial_state [B, H, dk, dv] fp32, or NULL for zeros (read only)
 *   o           [B, T, H, dv]  o_dtype, written
 *   final_state [B, H, dk, dv] fp32, or NULL if not wanted; written.  It may
 *               alias initial_state (in-place state update).
 *   workspace   device scratch of at least kda_chunk_fwd_workspace_size()
 *               bytes for these sizes (256-byte aligned), or NULL when that
 *               size is 0; a smaller workspace_bytes returns
 *               KDA_ERR_INVALID_ARG before anything is launched.
 *   B >= 0, T >= 0 (B*T == 0 is a no-op that still writes final_state from
 *   initial_state), H >= 1, chunk must be 64.
 */
kda_status kda_chunk_fwd(const void* q, const void* k, const void* v,
                         const float* beta, const float* log_alpha,
                         const float* initial_state, void* o, float* final_state,
                         int B, int T, int H, int dk, int dv, int chunk,
                         kda_dtype dtype, kda_dtype o_dtype,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * Bytes of workspace kda_chunk_fwd / kda_chunk_fwd_mode need for these
 * arguments (`mode` as in kda_chunk_fwd_mode; 0 for the plain call), written
 * to *bytes.  Pure host computation (it reads the current device's SM count);
 * 0 when the call runs on the CUDA-core kernel.  Argument errors as in the
 * forward call.
 */
kda_status kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int chunk,
                                        kda_dtype dtype, int mode, size_t* bytes);

/*
 * kda_chunk_fwd computed without allocating any memory.  The method the pages
 * describe has no counterpart of this call: it differs from kda_chunk_fwd
 * only in where the tensor-core path keeps its intermediates (the per-chunk
 * operand records and, when final_state is NULL, the state carried between
 * blocks of chunks), namely a fixed 64 MiB area the library owns on each
 * device, instead of a caller-provided workspace.  Arguments, layouts and
 * results are those of kda_chunk_fwd (results bit-identical to it).
 *
 *   - Problems whose records for one 64-token chunk of every (sequence, head),
 *     twice over, plus the carried state do not fit the area return
 *     KDA_ERR_UNSUPPORTED before anything is launched (bf16 inputs, d_k = 128:
 *     B * H up to 577 with final_state, fewer without).
 *   - The area is shared by all calls on a device: calls of this function
 *     must be ordered with respect to each other (one stream, or synchronised
 *     by the caller).  Inputs the tensor-core path does not take (fp32) run on
 *     the CUDA-core kernel, which needs no scratch.
 */
kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                 const float* beta, const float* log_alpha,
                                 const float* initial_state, void* o, float* final_state,
                                 int B, int T, int H, int dk, int dv, int chunk,
                                 kda_dtype dtype, kda_dtype o_dtype, void* stream);

/*
 * Same computation over N variable-length sequences packed along one token
 * axis (B = 1).  The state restarts (from initial_state[n] or zero) at every
 * sequence boundary; the last chunk of each sequence may be shorter than 64.
 *
 *   q, k [T, H, dk], v [T, H, dv] (dtype), beta [T, H], log_alpha [T, H, dk],
 *   o [T, H, dv] (o_dtype)
 *   cu_seqlens  [N + 1] int32, DEVICE pointer, cu_seqlens[0] = 0,
 *               non-decreasing, cu_seqlens[N] = T.  The boundaries are read on
 *               the device and guarded there: a sequence whose token range
 *               leaves [0, T) is skipped (its o rows are not written, its
 *               final state is its initial state) and the next kda_check()
 *               reports KDA_ERR_INVALID_ARG; a decreasing pair counts as an
 *               empty sequence; o rows outside every sequence are not written.
 *   initial_state / final_state [N, H, dk, dv] fp32 or NULL.
 *   workspace   as for kda_chunk_fwd, sized by kda_varlen_fwd_workspace_size().
 *   N <= 65535.  The tensor-core path scans the longest sequences first (an
 *   order computed on the device once per call).
 */
kda_status kda_varlen_fwd(const void* q, const void* k, const void* v,
                          const float* beta, const float* log_alpha,
                          const int32_t* cu_seqlens, int N,
                          const float* initial_state, void* o, float* final_state,
                          int T, int H, int dk, int dv, int chunk,
                          kda_dtype dtype, kda_dtype o_dtype,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes of kda_varlen_fwd / kda_varlen_fwd_mode (see
 * kda_chunk_fwd_workspace_size); T is the packed token count. */
kda_status kda_varlen_fwd_workspace_size(int N, int T, int H, int dk, int dv, int chunk,
                                         kda_dtype dtype, int mode, size_t* bytes);

/*
 * One decode step of the recurrence for N independent sequences (one new
 * token each), updating the state in place: the recurrent form of "Hybrid
 * Linear Attention Architecture: Making LLM Training and Inference More
 * Efficient", section 3.3, one state update and one state read per token
 * (its section I).  Memory bound: every state is read once and written once.
 * Needs no workspace.
 *
 *   q, k [N, H, dk], v [N, H, dv]  dtype
 *   beta [N, H], log_alpha [N, H, dk]  fp32
 *   state [N, H, dk, dv] fp32, read and overwritten in place
 *   o [N, H, dv] o_dtype, written
 */
kda_status kda_recurrent_step(const void* q, const void* k, const void* v,
                              const float* beta, const float* log_alpha,
                              float* state, void* o,
                              int N, int H, int dk, int dv,
                              kda_dtype dtype, kda_dtype o_dtype, void* stream);

/*
 * Variants of the layer, selected by the bit flags `mode` of the *_mode entry
 * points below (mode = 0 is the layer above; unknown bits return
 * KDA_ERR_INVALID_ARG).  Both are gate tiers of "Hybrid Linear Attention
 * Architecture: Making LLM Training and Inference More Efficient", section 3.3:
 *
 *  KDA_MODE_HEAD_GATE  one forget gate per (token, head), the scalar gate:
 *      log_alpha has no d_k axis ([B, T, H], [T, H] or [N, H]; 4-byte
 *      aligned) and alpha_t scales every key channel of the state alike.  With
 *      a scalar gate the decay commutes with the erase, so the section's two
 *      orderings coincide.
 *  KDA_MODE_NO_ERASE   no erase term: S_t = Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *      the element-wise gate without the delta rule (beta_t = 1 gives the
 *      section's form; per-channel decay of the key rows as in this layer).
 *
 * Two more flags move the inputs' pre-processing into the kernels (the pages
 * give unit-norm q, k and a gate from a sigmoid of a projection: section 3.4
 * of the same page):
 *
 *  KDA_MODE_NORM_QK      q and k are raw: every (token, head) row of q and of k
 *      is divided by its L2 norm (rows of norm below 1e-15 count as zero).
 *  KDA_MODE_GATE_LOGITS  log_alpha holds gate logits z: the layer uses
 *      log alpha = -softplus(z), i.e. alpha = sigmoid(-z).
 *
 * Execution options of the chunk forwards (they change how, not what, is
 * computed; used to cross-check the kernels against each other):
 *
 *  KDA_MODE_CUDA_CORES   run the fp32 CUDA-core kernel whatever the input
 *      dtype (the reference-precision path; it needs no workspace).
 *  KDA_MODE_BLOCKS(n)    tensor-core path, dense inputs: cut the chunk axis
 *      into n blocks (1 <= n <= 8) and overlap the parallel pass of block b + 1
 *      with the sequential pass of block b on a second stream; n = 1 runs the
 *      parallel pass over every chunk, then the sequential pass.  Results are
 *      bit-identical to the default schedule for every n.
 *
 * The flags combine.  Every other argument, layout and rule is that of the
 * plain entry point of the same name.
 */
#define KDA_MODE_HEAD_GATE 1
#define KDA_MODE_NO_ERASE 2
#define KDA_MODE_NORM_QK 4
#define KDA_MODE_GATE_LOGITS 8
#define KDA_MODE_CUDA_CORES 16
#define KDA_MODE_BLOCKS(n) ((n) << 8)

kda_status kda_chunk_fwd_mode(const void* q, const void* k, const void* v,
                              const float* beta, const float* log_alpha,
                              const float* initial_state, void* o, float* final_state,
                              int B, int T, int H, int dk, int dv, int chunk,
                              kda_dtype dtype, kda_dtype o_dtype, int mode,
                              void* workspace, size_t workspace_bytes, void* stream);

kda_status kda_varlen_fwd_mode(const void* q, const void* k, const void* v,
                               const float* beta, const float* log_alpha,
                               const int32_t* cu_seqlens, int N,
                               const float* initial_state, void* o, float* final_state,
                               int T, int H, int dk, int dv, int chunk,
                               kda_dtype dtype, kda_dtype o_dtype, int mode,
                               void* workspace, size_t workspace_bytes, void* stream);

kda_status kda_recurrent_step_mode(const void* q, const void* k, const void* v,
                                   const float* beta, const float* log_alpha,
                                   float* state, void* o,
                                   int N, int H, int dk, int dv,
                                   kda_dtype dtype, kda_dtype o_dtype, int mode, void* stream);

/*
 * Chunkwise backward pass: gradients of L = sum(o * grad_o) + sum(S_T * grad_final_state)
 * through kda_chunk_fwd's computation ("Hybrid Linear Attention Architecture:
 * Making LLM Training and Inference More Efficient", section IV: backpropagation
 * reuses the chunked structure of the forward pass).  Per (chunk, head) it
 * forms the chunk's factors once; a forward walk stores the state entering
 * every chunk, a reverse walk carries the state's gradient; the products that
 * sum over value columns and the adjoint of the UT transform and of the gate
 * factors then run per (chunk, head).  Everything between the launches lives
 * in the workspace (one record of factors, the states, U, dU, dY, V - X and
 * the state gradients per chunk).  fp32 arithmetic on CUDA cores throughout;
 * the plain layer only (no KDA_MODE_* variants).
 *
 *   q, k, v, beta, log_alpha, initial_state: as in kda_chunk_fwd (dtype bf16 or fp32)
 *   grad_o           [B, T, H, dv] fp32
 *   grad_final_state [B, H, dk, dv] fp32, or NULL (zero)
 *   grad_q, grad_k   [B, T, H, dk] fp32, written
 *   grad_v           [B, T, H, dv] fp32, written
 *   grad_beta        [B, T, H]     fp32, written
 *   grad_log_alpha   [B, T, H, dk] fp32, written
 *   grad_initial_state [B, H, dk, dv] fp32, or NULL if not wanted
 *   workspace        at least kda_chunk_bwd_workspace_size() bytes, 256-byte aligned,
 *                    owned by the caller, not read across calls.  Undersized,
 *                    missing or unaligned: KDA_ERR_INVALID_ARG before any launch.
 * Packed batches: a sequence whose token range leaves [0, T) is skipped (zero
 * gradients for its rows except grad_v, which is not written; its initial
 * state gradient is grad_final_state) and reported by the next kda_check().
 * All tensor pointers 16-byte aligned (beta, grad_beta: 4).  d_k, d_v in
 * {64, 128}, chunk 64.  The gradient buffers must not alias the inputs.
 */
kda_status kda_chunk_bwd(const void* q, const void* k, const void* v, const float* beta,
                         const float* log_alpha, const float* initial_state,
                         const float* grad_o, const float* grad_final_state,
                         float* grad_q, float* grad_k, float* grad_v, float* grad_beta,
                         float* grad_log_alpha, float* grad_initial_state,
                         int B, int T, int H, int dk, int dv, int chunk, kda_dtype dtype,
                         void* workspace, size_t workspace_bytes, void* stream);

kda_status kda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int chunk,
                                        kda_dtype dtype, size_t* bytes);

/* The same over N packed variable-length sequences (layouts of
 * kda_varlen_fwd; initial/final state gradients [N, H, dk, dv]). */
kda_status kda_varlen_bwd(const void* q, const void* k, const void* v, const float* beta,
                          const float* log_alpha, const int32_t* cu_seqlens, int N,
                          const float* initial_state, const float* grad_o, const float* grad_final_state,
                          float* grad_q, float* grad_k, float* grad_v, float* grad_beta,
                          float* grad_log_alpha, float* grad_initial_state,
                          int T, int H, int dk, int dv, int chunk, kda_dtype dtype,
                          void* workspace, size_t workspace_bytes, void* stream);

kda_status kda_varlen_bwd_workspace_size(int N, int T, int H, int dk, int dv, int chunk,
                                         kda_dtype dtype, size_t* bytes);

/*
 * Chunkwise forward of the diagonal-plus-low-rank transition, the "finer
 * granularity" gate of "Hybrid Linear Attention Architecture: Making LLM
 * Training and Inference More Efficient", section 3.3 (a low-rank correction
 * on top of the element-wise decay; also the RWKV-7 line of "... Technical Deep
 * Dive ...", section 3), in this library's d_k x d_v orientation:
 *
 *     S_t = (Diag(alpha_t) + b_t a_t^T) S_{t-1} + k_t v_t^T,     o_t = S_t^T q_t
 *
 * (the pages write S_{t-1} (Diag(alpha_t) + a_t b_t^T) + v_t k_t^T for the
 * transposed d_v x d_k state).  With a_t = alpha_t * k_t, b_t = -beta_t k_t and
 * the key beta_t k_t it is the KDA layer.  fp32 arithmetic on CUDA cores.
 *
 *   q, k, a, b  [B, T, H, dk]  dtype;   v [B, T, H, dv]  dtype
 *   log_alpha   [B, T, H, dk]  fp32 (<= 0)
 *   initial_state / final_state [B, H, dk, dv] fp32 or NULL (final may alias initial)
 *   o           [B, T, H, dv]  o_dtype
 *   workspace   device scratch of at least kda_dplr_fwd_workspace_size() bytes,
 *               256-byte aligned, owned by the caller, not read across calls
 *               (one record of chunk factors per (chunk, head)); NULL when
 *               that size is 0.  Undersized or unaligned: KDA_ERR_INVALID_ARG.
 * d_k, d_v in {64, 128}, chunk 64; pointers 16-byte aligned.
 */
kda_status kda_dplr_fwd(const void* q, const void* k, const void* v, const void* a, const void* b,
                        const float* log_alpha, const float* initial_state, void* o, float* final_state,
                        int B, int T, int H, int dk, int dv, int chunk,
                        kda_dtype dtype, kda_dtype o_dtype, void* workspace, size_t workspace_bytes,
                        void* stream);

/* Bytes of workspace kda_dplr_fwd needs for these sizes (0 for empty input). */
kda_status kda_dplr_fwd_workspace_size(int B, int T, int H, int dk, int dv, int chunk, kda_dtype dtype,
                                       size_t* bytes);

/* The same over N packed variable-length sequences (layouts and boundary
 * rules of kda_varlen_fwd). */
kda_status kda_dplr_varlen_fwd(const void* q, const void* k, const void* v, const void* a, const void* b,
                               const float* log_alpha, const int32_t* cu_seqlens, int N,
                               const float* initial_state, void* o, float* final_state,
                               int T, int H, int dk, int dv, int chunk,
                               kda_dtype dtype, kda_dtype o_dtype, void* workspace, size_t workspace_bytes,
                               void* stream);

kda_status kda_dplr_varlen_fwd_workspace_size(int N, int T, int H, int dk, int dv, int chunk, kda_dtype dtype,
                                              size_t* bytes);

/*
 * Synchronises `stream` and reports (then clears) the current device's
 * status word: KDA_ERR_TIMEOUT if a device-side bounded wait ran out since the
 * last check, KDA_ERR_INVALID_ARG if a kernel found device-resident sequence
 * boundaries (cu_seqlens) outside the token range and skipped that sequence,
 * KDA_WARN_DOMAIN if a chunk kernel met a gate outside the numerical domain
 * (see "Numerical domain" above), KDA_ERR_CUDA if the stream reports an error,
 * else KDA_OK (in that order of precedence).
 */
kda_status kda_check(void* stream);

/*
 * Diagnostic: launches one CTA that waits on a shared-memory barrier no thread
 * ever arrives on, through the same bounded wait the chunk kernel uses, with a
 * budget of `limit_cycles` SM clock cycles (1 .. 2^32).  The wait gives up,
 * records KDA_ERR_TIMEOUT in the device status word and the kernel exits
 * normally: the next kda_check() must report KDA_ERR_TIMEOUT and the
 * one after it KDA_OK.  Exercises the failure path without any GPU fault.
 * Returns KDA_ERR_INVALID_ARG for a budget out of range.
 */
kda_status kda_selftest_timeout(long long limit_cycles, void* stream);

/* Static, human-readable name of a status code (never NULL). */
const char* kda_status_string(kda_status status);

/* Interface version: major * 10000 + minor * 100 + patch. */
int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
