// Internal launchers of the KDA CUDA library (not part of the C ABI).
#pragma once

#include "kda_common.cuh"

namespace kda {

// Decode step over NH = N * H independent (sequence, head) states.
// `mode`: KDA_MODE_* flags of kda.h (0 = the KDA layer).
cudaError_t decode_step(const void* q, const void* k, const void* v, const float* beta,
                        const float* log_alpha, float* state, void* o, long long NH, int dk,
                        int dv, kda_dtype dtype, kda_dtype o_dtype, int mode, cudaStream_t stream);

// Chunkwise forward on CUDA cores (fp32 arithmetic).  cu == nullptr: nseq
// sequences of T tokens each; otherwise nseq packed sequences given by cu
// over a token axis of length `tokens` (sequences outside it are skipped and
// flagged).
cudaError_t chunk_fwd_simt(const void* q, const void* k, const void* v, const float* beta,
                           const float* log_alpha, const float* s0, void* o, float* sT,
                           const int32_t* cu, int nseq, int T, long long tokens, int H, int dk, int dv,
                           kda_dtype dtype, kda_dtype o_dtype, int mode, cudaStream_t stream);

// Two-pass tensor-core forward (bf16 q/k/v, d_k, d_v in {64, 128}): a
// parallel pass over every (chunk, head) pair writes fp16 operand records to
// the caller's workspace, then a sequential pass per (sequence, head, 64 value
// columns) carries the state.  `tokens` is the length of the packed token
// axis (B * T, or the varlen total).  chunk_fwd_split_workspace gives the
// bytes of workspace a call with the same sizes needs.
bool chunk_fwd_split_supported(int dk, int dv, kda_dtype dtype);
size_t chunk_fwd_split_workspace(int nseq, int T, long long tokens, int H, int dk, int dv, bool varlen, int mode);
cudaError_t chunk_fwd_split(const void* q, const void* k, const void* v, const float* beta,
                            const float* log_alpha, const float* s0, void* o, float* sT, const int32_t* cu,
                            int nseq, int T, long long tokens, int H, int dk, int dv, kda_dtype o_dtype,
                            long long timeout_cycles, int mode, void* ws, size_t ws_bytes, cudaStream_t stream);

// Same as chunk_fwd_split for dense inputs, with every intermediate in a
// fixed library-owned device area instead of a caller workspace;
// chunk_fwd_noalloc_fits tells whether a problem fits that area.
bool chunk_fwd_noalloc_fits(int nseq, int T, int H, int dk, int dv, bool has_final);
cudaError_t chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* beta,
                              const float* log_alpha, const float* s0, void* o, float* sT, int nseq, int T,
                              long long tokens, int H, int dk, int dv, kda_dtype o_dtype, long long timeout_cycles,
                              cudaStream_t stream);

// Chunkwise backward on CUDA cores (fp32): gradients of sum(o * dout) +
// sum(S_T * dsT) into fp32 dq, dk, dv, dbeta, dla (the library zeroes the
// accumulated ones) and ds0 (or nullptr).  chunk_bwd_workspace gives the bytes
// of workspace a call needs.
size_t chunk_bwd_workspace(int nseq, int T, long long tokens, int H, int dk, int dv, bool varlen);
cudaError_t chunk_bwd(const void* q, const void* k, const void* v, const float* beta, const float* log_alpha,
                      const float* s0, const float* dout, const float* dsT, float* dq, float* dk, float* dv,
                      float* dbeta, float* dla, float* ds0, const int32_t* cu, int nseq, int T, long long tokens,
                      int H, int dkd, int dvd, kda_dtype dtype, void* ws, size_t ws_bytes, cudaStream_t stream);

// Chunkwise forward of the diagonal-plus-low-rank transition on CUDA cores
// (fp32): S_t = (Diag(alpha_t) + b_t a_t^T) S_{t-1} + k_t v_t^T, o_t = S_t^T q_t.
// dplr_fwd_workspace gives the bytes of workspace a call needs.
size_t dplr_fwd_workspace(int nseq, int T, long long tokens, int H, int dk, int dv, bool varlen);
cudaError_t dplr_fwd(const void* q, const void* k, const void* v, const void* a, const void* b, const float* log_alpha,
                     const float* s0, void* o, float* sT, const int32_t* cu, int nseq, int T, long long tokens, int H,
                     int dk, int dv, kda_dtype dtype, kda_dtype o_dtype, void* ws, size_t ws_bytes, cudaStream_t s);

}  // namespace kda
