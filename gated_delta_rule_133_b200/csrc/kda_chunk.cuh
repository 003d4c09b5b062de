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
// sequences of T tokens each; otherwise nseq packed sequences given by cu.
cudaError_t chunk_fwd_simt(const void* q, const void* k, const void* v, const float* beta,
                           const float* log_alpha, const float* s0, void* o, float* sT,
                           const int32_t* cu, int nseq, int T, int H, int dk, int dv,
                           kda_dtype dtype, kda_dtype o_dtype, int mode, cudaStream_t stream);

// Chunkwise forward on the tensor cores (bf16 q/k/v only).  `tokens` is the
// length of the packed token axis (B * T, or the varlen total).
bool chunk_fwd_tc_supported(int dk, int dv, kda_dtype dtype);
cudaError_t chunk_fwd_tc(const void* q, const void* k, const void* v, const float* beta,
                         const float* log_alpha, const float* s0, void* o, float* sT, const int32_t* cu,
                         int nseq, int T, long long tokens, int H, int dk, int dv, kda_dtype o_dtype,
                         long long timeout_cycles, cudaStream_t stream);

// Two-pass tensor-core forward (bf16 q/k/v only, same arguments): a parallel
// pass over every (chunk, head) pair writes fp16 operand records to a
// stream-ordered workspace, then a sequential pass per (sequence, head, 64
// value columns) carries the state.
cudaError_t chunk_fwd_split(const void* q, const void* k, const void* v, const float* beta,
                            const float* log_alpha, const float* s0, void* o, float* sT, const int32_t* cu,
                            int nseq, int T, long long tokens, int H, int dk, int dv, kda_dtype o_dtype,
                            long long timeout_cycles, int mode, cudaStream_t stream);

// Same as chunk_fwd_split for dense inputs, with every intermediate in a
// fixed library-owned device area instead of a stream-ordered allocation;
// chunk_fwd_noalloc_fits tells whether a problem fits that area.
bool chunk_fwd_noalloc_fits(int nseq, int T, int H, int dk, int dv, bool has_final);
cudaError_t chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* beta,
                              const float* log_alpha, const float* s0, void* o, float* sT, int nseq, int T,
                              long long tokens, int H, int dk, int dv, kda_dtype o_dtype, long long timeout_cycles,
                              cudaStream_t stream);

}  // namespace kda
