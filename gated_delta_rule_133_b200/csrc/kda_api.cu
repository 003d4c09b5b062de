// C ABI of the KDA library: argument validation, path selection, status codes.
// Declarations and the contract of every entry point are in include/kda.h.
#include <string.h>
#include <cuda_runtime.h>

#include "kda_chunk.cuh"
#include "kda_sm100.cuh"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool supported_d(int d) { return d == 64 || d == 128; }

bool valid_dtype(kda_dtype t) { return t == KDA_F32 || t == KDA_BF16; }

kda_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

// Budget of every device-side bounded wait of the tensor-core kernels, in SM
// clock cycles (about one second).
constexpr long long kTimeoutCycles = 1LL << 31;

constexpr int kLayerBits = KDA_MODE_HEAD_GATE | KDA_MODE_NO_ERASE | KDA_MODE_NORM_QK | KDA_MODE_GATE_LOGITS;

int mode_blocks(int mode) { return (mode >> 8) & 0xff; }

bool valid_mode(int mode, bool chunk_call)
{
    if (!chunk_call) return (mode & ~kLayerBits) == 0;
    const int nb = mode_blocks(mode);
    return (mode & ~(kLayerBits | KDA_MODE_CUDA_CORES | KDA_MODE_BLOCKS(0xff))) == 0 && nb <= 8;
}

// bf16 inputs with supported head sizes run on the tensor cores unless the
// caller asks for the CUDA-core kernel; fp32 inputs always run on the CUDA
// cores (their fp32 arithmetic is what meets the fp32 bar).
bool use_tensor_cores(int dk, int dv, kda_dtype dtype, int mode)
{
    return kda::chunk_fwd_split_supported(dk, dv, dtype) && !(mode & KDA_MODE_CUDA_CORES);
}

// Shared checks of the forward entry points.
kda_status check_fwd(const void* q, const void* k, const void* v, const float* beta,
                     const float* log_alpha, const float* s0, const void* o, const float* sT,
                     long long tokens, int H, int dk, int dv, int chunk, kda_dtype dtype,
                     kda_dtype o_dtype, int mode)
{
    if (H <= 0 || dk <= 0 || dv <= 0 || tokens < 0) return KDA_ERR_INVALID_ARG;
    if (!valid_dtype(dtype) || !valid_dtype(o_dtype) || !valid_mode(mode, true)) return KDA_ERR_INVALID_ARG;
    const bool gate_ok = (mode & KDA_MODE_HEAD_GATE) ? aligned4(log_alpha) : aligned16(log_alpha);
    if (tokens > 0) {
        if (!q || !k || !v || !beta || !log_alpha || !o) return KDA_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(beta) || !gate_ok || !aligned16(o))
            return KDA_ERR_INVALID_ARG;
    }
    if ((s0 && !aligned16(s0)) || (sT && !aligned16(sT))) return KDA_ERR_INVALID_ARG;
    if (chunk != 64 || !supported_d(dk) || !supported_d(dv)) return KDA_ERR_UNSUPPORTED;
    return KDA_OK;
}

// Size checks shared by the workspace queries and the forward calls.
kda_status check_sizes(int H, int dk, int dv, int chunk, kda_dtype dtype, int mode)
{
    if (H <= 0 || dk <= 0 || dv <= 0 || !valid_dtype(dtype) || !valid_mode(mode, true)) return KDA_ERR_INVALID_ARG;
    if (chunk != 64 || !supported_d(dk) || !supported_d(dv)) return KDA_ERR_UNSUPPORTED;
    return KDA_OK;
}

size_t workspace_bytes(int nseq, int T, long long tokens, int H, int dk, int dv, kda_dtype dtype, int mode,
                       bool varlen)
{
    if (!use_tensor_cores(dk, dv, dtype, mode) || tokens <= 0) return 0;
    return kda::chunk_fwd_split_workspace(nseq, T, tokens, H, dk, dv, varlen, mode);
}

kda_status check_workspace(const void* ws, size_t have, size_t need)
{
    if (need == 0) return KDA_OK;
    if (!ws || have < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return KDA_ERR_INVALID_ARG;
    return KDA_OK;
}

kda_status run_chunk(const void* q, const void* k, const void* v, const float* beta,
                     const float* log_alpha, const float* s0, void* o, float* sT, const int32_t* cu,
                     int nseq, int T, long long tokens, int H, int dk, int dv, kda_dtype dtype,
                     kda_dtype o_dtype, int mode, void* ws, size_t ws_bytes, cudaStream_t s)
{
    if (use_tensor_cores(dk, dv, dtype, mode))
        return from_cuda(kda::chunk_fwd_split(q, k, v, beta, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dk, dv,
                                              o_dtype, kTimeoutCycles, mode, ws, ws_bytes, s));
    return from_cuda(kda::chunk_fwd_simt(q, k, v, beta, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dk, dv, dtype,
                                         o_dtype, mode & kLayerBits, s));
}

// Writes final = initial (or zeros) for sequences that have no tokens at all.
kda_status copy_state(const float* s0, float* sT, size_t elems, cudaStream_t s)
{
    if (!sT || elems == 0) return KDA_OK;
    if (s0 == sT) return KDA_OK;
    if (s0) return from_cuda(cudaMemcpyAsync(sT, s0, elems * sizeof(float), cudaMemcpyDeviceToDevice, s));
    return from_cuda(cudaMemsetAsync(sT, 0, elems * sizeof(float), s));
}

// One CTA waits, with the chunk kernel's bounded wait, on an mbarrier that
// nobody arrives on; the wait records the timeout and the kernel returns.
__global__ void selftest_timeout_kernel(long long limit_cycles)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        kda::sm100::mbar_init(&bar, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    (void)kda::sm100::mbar_wait(&bar, 0u, &abort_flag, limit_cycles);
}

}  // namespace

extern "C" {

kda_status kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int chunk, kda_dtype dtype, int mode,
                                        size_t* bytes)
{
    if (!bytes || B < 0 || T < 0) return KDA_ERR_INVALID_ARG;
    const kda_status st = check_sizes(H, dk, dv, chunk, dtype, mode);
    if (st != KDA_OK) return st;
    const long long tokens = (long long)B * T;
    if (tokens > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    *bytes = workspace_bytes(B, T, tokens, H, dk, dv, dtype, mode, false);
    return KDA_OK;
}

kda_status kda_varlen_fwd_workspace_size(int N, int T, int H, int dk, int dv, int chunk, kda_dtype dtype, int mode,
                                         size_t* bytes)
{
    if (!bytes || N < 0 || N > 65535 || T < 0 || (mode_blocks(mode) != 0)) return KDA_ERR_INVALID_ARG;
    const kda_status st = check_sizes(H, dk, dv, chunk, dtype, mode);
    if (st != KDA_OK) return st;
    *bytes = N == 0 ? 0 : workspace_bytes(N, 0, T, H, dk, dv, dtype, mode, true);
    return KDA_OK;
}

kda_status kda_chunk_fwd_mode(const void* q, const void* k, const void* v, const float* beta,
                              const float* log_alpha, const float* initial_state, void* o,
                              float* final_state, int B, int T, int H, int dk, int dv, int chunk,
                              kda_dtype dtype, kda_dtype o_dtype, int mode, void* workspace,
                              size_t workspace_bytes_, void* stream)
{
    if (B < 0 || T < 0) return KDA_ERR_INVALID_ARG;
    const long long tokens = (long long)B * T;
    kda_status st = check_fwd(q, k, v, beta, log_alpha, initial_state, o, final_state, tokens, H,
                              dk, dv, chunk, dtype, o_dtype, mode);
    if (st != KDA_OK) return st;
    if (tokens > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    st = check_workspace(workspace, workspace_bytes_, workspace_bytes(B, T, tokens, H, dk, dv, dtype, mode, false));
    if (st != KDA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (tokens == 0) return copy_state(initial_state, final_state, (size_t)B * H * dk * dv, s);
    return run_chunk(q, k, v, beta, log_alpha, initial_state, o, final_state, nullptr, B, T, tokens, H, dk,
                     dv, dtype, o_dtype, mode, workspace, workspace_bytes_, s);
}

kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const float* beta,
                         const float* log_alpha, const float* initial_state, void* o,
                         float* final_state, int B, int T, int H, int dk, int dv, int chunk,
                         kda_dtype dtype, kda_dtype o_dtype, void* workspace, size_t workspace_bytes_,
                         void* stream)
{
    return kda_chunk_fwd_mode(q, k, v, beta, log_alpha, initial_state, o, final_state, B, T, H, dk, dv, chunk,
                              dtype, o_dtype, 0, workspace, workspace_bytes_, stream);
}

kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* beta,
                                 const float* log_alpha, const float* initial_state, void* o,
                                 float* final_state, int B, int T, int H, int dk, int dv, int chunk,
                                 kda_dtype dtype, kda_dtype o_dtype, void* stream)
{
    if (B < 0 || T < 0) return KDA_ERR_INVALID_ARG;
    const long long tokens = (long long)B * T;
    kda_status st = check_fwd(q, k, v, beta, log_alpha, initial_state, o, final_state, tokens, H,
                              dk, dv, chunk, dtype, o_dtype, 0);
    if (st != KDA_OK) return st;
    if (tokens > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (tokens == 0) return copy_state(initial_state, final_state, (size_t)B * H * dk * dv, s);
    if (!kda::chunk_fwd_split_supported(dk, dv, dtype))   // the CUDA-core kernel needs no scratch
        return from_cuda(kda::chunk_fwd_simt(q, k, v, beta, log_alpha, initial_state, o, final_state, nullptr, B,
                                             T, tokens, H, dk, dv, dtype, o_dtype, 0, s));
    if (!kda::chunk_fwd_noalloc_fits(B, T, H, dk, dv, final_state != nullptr)) return KDA_ERR_UNSUPPORTED;
    return from_cuda(kda::chunk_fwd_noalloc(q, k, v, beta, log_alpha, initial_state, o, final_state, B, T, tokens,
                                            H, dk, dv, o_dtype, kTimeoutCycles, s));
}

kda_status kda_varlen_fwd_mode(const void* q, const void* k, const void* v, const float* beta,
                               const float* log_alpha, const int32_t* cu_seqlens, int N,
                               const float* initial_state, void* o, float* final_state, int T, int H,
                               int dk, int dv, int chunk, kda_dtype dtype, kda_dtype o_dtype, int mode,
                               void* workspace, size_t workspace_bytes_, void* stream)
{
    if (N < 0 || N > 65535 || T < 0 || mode_blocks(mode) != 0) return KDA_ERR_INVALID_ARG;
    kda_status st = check_fwd(q, k, v, beta, log_alpha, initial_state, o, final_state, T, H, dk,
                              dv, chunk, dtype, o_dtype, mode);
    if (st != KDA_OK) return st;
    if (N == 0) return T == 0 ? KDA_OK : KDA_ERR_INVALID_ARG;
    if (!cu_seqlens || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return KDA_ERR_INVALID_ARG;
    st = check_workspace(workspace, workspace_bytes_, workspace_bytes(N, 0, T, H, dk, dv, dtype, mode, true));
    if (st != KDA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) return copy_state(initial_state, final_state, (size_t)N * H * dk * dv, s);
    return run_chunk(q, k, v, beta, log_alpha, initial_state, o, final_state, cu_seqlens, N, T, T, H, dk,
                     dv, dtype, o_dtype, mode, workspace, workspace_bytes_, s);
}

kda_status kda_varlen_fwd(const void* q, const void* k, const void* v, const float* beta,
                          const float* log_alpha, const int32_t* cu_seqlens, int N,
                          const float* initial_state, void* o, float* final_state, int T, int H,
                          int dk, int dv, int chunk, kda_dtype dtype, kda_dtype o_dtype,
                          void* workspace, size_t workspace_bytes_, void* stream)
{
    return kda_varlen_fwd_mode(q, k, v, beta, log_alpha, cu_seqlens, N, initial_state, o, final_state, T, H,
                               dk, dv, chunk, dtype, o_dtype, 0, workspace, workspace_bytes_, stream);
}

kda_status kda_recurrent_step_mode(const void* q, const void* k, const void* v, const float* beta,
                                   const float* log_alpha, float* state, void* o, int N, int H, int dk,
                                   int dv, kda_dtype dtype, kda_dtype o_dtype, int mode, void* stream)
{
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (!valid_dtype(dtype) || !valid_dtype(o_dtype) || !valid_mode(mode, false)) return KDA_ERR_INVALID_ARG;
    if (N == 0) return KDA_OK;
    if (!q || !k || !v || !beta || !log_alpha || !state || !o) return KDA_ERR_INVALID_ARG;
    const bool gate_ok = (mode & KDA_MODE_HEAD_GATE) ? aligned4(log_alpha) : aligned16(log_alpha);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(beta) || !gate_ok ||
        !aligned16(state) || !aligned16(o))
        return KDA_ERR_INVALID_ARG;
    if (!supported_d(dk) || !supported_d(dv)) return KDA_ERR_UNSUPPORTED;
    return from_cuda(kda::decode_step(q, k, v, beta, log_alpha, state, o, (long long)N * H, dk,
                                      dv, dtype, o_dtype, mode, static_cast<cudaStream_t>(stream)));
}

kda_status kda_recurrent_step(const void* q, const void* k, const void* v, const float* beta,
                              const float* log_alpha, float* state, void* o, int N, int H, int dk,
                              int dv, kda_dtype dtype, kda_dtype o_dtype, void* stream)
{
    return kda_recurrent_step_mode(q, k, v, beta, log_alpha, state, o, N, H, dk, dv, dtype, o_dtype, 0, stream);
}

kda_status kda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int chunk, kda_dtype dtype,
                                        size_t* bytes)
{
    if (!bytes || B < 0 || T < 0) return KDA_ERR_INVALID_ARG;
    const kda_status st = check_sizes(H, dk, dv, chunk, dtype, 0);
    if (st != KDA_OK) return st;
    const long long tokens = (long long)B * T;
    if (tokens > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    *bytes = tokens == 0 ? 0 : kda::chunk_bwd_workspace(B, T, tokens, H, dk, dv, false);
    return KDA_OK;
}

kda_status kda_varlen_bwd_workspace_size(int N, int T, int H, int dk, int dv, int chunk, kda_dtype dtype,
                                         size_t* bytes)
{
    if (!bytes || N < 0 || N > 65535 || T < 0) return KDA_ERR_INVALID_ARG;
    const kda_status st = check_sizes(H, dk, dv, chunk, dtype, 0);
    if (st != KDA_OK) return st;
    *bytes = (N == 0 || T == 0) ? 0 : kda::chunk_bwd_workspace(N, 0, T, H, dk, dv, true);
    return KDA_OK;
}

namespace {

kda_status check_bwd(const void* q, const void* k, const void* v, const float* beta, const float* log_alpha,
                     const float* s0, const float* go, const float* gsT, const float* gq, const float* gk,
                     const float* gv, const float* gb, const float* gla, const float* gs0, long long tokens, int H,
                     int dk, int dv, int chunk, kda_dtype dtype)
{
    if (H <= 0 || dk <= 0 || dv <= 0 || tokens < 0 || !valid_dtype(dtype)) return KDA_ERR_INVALID_ARG;
    if (tokens > 0) {
        if (!q || !k || !v || !beta || !log_alpha || !go || !gq || !gk || !gv || !gb || !gla)
            return KDA_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(beta) || !aligned16(log_alpha) ||
            !aligned16(go) || !aligned16(gq) || !aligned16(gk) || !aligned16(gv) || !aligned4(gb) || !aligned16(gla))
            return KDA_ERR_INVALID_ARG;
    }
    if ((s0 && !aligned16(s0)) || (gsT && !aligned16(gsT)) || (gs0 && !aligned16(gs0))) return KDA_ERR_INVALID_ARG;
    if (chunk != 64 || !supported_d(dk) || !supported_d(dv)) return KDA_ERR_UNSUPPORTED;
    return KDA_OK;
}

}  // namespace

kda_status kda_chunk_bwd(const void* q, const void* k, const void* v, const float* beta, const float* log_alpha,
                         const float* initial_state, const float* grad_o, const float* grad_final_state,
                         float* grad_q, float* grad_k, float* grad_v, float* grad_beta, float* grad_log_alpha,
                         float* grad_initial_state, int B, int T, int H, int dk, int dv, int chunk, kda_dtype dtype,
                         void* workspace, size_t workspace_bytes_, void* stream)
{
    if (B < 0 || T < 0) return KDA_ERR_INVALID_ARG;
    const long long tokens = (long long)B * T;
    kda_status st = check_bwd(q, k, v, beta, log_alpha, initial_state, grad_o, grad_final_state, grad_q, grad_k,
                              grad_v, grad_beta, grad_log_alpha, grad_initial_state, tokens, H, dk, dv, chunk, dtype);
    if (st != KDA_OK) return st;
    if (tokens > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    const size_t need = tokens == 0 ? 0 : kda::chunk_bwd_workspace(B, T, tokens, H, dk, dv, false);
    st = check_workspace(workspace, workspace_bytes_, need);
    if (st != KDA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (tokens == 0) return copy_state(grad_final_state, grad_initial_state, (size_t)B * H * dk * dv, s);
    return from_cuda(kda::chunk_bwd(q, k, v, beta, log_alpha, initial_state, grad_o, grad_final_state, grad_q, grad_k,
                                    grad_v, grad_beta, grad_log_alpha, grad_initial_state, nullptr, B, T, tokens, H, dk,
                                    dv, dtype, workspace, workspace_bytes_, s));
}

kda_status kda_varlen_bwd(const void* q, const void* k, const void* v, const float* beta, const float* log_alpha,
                          const int32_t* cu_seqlens, int N, const float* initial_state, const float* grad_o,
                          const float* grad_final_state, float* grad_q, float* grad_k, float* grad_v,
                          float* grad_beta, float* grad_log_alpha, float* grad_initial_state, int T, int H, int dk,
                          int dv, int chunk, kda_dtype dtype, void* workspace, size_t workspace_bytes_, void* stream)
{
    if (N < 0 || N > 65535 || T < 0) return KDA_ERR_INVALID_ARG;
    kda_status st = check_bwd(q, k, v, beta, log_alpha, initial_state, grad_o, grad_final_state, grad_q, grad_k,
                              grad_v, grad_beta, grad_log_alpha, grad_initial_state, T, H, dk, dv, chunk, dtype);
    if (st != KDA_OK) return st;
    if (N == 0) return T == 0 ? KDA_OK : KDA_ERR_INVALID_ARG;
    if (!cu_seqlens || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return KDA_ERR_INVALID_ARG;
    const size_t need = T == 0 ? 0 : kda::chunk_bwd_workspace(N, 0, T, H, dk, dv, true);
    st = check_workspace(workspace, workspace_bytes_, need);
    if (st != KDA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) return copy_state(grad_final_state, grad_initial_state, (size_t)N * H * dk * dv, s);
    return from_cuda(kda::chunk_bwd(q, k, v, beta, log_alpha, initial_state, grad_o, grad_final_state, grad_q, grad_k,
                                    grad_v, grad_beta, grad_log_alpha, grad_initial_state, cu_seqlens, N, 0, T, H, dk,
                                    dv, dtype, workspace, workspace_bytes_, s));
}

kda_status kda_dplr_fwd_workspace_size(int B, int T, int H, int dk, int dv, int chunk, kda_dtype dtype,
                                       size_t* bytes)
{
    if (!bytes || B < 0 || T < 0) return KDA_ERR_INVALID_ARG;
    const kda_status st = check_sizes(H, dk, dv, chunk, dtype, 0);
    if (st != KDA_OK) return st;
    const long long tokens = (long long)B * T;
    if (tokens > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    *bytes = tokens == 0 ? 0 : kda::dplr_fwd_workspace(B, T, tokens, H, dk, dv, false);
    return KDA_OK;
}

kda_status kda_dplr_varlen_fwd_workspace_size(int N, int T, int H, int dk, int dv, int chunk, kda_dtype dtype,
                                              size_t* bytes)
{
    if (!bytes || N < 0 || N > 65535 || T < 0) return KDA_ERR_INVALID_ARG;
    const kda_status st = check_sizes(H, dk, dv, chunk, dtype, 0);
    if (st != KDA_OK) return st;
    *bytes = (N == 0 || T == 0) ? 0 : kda::dplr_fwd_workspace(N, 0, T, H, dk, dv, true);
    return KDA_OK;
}

kda_status kda_dplr_fwd(const void* q, const void* k, const void* v, const void* a, const void* b,
                        const float* log_alpha, const float* initial_state, void* o, float* final_state, int B, int T,
                        int H, int dk, int dv, int chunk, kda_dtype dtype, kda_dtype o_dtype, void* workspace,
                        size_t workspace_bytes, void* stream)
{
    if (B < 0 || T < 0) return KDA_ERR_INVALID_ARG;
    const long long tokens = (long long)B * T;
    kda_status st = check_fwd(q, k, v, (const float*)q, log_alpha, initial_state, o, final_state, tokens, H, dk, dv,
                              chunk, dtype, o_dtype, 0);
    if (st != KDA_OK) return st;
    if (tokens > 0 && (!a || !b || !aligned16(a) || !aligned16(b))) return KDA_ERR_INVALID_ARG;
    if (tokens > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (tokens == 0) return copy_state(initial_state, final_state, (size_t)B * H * dk * dv, s);
    st = check_workspace(workspace, workspace_bytes, kda::dplr_fwd_workspace(B, T, tokens, H, dk, dv, false));
    if (st != KDA_OK) return st;
    return from_cuda(kda::dplr_fwd(q, k, v, a, b, log_alpha, initial_state, o, final_state, nullptr, B, T, tokens, H, dk,
                                   dv, dtype, o_dtype, workspace, workspace_bytes, s));
}

kda_status kda_dplr_varlen_fwd(const void* q, const void* k, const void* v, const void* a, const void* b,
                               const float* log_alpha, const int32_t* cu_seqlens, int N, const float* initial_state,
                               void* o, float* final_state, int T, int H, int dk, int dv, int chunk, kda_dtype dtype,
                               kda_dtype o_dtype, void* workspace, size_t workspace_bytes, void* stream)
{
    if (N < 0 || N > 65535 || T < 0) return KDA_ERR_INVALID_ARG;
    kda_status st = check_fwd(q, k, v, (const float*)q, log_alpha, initial_state, o, final_state, T, H, dk, dv, chunk,
                              dtype, o_dtype, 0);
    if (st != KDA_OK) return st;
    if (T > 0 && (!a || !b || !aligned16(a) || !aligned16(b))) return KDA_ERR_INVALID_ARG;
    if (N == 0) return T == 0 ? KDA_OK : KDA_ERR_INVALID_ARG;
    if (!cu_seqlens || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return KDA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) return copy_state(initial_state, final_state, (size_t)N * H * dk * dv, s);
    st = check_workspace(workspace, workspace_bytes, kda::dplr_fwd_workspace(N, 0, T, H, dk, dv, true));
    if (st != KDA_OK) return st;
    return from_cuda(kda::dplr_fwd(q, k, v, a, b, log_alpha, initial_state, o, final_state, cu_seqlens, N, 0, T, H, dk,
                                   dv, dtype, o_dtype, workspace, workspace_bytes, s));
}

kda_status kda_check(void* stream)
{
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
    unsigned word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, kda::g_status, sizeof(word)) != cudaSuccess) return KDA_ERR_CUDA;
    if (word && cudaMemcpyToSymbol(kda::g_status, &zero, sizeof(zero)) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (word & kda::KDA_DEV_ERR_TIMEOUT) return KDA_ERR_TIMEOUT;
    if (word & kda::KDA_DEV_ERR_BAD_INPUT) return KDA_ERR_INVALID_ARG;
    if (word & kda::KDA_DEV_WARN_DOMAIN) return KDA_WARN_DOMAIN;
    return KDA_OK;
}

kda_status kda_selftest_timeout(long long limit_cycles, void* stream)
{
    if (limit_cycles < 1 || limit_cycles > (1LL << 32)) return KDA_ERR_INVALID_ARG;
    selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles);
    return from_cuda(cudaGetLastError());
}

const char* kda_status_string(kda_status status)
{
    switch (status) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: null, misaligned or out-of-range argument";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: size or type not implemented";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: a CUDA runtime call or kernel launch failed";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a device-side bounded wait ran out";
    case KDA_WARN_DOMAIN:
        return "KDA_WARN_DOMAIN: a chunk's gate decay left the mid-chunk factorisation range (results inexact)";
    }
    return "KDA_ERR_UNKNOWN";
}

int kda_version(void) { return 200; }

}  // extern "C"
