// C ABI of the KDA library: argument validation, path selection, status codes.
// Declarations and the contract of every entry point are in include/kda.h.
#include <string.h>
#include <cuda_runtime.h>
#include <stdlib.h>

#include "kda_chunk.cuh"
#include "kda_sm100.cuh"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool supported_d(int d) { return d == 64 || d == 128; }

bool valid_dtype(kda_dtype t) { return t == KDA_F32 || t == KDA_BF16; }

kda_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

// Kernel selection for bf16 inputs: the two-pass tensor-core forward by
// default; KDA_CHUNK_KERNEL=fused selects the single-pass tensor-core kernel
// and KDA_CHUNK_KERNEL=simt (or KDA_FORCE_SIMT=1) the CUDA-core kernel (used
// by tests that compare the kernels).  KDA_TIMEOUT_CYCLES bounds every
// device-side wait of the tensor-core kernels (default 2^31 SM cycles, about
// one second).
enum class ChunkKernel { split, fused, simt };
ChunkKernel chunk_kernel()
{
    const char* f = getenv("KDA_FORCE_SIMT");
    if (f && f[0] == '1') return ChunkKernel::simt;
    const char* e = getenv("KDA_CHUNK_KERNEL");
    if (e && strcmp(e, "fused") == 0) return ChunkKernel::fused;
    if (e && strcmp(e, "simt") == 0) return ChunkKernel::simt;
    return ChunkKernel::split;
}

long long timeout_cycles()
{
    const char* e = getenv("KDA_TIMEOUT_CYCLES");
    long long v = e ? atoll(e) : 0;
    return v > 0 ? v : (1LL << 31);
}

kda_status run_chunk(const void* q, const void* k, const void* v, const float* beta,
                     const float* log_alpha, const float* s0, void* o, float* sT, const int32_t* cu,
                     int nseq, int T, long long tokens, int H, int dk, int dv, kda_dtype dtype,
                     kda_dtype o_dtype, int mode, cudaStream_t s)
{
    const ChunkKernel kind = chunk_kernel();
    // the single-pass kernel implements the plain layer only: variants take the two-pass path
    if (kda::chunk_fwd_tc_supported(dk, dv, dtype) && kind == ChunkKernel::fused && mode == 0)
        return from_cuda(kda::chunk_fwd_tc(q, k, v, beta, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dk,
                                           dv, o_dtype, timeout_cycles(), s));
    if (kda::chunk_fwd_tc_supported(dk, dv, dtype) && kind != ChunkKernel::simt)
        return from_cuda(kda::chunk_fwd_split(q, k, v, beta, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dk,
                                              dv, o_dtype, timeout_cycles(), mode, s));
    return from_cuda(kda::chunk_fwd_simt(q, k, v, beta, log_alpha, s0, o, sT, cu, nseq, T, H, dk, dv, dtype,
                                         o_dtype, mode, s));
}

bool valid_mode(int mode)
{
    return (mode & ~(KDA_MODE_HEAD_GATE | KDA_MODE_NO_ERASE | KDA_MODE_NORM_QK | KDA_MODE_GATE_LOGITS)) == 0;
}

// Shared checks of the forward entry points.
kda_status check_fwd(const void* q, const void* k, const void* v, const float* beta,
                     const float* log_alpha, const float* s0, const void* o, const float* sT,
                     long long tokens, int H, int dk, int dv, int chunk, kda_dtype dtype,
                     kda_dtype o_dtype, int mode)
{
    if (H <= 0 || dk <= 0 || dv <= 0 || tokens < 0) return KDA_ERR_INVALID_ARG;
    if (!valid_dtype(dtype) || !valid_dtype(o_dtype) || !valid_mode(mode)) return KDA_ERR_INVALID_ARG;
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

kda_status kda_chunk_fwd_mode(const void* q, const void* k, const void* v, const float* beta,
                              const float* log_alpha, const float* initial_state, void* o,
                              float* final_state, int B, int T, int H, int dk, int dv, int chunk,
                              kda_dtype dtype, kda_dtype o_dtype, int mode, void* stream)
{
    if (B < 0 || T < 0) return KDA_ERR_INVALID_ARG;
    const long long tokens = (long long)B * T;
    kda_status st = check_fwd(q, k, v, beta, log_alpha, initial_state, o, final_state, tokens, H,
                              dk, dv, chunk, dtype, o_dtype, mode);
    if (st != KDA_OK) return st;
    if (tokens > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (tokens == 0) return copy_state(initial_state, final_state, (size_t)B * H * dk * dv, s);
    return run_chunk(q, k, v, beta, log_alpha, initial_state, o, final_state, nullptr, B, T, tokens, H, dk,
                     dv, dtype, o_dtype, mode, s);
}

kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const float* beta,
                         const float* log_alpha, const float* initial_state, void* o,
                         float* final_state, int B, int T, int H, int dk, int dv, int chunk,
                         kda_dtype dtype, kda_dtype o_dtype, void* stream)
{
    return kda_chunk_fwd_mode(q, k, v, beta, log_alpha, initial_state, o, final_state, B, T, H, dk, dv, chunk,
                              dtype, o_dtype, 0, stream);
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
    if (!kda::chunk_fwd_tc_supported(dk, dv, dtype))   // the CUDA-core kernel needs no scratch
        return from_cuda(kda::chunk_fwd_simt(q, k, v, beta, log_alpha, initial_state, o, final_state, nullptr, B,
                                             T, H, dk, dv, dtype, o_dtype, 0, s));
    if (!kda::chunk_fwd_noalloc_fits(B, T, H, dk, dv, final_state != nullptr)) return KDA_ERR_UNSUPPORTED;
    return from_cuda(kda::chunk_fwd_noalloc(q, k, v, beta, log_alpha, initial_state, o, final_state, B, T, tokens,
                                            H, dk, dv, o_dtype, timeout_cycles(), s));
}

kda_status kda_varlen_fwd_mode(const void* q, const void* k, const void* v, const float* beta,
                               const float* log_alpha, const int32_t* cu_seqlens, int N,
                               const float* initial_state, void* o, float* final_state, int T, int H,
                               int dk, int dv, int chunk, kda_dtype dtype, kda_dtype o_dtype, int mode,
                               void* stream)
{
    if (N < 0 || N > 65535 || T < 0) return KDA_ERR_INVALID_ARG;
    kda_status st = check_fwd(q, k, v, beta, log_alpha, initial_state, o, final_state, T, H, dk,
                              dv, chunk, dtype, o_dtype, mode);
    if (st != KDA_OK) return st;
    if (N == 0) return T == 0 ? KDA_OK : KDA_ERR_INVALID_ARG;
    if (!cu_seqlens || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return KDA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) return copy_state(initial_state, final_state, (size_t)N * H * dk * dv, s);
    return run_chunk(q, k, v, beta, log_alpha, initial_state, o, final_state, cu_seqlens, N, T, T, H, dk,
                     dv, dtype, o_dtype, mode, s);
}

kda_status kda_varlen_fwd(const void* q, const void* k, const void* v, const float* beta,
                          const float* log_alpha, const int32_t* cu_seqlens, int N,
                          const float* initial_state, void* o, float* final_state, int T, int H,
                          int dk, int dv, int chunk, kda_dtype dtype, kda_dtype o_dtype,
                          void* stream)
{
    return kda_varlen_fwd_mode(q, k, v, beta, log_alpha, cu_seqlens, N, initial_state, o, final_state, T, H,
                               dk, dv, chunk, dtype, o_dtype, 0, stream);
}

kda_status kda_recurrent_step_mode(const void* q, const void* k, const void* v, const float* beta,
                                   const float* log_alpha, float* state, void* o, int N, int H, int dk,
                                   int dv, kda_dtype dtype, kda_dtype o_dtype, int mode, void* stream)
{
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (!valid_dtype(dtype) || !valid_dtype(o_dtype) || !valid_mode(mode)) return KDA_ERR_INVALID_ARG;
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
    }
    return "KDA_ERR_UNKNOWN";
}

int kda_version(void) { return 100; }

}  // extern "C"
