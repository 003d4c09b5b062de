// Shared device helpers of the KDA CUDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

// Per-device status word (the library is one translation unit, so this is its
// only definition).  Kernels set bits here when a bounded wait gives up or
// when device-resident arguments (sequence boundaries) fall outside the
// buffers they index, in which case the affected sequence is skipped, or
// when a chunk's gate decay leaves the range of the mid-chunk factorisation;
// kda_check() reads and clears it.
enum : unsigned { KDA_DEV_ERR_TIMEOUT = 1u, KDA_DEV_ERR_BAD_INPUT = 2u, KDA_DEV_WARN_DOMAIN = 4u };
__device__ unsigned g_status = 0;

__device__ __forceinline__ void flag_timeout() { atomicOr(&g_status, KDA_DEV_ERR_TIMEOUT); }
__device__ __forceinline__ void flag_bad_input() { atomicOr(&g_status, KDA_DEV_ERR_BAD_INPUT); }

// Factors exp(G - G_m) of a chunk are clamped at exp(+-80); G is monotone
// (log alpha <= 0), so for one channel the extremes are the first row, G_0,
// and the last, G_last.  Flags the chunk when either lies outside the clamp.
__device__ __forceinline__ void check_domain(float g0, float gm, float glast)
{
    if (g0 - gm > 80.f || gm - glast > 80.f) atomicOr(&g_status, KDA_DEV_WARN_DOMAIN);
}

// Element access for the two supported q/k/v/o element types.
template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float* p) { return *p; }
    static __device__ __forceinline__ void store(float* p, float x) { *p = x; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// log alpha from a gate logit z (KDA_MODE_GATE_LOGITS): -softplus(z) =
// -(max(z, 0) + log(1 + e^-|z|)), without overflow for any finite z.
__device__ __forceinline__ float neg_softplus(float z) { return -(fmaxf(z, 0.f) + log1pf(expf(-fabsf(z)))); }

// 1 / max(||x||, 1e-15) from ||x||^2 (KDA_MODE_NORM_QK; rows of zero norm stay zero).
__device__ __forceinline__ float inv_norm(float sq) { return rsqrtf(fmaxf(sq, 1e-30f)); }

}  // namespace kda
