// Building blocks of the tensor-core chunk kernels: operand descriptors and
// layouts, the hardware reciprocal, and the TMA tensor maps of the
// [tokens, H, d] inputs.
#pragma once

#include "kda_sm100.cuh"

#include <cudaTypedefs.h>

// Phase markers: empty in the library build.  A profiling build may define
// them to accumulate clock64() deltas per kernel (id) and chunk stage (i).
#ifndef KDA_PHASE
#define KDA_PHASE_DECL(id)
#define KDA_PHASE(i) ((void)0)
#define KDA_PHASE_FLUSH
#endif

namespace kda {
namespace tcu {

using namespace sm100;

constexpr int C = 64;      // chunk length

__device__ __forceinline__ unsigned char* align1024(unsigned char* p)
{
    const uint32_t a = smem_u32(p);
    return p + (((a + 1023u) & ~1023u) - a);
}

// 1/x by the hardware reciprocal (PTX rcp.approx.ftz.f32: relative error
// within 2^-23 for normal x; subnormal inputs and results flush to zero).
// Used for factors e^(G_m - G) in [e^-80, e^80], whose products are then
// rounded to tf32 (2^-11).
__device__ __forceinline__ float rcp_approx(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// K-major SW128 operand descriptor for MMA k-step kk (32 bytes of K per step:
// 8 tf32 or 16 fp16 elements): 4 steps per 128-byte atom column, atom columns
// `atom_stride` bytes apart.
__device__ __forceinline__ uint64_t kdesc(const unsigned char* tile, int kk, int atom_stride)
{
    return sdesc_sw128(smem_u32(tile) + (kk >> 2) * atom_stride + (kk & 3) * 32, 16, 1024);
}

__device__ __forceinline__ float4 bf16x4(const __nv_bfloat16* p)
{
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ float4 tf32r4(float a, float b, float c, float d)
{
    return make_float4(tf32r(a), tf32r(b), tf32r(c), tf32r(d));
}

}  // namespace tcu

namespace tcu_host {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// [tokens, H, D] (bf16 or fp32), box = 64 tokens x 1 head x `box_d` channels
// (all D by default), no swizzle or the 128-byte swizzle (box_d x element
// size must then be 128 bytes); rows past the end of the tensor are filled
// with zeros.
inline bool make_tmap(CUtensorMap* m, const void* base, long long tokens, int H, int D, bool fp32, int box_d = 0,
                      bool swizzle128 = false)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t es = fp32 ? 4 : 2;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)tokens};
    const cuuint64_t strides[2] = {(cuuint64_t)D * es, (cuuint64_t)H * D * es};
    const cuuint32_t box[3] = {(cuuint32_t)(box_d > 0 ? box_d : D), 1, (cuuint32_t)tcu::C};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tcu_host
}  // namespace kda
