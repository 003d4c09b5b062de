// Building blocks shared by the tensor-core chunk kernels: the UT-transform
// inversion on CUDA cores, operand descriptors and layouts, sequence ordering
// and the TMA tensor maps of the [tokens, H, d] inputs.
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
constexpr int LDA = 65;    // fp32 pitch of the UT-transform scratch

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

// T[k][j] of the unit lower-triangular T, kept transposed in the upper
// triangle (diagonal included) of the UT scratch.
__device__ __forceinline__ float Tget(const float* As, int k, int j) { return k >= j ? As[j * LDA + k] : 0.f; }

// UT transform, run by the first 128 threads (named barrier 1; the other
// warps are free meanwhile).  On entry As[r*LDA + s] (s < r) holds the
// strictly lower A; on return As[j*LDA + s] (s >= j) holds T[s][j],
// T = (I + A)^-1, with A left intact below the diagonal.  Diagonal 16x16
// blocks by column-sweep forward substitution (one lane per column), then
// T10 = -T11 A10 T00, T32 = -T33 A32 T22 (2x2 register tiles) and the
// lower-left 32x32 block -T_BB A_BA T_AA (2x4 register tiles).
__device__ __forceinline__ void ut_transform(float* As, float* X)
{
    const int tid = threadIdx.x;
    if (tid < 64) {
        const int b0 = 16 * (tid >> 4), j = tid & 15;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
        for (int s = 0; s < 15; ++s) {
            const float xs = x[s];
#pragma unroll
            for (int r = s + 1; r < 16; ++r) x[r] = fmaf(-As[(b0 + r) * LDA + b0 + s], xs, x[r]);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r)
            if (r >= j) As[(b0 + j) * LDA + b0 + r] = x[r];
    }
    bar_sync(1, 128);
    {
        const int blk = tid >> 6, tile = tid & 63, i0 = (tile >> 3) * 2, j0 = (tile & 7) * 2;
        const int rb = blk ? 48 : 16, cb = blk ? 32 : 0;
        float a[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float u0 = As[(rb + i0) * LDA + cb + k], u1 = As[(rb + i0 + 1) * LDA + cb + k];
            const float t0 = Tget(As, cb + k, cb + j0), t1 = Tget(As, cb + k, cb + j0 + 1);
            a[0][0] = fmaf(u0, t0, a[0][0]); a[0][1] = fmaf(u0, t1, a[0][1]);
            a[1][0] = fmaf(u1, t0, a[1][0]); a[1][1] = fmaf(u1, t1, a[1][1]);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int v = 0; v < 2; ++v) X[(blk * 16 + i0 + u) * 33 + j0 + v] = a[u][v];
        bar_sync(1, 128);
        float t[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float w0 = Tget(As, rb + i0, rb + k), w1 = Tget(As, rb + i0 + 1, rb + k);
            const float x0 = X[(blk * 16 + k) * 33 + j0], x1 = X[(blk * 16 + k) * 33 + j0 + 1];
            t[0][0] = fmaf(w0, x0, t[0][0]); t[0][1] = fmaf(w0, x1, t[0][1]);
            t[1][0] = fmaf(w1, x0, t[1][0]); t[1][1] = fmaf(w1, x1, t[1][1]);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int v = 0; v < 2; ++v) As[(cb + j0 + v) * LDA + rb + i0 + u] = -t[u][v];
    }
    bar_sync(1, 128);
    {
        const int i0 = (tid >> 3) * 2, j0 = (tid & 7) * 4;
        float a[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
            const float u0 = As[(32 + i0) * LDA + k], u1 = As[(32 + i0 + 1) * LDA + k];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const float tv = Tget(As, k, j0 + v);
                a[0][v] = fmaf(u0, tv, a[0][v]);
                a[1][v] = fmaf(u1, tv, a[1][v]);
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) X[(i0 + u) * 33 + j0 + v] = a[u][v];
        bar_sync(1, 128);
        float t[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
            const float w0 = Tget(As, 32 + i0, 32 + k), w1 = Tget(As, 32 + i0 + 1, 32 + k);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const float xv = X[k * 33 + j0 + v];
                t[0][v] = fmaf(w0, xv, t[0][v]);
                t[1][v] = fmaf(w1, xv, t[1][v]);
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) As[(j0 + v) * LDA + 32 + i0 + u] = -t[u][v];
    }
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
