// Recurrent (decode) step of the KDA layer: one new token per sequence.
//
// Recurrent form of "Hybrid Linear Attention Architecture: Making LLM Training
// and Inference More Efficient", section 3.3 (decay per channel, then erase
// and write), output read after the write ("Demystifying Hybrid LLM
// Architectures", section 2.3).  Per (sequence, head), with Shat = Diag(a) S:
//   r = Shat^T k,  y = Shat^T q,  delta = beta (v - r),
//   S' = Shat + k delta^T,  o = S'^T q = y + delta (k . q).
// The fp32 state is streamed exactly once: every thread keeps its share of S in
// registers between the column reductions and the write-back, so HBM sees one
// read and one write of each state per step (the roofline of this kernel).
//
// Layout: one CTA of 256 threads per (sequence, head, 64 value columns).  A
// thread owns 4 adjacent columns (one 16-byte vector) of every 16th key row;
// 16 consecutive threads read one contiguous 256-byte row segment.
#include "kda_common.cuh"

namespace kda {

template <typename T, typename TO, int DK, int DV>
__global__ void __launch_bounds__(256)
decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   const float* __restrict__ beta, const float* __restrict__ log_alpha,
                   float* __restrict__ state, TO* __restrict__ o, int mode)
{
    const bool head_gate = (mode & KDA_MODE_HEAD_GATE) != 0;   // log_alpha [NH]: one gate per head
    const bool erase = (mode & KDA_MODE_NO_ERASE) == 0;
    const bool logits = (mode & KDA_MODE_GATE_LOGITS) != 0;
    const bool norm_qk = (mode & KDA_MODE_NORM_QK) != 0;
    constexpr int COLS = 64;
    constexpr int SPLIT = DV / COLS;
    constexpr int RPT = DK / 16;          // key rows per thread
    const int head = blockIdx.x / SPLIT;  // flattened (sequence, head)
    const int col0 = (blockIdx.x % SPLIT) * COLS;
    const int t = threadIdx.x, cg = t & 15, rg = t >> 4, lane = t & 31, w = t >> 5;

    float* S = state + (size_t)head * DK * DV + col0 + 4 * cg;

    // Issue the whole state read first: RPT independent 16-byte loads per thread.
    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
        s[i] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)(rg + 16 * i) * DV));

    __shared__ float sk[DK], sq[DK], sa[DK];
    __shared__ float red[8][16][8];
    __shared__ float s_kq;
    for (int i = t; i < DK; i += 256) {
        sk[i] = Elem<T>::load(k + (size_t)head * DK + i);
        sq[i] = Elem<T>::load(q + (size_t)head * DK + i);
        const float g = head_gate ? log_alpha[head] : log_alpha[(size_t)head * DK + i];
        sa[i] = logits ? 1.f / (1.f + expf(g)) : expf(g);   // sigmoid(-z) = exp(-softplus(z))
    }
    __syncthreads();
    if (norm_qk) {   // raw q, k: divide each by its L2 norm
        __shared__ float s_inv[2];
        if (w == 0) {
            float nk = 0.f, nq = 0.f;
            for (int i = lane; i < DK; i += 32) { nk = fmaf(sk[i], sk[i], nk); nq = fmaf(sq[i], sq[i], nq); }
            nk = warp_sum(nk);
            nq = warp_sum(nq);
            if (lane == 0) { s_inv[0] = inv_norm(nk); s_inv[1] = inv_norm(nq); }
        }
        __syncthreads();
        for (int i = t; i < DK; i += 256) { sk[i] *= s_inv[0]; sq[i] *= s_inv[1]; }
        __syncthreads();
    }

    float r[4] = {0.f, 0.f, 0.f, 0.f}, y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int row = rg + 16 * i;
        const float a = sa[row], kk = sk[row], qq = sq[row];
        s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
        r[0] = fmaf(kk, s[i].x, r[0]); r[1] = fmaf(kk, s[i].y, r[1]);
        r[2] = fmaf(kk, s[i].z, r[2]); r[3] = fmaf(kk, s[i].w, r[3]);
        y[0] = fmaf(qq, s[i].x, y[0]); y[1] = fmaf(qq, s[i].y, y[1]);
        y[2] = fmaf(qq, s[i].z, y[2]); y[3] = fmaf(qq, s[i].w, y[3]);
    }
    // Lanes l and l^16 hold the same columns for two row groups.
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        r[j] += __shfl_xor_sync(0xffffffffu, r[j], 16);
        y[j] += __shfl_xor_sync(0xffffffffu, y[j], 16);
    }
    if (lane < 16) {
#pragma unroll
        for (int j = 0; j < 4; ++j) { red[w][cg][j] = r[j]; red[w][cg][4 + j] = y[j]; }
    }
    if (w == 0) {
        float p = 0.f;
        for (int i = lane; i < DK; i += 32) p = fmaf(sk[i], sq[i], p);
        p = warp_sum(p);
        if (lane == 0) s_kq = p;
    }
    __syncthreads();

    float R[4] = {0.f, 0.f, 0.f, 0.f}, Y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ww = 0; ww < 8; ++ww)
#pragma unroll
        for (int j = 0; j < 4; ++j) { R[j] += red[ww][cg][j]; Y[j] += red[ww][cg][4 + j]; }

    const float b = beta[head];
    float d[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        d[j] = b * (Elem<T>::load(v + (size_t)head * DV + col0 + 4 * cg + j) - (erase ? R[j] : 0.f));

#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const float kk = sk[rg + 16 * i];
        s[i].x = fmaf(kk, d[0], s[i].x); s[i].y = fmaf(kk, d[1], s[i].y);
        s[i].z = fmaf(kk, d[2], s[i].z); s[i].w = fmaf(kk, d[3], s[i].w);
        __stcs(reinterpret_cast<float4*>(S + (size_t)(rg + 16 * i) * DV), s[i]);
    }
    if (rg == 0) {
        const float kq = s_kq;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            Elem<TO>::store(o + (size_t)head * DV + col0 + 4 * cg + j, fmaf(d[j], kq, Y[j]));
    }
}

template <typename T, typename TO, int DK, int DV>
static cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* beta,
                                 const float* log_alpha, float* state, void* o, long long NH,
                                 int mode, cudaStream_t stream)
{
    const long long blocks = NH * (DV / 64);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    decode_step_kernel<T, TO, DK, DV><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), beta,
        log_alpha, state, static_cast<TO*>(o), mode);
    return cudaGetLastError();
}

template <typename T, typename TO>
static cudaError_t decode_dims(const void* q, const void* k, const void* v, const float* beta,
                               const float* log_alpha, float* state, void* o, long long NH, int dk,
                               int dv, int mode, cudaStream_t s)
{
    if (dk == 128 && dv == 128) return launch_decode<T, TO, 128, 128>(q, k, v, beta, log_alpha, state, o, NH, mode, s);
    if (dk == 128 && dv == 64) return launch_decode<T, TO, 128, 64>(q, k, v, beta, log_alpha, state, o, NH, mode, s);
    if (dk == 64 && dv == 128) return launch_decode<T, TO, 64, 128>(q, k, v, beta, log_alpha, state, o, NH, mode, s);
    if (dk == 64 && dv == 64) return launch_decode<T, TO, 64, 64>(q, k, v, beta, log_alpha, state, o, NH, mode, s);
    return cudaErrorInvalidValue;
}

cudaError_t decode_step(const void* q, const void* k, const void* v, const float* beta,
                        const float* log_alpha, float* state, void* o, long long NH, int dk,
                        int dv, kda_dtype dtype, kda_dtype o_dtype, int mode, cudaStream_t s)
{
    using bf = __nv_bfloat16;
    if (dtype == KDA_BF16 && o_dtype == KDA_BF16) return decode_dims<bf, bf>(q, k, v, beta, log_alpha, state, o, NH, dk, dv, mode, s);
    if (dtype == KDA_BF16 && o_dtype == KDA_F32) return decode_dims<bf, float>(q, k, v, beta, log_alpha, state, o, NH, dk, dv, mode, s);
    if (dtype == KDA_F32 && o_dtype == KDA_BF16) return decode_dims<float, bf>(q, k, v, beta, log_alpha, state, o, NH, dk, dv, mode, s);
    return decode_dims<float, float>(q, k, v, beta, log_alpha, state, o, NH, dk, dv, mode, s);
}

}  // namespace kda
