// Chunkwise forward of the diagonal-plus-low-rank transition on CUDA cores
// (fp32 arithmetic): the "finer granularity" gate of "Hybrid Linear Attention
// Architecture: Making LLM Training and Inference More Efficient", section 3.3
// (a low-rank correction on top of the element-wise decay), in this library's
// d_k x d_v orientation:
//
//   S_t = (Diag(alpha_t) + b_t a_t^T) S_{t-1} + k_t v_t^T,     o_t = S_t^T q_t.
//
// Per chunk, with G the inclusive cumulative sum of log alpha, Gx the
// exclusive one, u_s = S_{s-1}^T a_s and the state before the chunk S:
//
//   A_ab[s][t] = a_s . (e^{Gx_s - G_t} b_t),  A_ak[s][t] = a_s . (e^{Gx_s - G_t} k_t)   (t < s)
//   P_qb[r][s] = q_r . (e^{G_r - G_s} b_s),   P_qk[r][s] = q_r . (e^{G_r - G_s} k_s)    (s <= r)
//   U = (I - A_ab)^-1 ((e^{Gx} a) S + A_ak V)
//   O = (e^G q) S + P_qb U + P_qk V
//   S <- Diag(e^{G_last}) S + (e^{G_last - G} b)^T U + (e^{G_last - G} k)^T V
//
// The relative decays are factored around the chunk's middle row m (every
// factor bounded by the decay of 32 tokens): ax = a e^{Gx - G_m},
// qx = q e^{G - G_m}, bf = b e^{G_m - G}, kf = k e^{G_m - G}, and the
// per-channel e^{G_m}, e^{G_last - G_m} are folded into the state products.
//
// One CTA (256 threads) per (sequence, head, 16 value columns); columns of S
// evolve independently (the transition acts on the d_k side).  The operand
// tiles are retired in two rounds so that everything fits in shared memory.
#include "kda_chunk.cuh"

namespace kda {

namespace dplr {

using simt::mma_tile;

constexpr int C = 64;
constexpr int NV = 16;
constexpr int NT = 256;

template <int DK>
struct Smem {
    static constexpr int LDK = DK + 1;
    static constexpr int LDC = C + 1;
    float ax[C * LDK];    // a e^{Gx - G_m}, then q e^{G - G_m}
    float bf[C * LDK];    // b e^{G_m - G}
    float kf[C * LDK];    // k e^{G_m - G}
    float gq[C * LDK];    // cumulative gate G
    float M1[C * LDC];    // A_ab, then P_qb
    float M2[C * LDC];    // A_ak, then P_qk
    float T[C * LDC];     // (I - A_ab)^-1
    float S[DK * NV];     // state slice
    float Sm[DK * NV];    // e^{G_m} S
    float V[C * NV];
    float W[C * NV];      // (e^{Gx} a) S + A_ak V, then U
    float O[C * NV];      // (e^G q) S, then the output rows
    float gm[DK], gam[DK], glm[DK];
};

template <typename TIn, typename TOut, int DK>
__global__ void __launch_bounds__(NT)
dplr_fwd_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                const TIn* __restrict__ a, const TIn* __restrict__ b, const float* __restrict__ log_alpha,
                const float* s0, TOut* __restrict__ o, float* sT, const int32_t* __restrict__ cu, int nseq, int T,
                long long tokens, int H, int DV)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem<DK>& sm = *reinterpret_cast<Smem<DK>*>(smem_raw);
    constexpr int LDK = Smem<DK>::LDK, LDC = Smem<DK>::LDC;
    constexpr int TK = DK / 16;
    const int nslice = DV / NV;
    const int slice = blockIdx.x % nslice;
    const int h = (blockIdx.x / nslice) % H;
    const int n = blockIdx.x / (nslice * H);
    const int col0 = slice * NV;
    const int tid = threadIdx.x, tn = tid % 16, tm = tid / 16;
    int tok0, len;
    if (cu) {   // a range outside the token axis is skipped (its final state is its initial one)
        tok0 = cu[n];
        len = max(0, cu[n + 1] - tok0);
        if (tok0 < 0 || (long long)tok0 + len > tokens) {
            if (tid == 0) flag_bad_input();
            tok0 = 0;
            len = 0;
        }
    } else {
        tok0 = n * T;
        len = T;
    }
    for (int e = tid; e < DK * NV; e += NT) {
        const int c = e / NV, j = e % NV;
        sm.S[e] = s0 ? s0[(((size_t)n * H + h) * DK + c) * DV + col0 + j] : 0.f;
    }

    for (int t0 = 0; t0 < len; t0 += C) {
        const int L = min(C, len - t0);
        __syncthreads();
        // ---- load (rows >= L are zero: no key, no value, no decay)
        for (int e = tid; e < C * DK; e += NT) {
            const int r = e / DK, c = e % DK;
            float av = 0.f, bv = 0.f, kv = 0.f, gv = 0.f;
            if (r < L) {
                const size_t off = ((size_t)(tok0 + t0 + r) * H + h) * DK + c;
                av = Elem<TIn>::load(a + off);
                bv = Elem<TIn>::load(b + off);
                kv = Elem<TIn>::load(k + off);
                gv = log_alpha[off];
            }
            sm.ax[r * LDK + c] = av;
            sm.bf[r * LDK + c] = bv;
            sm.kf[r * LDK + c] = kv;
            sm.gq[r * LDK + c] = gv;
        }
        for (int e = tid; e < C * NV; e += NT) {
            const int r = e / NV, j = e % NV;
            sm.V[e] = r < L ? Elem<TIn>::load(v + ((size_t)(tok0 + t0 + r) * H + h) * DV + col0 + j) : 0.f;
        }
        __syncthreads();
        // ---- gate cumsum per channel and the factor split around the middle row
        if (tid < DK) {
            const int c = tid;
            float acc = 0.f;
            for (int r = 0; r < C; ++r) { acc += sm.gq[r * LDK + c]; sm.gq[r * LDK + c] = acc; }
            const float Gm = sm.gq[(C / 2 - 1) * LDK + c];
            sm.gm[c] = expf(Gm);
            sm.gam[c] = expf(acc);
            sm.glm[c] = expf(acc - Gm);
            float gprev = 0.f;   // Gx of row r = G of row r - 1
            for (int r = 0; r < C; ++r) {
                const float G = sm.gq[r * LDK + c];
                const float f = expf(fminf(Gm - G, 80.f));
                sm.ax[r * LDK + c] *= expf(fminf(gprev - Gm, 80.f));
                sm.bf[r * LDK + c] *= f;
                sm.kf[r * LDK + c] *= f;
                gprev = G;
            }
        }
        __syncthreads();
        for (int e = tid; e < DK * NV; e += NT) sm.Sm[e] = sm.gm[e / NV] * sm.S[e];
        // ---- round 1: A_ab, A_ak (strictly lower) and (e^{Gx} a) S = ax Sm
        {
            float p1[4][4] = {}, p2[4][4] = {};
            mma_tile<4, 4>(p1, sm.ax, LDK, 1, sm.bf, 1, LDK, DK, tm, 16, tn, 16);
            mma_tile<4, 4>(p2, sm.ax, LDK, 1, sm.kf, 1, LDK, DK, tm, 16, tn, 16);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int r = tm + 16 * i, s = tn + 16 * j;
                    sm.M1[r * LDC + s] = s < r ? p1[i][j] : 0.f;
                    sm.M2[r * LDC + s] = s < r ? p2[i][j] : 0.f;
                }
        }
        __syncthreads();
        {
            float w[4][1] = {};
            mma_tile<4, 1>(w, sm.ax, LDK, 1, sm.Sm, NV, 1, DK, tm, 16, tn, 16);
            mma_tile<4, 1>(w, sm.M2, LDC, 1, sm.V, NV, 1, C, tm, 16, tn, 16);
            __syncthreads();
#pragma unroll
            for (int i = 0; i < 4; ++i) sm.W[(tm + 16 * i) * NV + tn] = w[i][0];
        }
        // ---- T = (I - A_ab)^-1 by forward substitution (column j per 4 lanes)
        {
            const int j = tid >> 2, pq = tid & 3;
            for (int r = 0; r < C; ++r) {
                float acc = 0.f;
                if (r > j)
                    for (int s = j + pq; s < r; s += 4) acc = fmaf(sm.M1[r * LDC + s], sm.T[s * LDC + j], acc);
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                if (pq == 0) sm.T[r * LDC + j] = (r == j ? 1.f : 0.f) + (r > j ? acc : 0.f);
                __syncwarp();
            }
        }
        // ---- reload q as q e^{G - G_m} into ax (ax is retired)
        __syncthreads();
        for (int e = tid; e < C * DK; e += NT) {
            const int r = e / DK, c = e % DK;
            float qv = 0.f;
            if (r < L) qv = Elem<TIn>::load(q + ((size_t)(tok0 + t0 + r) * H + h) * DK + c);
            const float G = sm.gq[r * LDK + c], Gm = sm.gq[(C / 2 - 1) * LDK + c];
            sm.ax[r * LDK + c] = qv * expf(fminf(G - Gm, 80.f));
        }
        __syncthreads();
        // ---- round 2: P_qb, P_qk (lower incl.), (e^G q) S = qx Sm; U = T W
        {
            float p1[4][4] = {}, p2[4][4] = {};
            mma_tile<4, 4>(p1, sm.ax, LDK, 1, sm.bf, 1, LDK, DK, tm, 16, tn, 16);
            mma_tile<4, 4>(p2, sm.ax, LDK, 1, sm.kf, 1, LDK, DK, tm, 16, tn, 16);
            float oq[4][1] = {}, u[4][1] = {};
            mma_tile<4, 1>(oq, sm.ax, LDK, 1, sm.Sm, NV, 1, DK, tm, 16, tn, 16);
            mma_tile<4, 1>(u, sm.T, LDC, 1, sm.W, NV, 1, C, tm, 16, tn, 16);
            __syncthreads();
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int r = tm + 16 * i, s = tn + 16 * j;
                    sm.M1[r * LDC + s] = s <= r ? p1[i][j] : 0.f;
                    sm.M2[r * LDC + s] = s <= r ? p2[i][j] : 0.f;
                }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                sm.O[(tm + 16 * i) * NV + tn] = oq[i][0];
                sm.W[(tm + 16 * i) * NV + tn] = u[i][0];
            }
        }
        __syncthreads();
        // ---- O = (e^G q) S + P_qb U + P_qk V  -> output rows < L
        {
            float ov[4][1] = {};
            mma_tile<4, 1>(ov, sm.M1, LDC, 1, sm.W, NV, 1, C, tm, 16, tn, 16);
            mma_tile<4, 1>(ov, sm.M2, LDC, 1, sm.V, NV, 1, C, tm, 16, tn, 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = tm + 16 * i;
                if (r < L)
                    Elem<TOut>::store(o + ((size_t)(tok0 + t0 + r) * H + h) * DV + col0 + tn,
                                      sm.O[r * NV + tn] + ov[i][0]);
            }
        }
        // ---- S <- gamma S + e^{G_last - G_m} (bf^T U + kf^T V)
        {
            float ds[TK][1] = {};
            mma_tile<TK, 1>(ds, sm.bf, 1, LDK, sm.W, NV, 1, C, tm, 16, tn, 16);
            mma_tile<TK, 1>(ds, sm.kf, 1, LDK, sm.V, NV, 1, C, tm, 16, tn, 16);
#pragma unroll
            for (int i = 0; i < TK; ++i) {
                const int c = tm + 16 * i, e = c * NV + tn;
                sm.S[e] = fmaf(sm.gam[c], sm.S[e], sm.glm[c] * ds[i][0]);
            }
        }
    }
    __syncthreads();
    if (sT)
        for (int e = tid; e < DK * NV; e += NT) {
            const int c = e / NV, j = e % NV;
            sT[(((size_t)n * H + h) * DK + c) * DV + col0 + j] = sm.S[e];
        }
}

template <typename TIn, typename TOut, int DK>
cudaError_t launch(const void* q, const void* k, const void* v, const void* a, const void* b, const float* la,
                   const float* s0, void* o, float* sT, const int32_t* cu, int nseq, int T, long long tokens, int H,
                   int dv, cudaStream_t stream)
{
    const size_t smem = sizeof(Smem<DK>);
    auto kern = dplr_fwd_kernel<TIn, TOut, DK>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const long long blocks = (long long)nseq * H * (dv / NV);
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    kern<<<(unsigned)blocks, NT, smem, stream>>>(
        static_cast<const TIn*>(q), static_cast<const TIn*>(k), static_cast<const TIn*>(v), static_cast<const TIn*>(a),
        static_cast<const TIn*>(b), la, s0, static_cast<TOut*>(o), sT, cu, nseq, T, tokens, H, dv);
    return cudaGetLastError();
}

template <typename TIn, typename TOut>
cudaError_t launch_dk(const void* q, const void* k, const void* v, const void* a, const void* b, const float* la,
                      const float* s0, void* o, float* sT, const int32_t* cu, int nseq, int T, long long tokens,
                      int H, int dk, int dv, cudaStream_t s)
{
    if (dk == 128) return launch<TIn, TOut, 128>(q, k, v, a, b, la, s0, o, sT, cu, nseq, T, tokens, H, dv, s);
    if (dk == 64) return launch<TIn, TOut, 64>(q, k, v, a, b, la, s0, o, sT, cu, nseq, T, tokens, H, dv, s);
    return cudaErrorInvalidValue;
}

}  // namespace dplr

cudaError_t dplr_fwd(const void* q, const void* k, const void* v, const void* a, const void* b, const float* log_alpha,
                     const float* s0, void* o, float* sT, const int32_t* cu, int nseq, int T, long long tokens, int H,
                     int dk, int dv, kda_dtype dtype, kda_dtype o_dtype, cudaStream_t s)
{
    using bf = __nv_bfloat16;
    if (dtype == KDA_BF16 && o_dtype == KDA_BF16)
        return dplr::launch_dk<bf, bf>(q, k, v, a, b, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dk, dv, s);
    if (dtype == KDA_BF16)
        return dplr::launch_dk<bf, float>(q, k, v, a, b, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dk, dv, s);
    if (o_dtype == KDA_BF16)
        return dplr::launch_dk<float, bf>(q, k, v, a, b, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dk, dv, s);
    return dplr::launch_dk<float, float>(q, k, v, a, b, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dk, dv, s);
}

}  // namespace kda
