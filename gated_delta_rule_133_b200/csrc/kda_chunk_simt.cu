// Chunkwise-parallel KDA forward on CUDA cores, fp32 arithmetic throughout.
//
// This is the precise path (fp32 q/k/v, where tensor-core operand rounding
// would exceed a 1e-4 relative budget) and the path for shapes the
// tensor-core kernel does not take.  It follows the chunk recurrence of "Hybrid
// Linear Attention Architecture: Making LLM Training and Inference More
// Efficient", section IV (also "... Technical Deep Dive ...", section 4, and
// "Linear Attention Architecture Deep Dive", section 5):
//
//   per chunk of C = 64 tokens, G = inclusive cumulative sum of log alpha
//   (accumulated in log space, fp32), gamma = exp(G_last);
//   A[r,s] = beta_r sum_c k_rc k_sc exp(G_rc - G_sc)   (s < r)   intra-chunk
//   T      = (I + A)^-1                                  UT transform
//   V'     = T diag(beta) (V - (exp(G) * K) S)          = U - W S  (WY form,
//                                                        applied factored)
//   O      = (exp(G) * Q) S + Tril_incl(P) V',   P[r,s] = sum_c q_rc k_sc exp(G_rc - G_sc)
//   S     <- Diag(gamma) S + (exp(G_last - G) * K)^T V'
//
// The intra-chunk decays exp(G_r - G_s) of P and A are split so that no
// factor overflows ("segmenting intra-chunk cumulative gates"):
//  - when every channel decays at most 80 nats from the chunk's first row to
//    its middle row m and from m to its last row, at m: e^(G_r - G_m) on the
//    row side, e^(G_m - G_s) on the column side, each at most e^80;
//  - otherwise by 16-row blocks (the sub-block references of the chunk
//    algorithm): row block I against the columns s < 16 I at row 16 I,
//    e^(G_r - G_16I) e^(G_16I - G_s), both factors at most 1 and each at least
//    the product, and the diagonal 16 x 16 blocks with e^(G_r - G_s) per
//    element.  These factors use the fast exponential __expf (CUDA documents
//    its error as 2 + floor(1.173 |x|) ulp: below 6e-6 relative for the
//    |x| < 88 whose results are not flushed to zero).
// The state-side operands q e^G, k e^G and k e^(G_last - G) have factors at
// most 1.  So this path has no limit on the gates' strength.
//
// One CTA (256 threads) per (sequence, head, 32-column slice of d_v); the
// columns of S evolve independently because the transition acts on the d_k
// side only.  The CTA walks its chunks in order; everything lives in shared
// memory.
#include "kda_chunk.cuh"

namespace kda {

namespace simt {

constexpr int C = 64;       // chunk length
constexpr int NV = 32;      // value columns per CTA
constexpr int NT = 256;     // threads per CTA
constexpr float kMidRange = 80.f;   // largest decay (nats) the middle-row split takes

// (d0, d1) = (x0 * y0 + d0, x1 * y1 + d1) as one packed fp32x2 FMA; each
// lane rounds exactly as fmaf does.
__device__ __forceinline__ void fma2(float& d0, float& d1, float x0, float x1, float y0, float y1)
{
    asm("{\n\t.reg .b64 xx, yy, dd;\n\t"
        "mov.b64 xx, {%2, %3};\n\tmov.b64 yy, {%4, %5};\n\tmov.b64 dd, {%0, %1};\n\t"
        "fma.rn.f32x2 dd, xx, yy, dd;\n\tmov.b64 {%0, %1}, dd;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(x0), "f"(x1), "f"(y0), "f"(y1));
}

// acc[i][j] += sum_kk A[(m0 + i*MS) * a_m + kk * a_k] * B[kk * b_k + (n0 + j*NS) * b_n]
// The FMAs go in pairs (along j, else along i) as packed fp32x2 FMAs; every
// element is accumulated in the same order and rounding as with fmaf.
template <int TM, int TN>
__device__ __forceinline__ void mma_tile(float (&acc)[TM][TN], const float* A, int a_m, int a_k,
                                         const float* B, int b_k, int b_n, int K, int m0, int MS,
                                         int n0, int NS)
{
#pragma unroll 4
    for (int kk = 0; kk < K; ++kk) {
        float a[TM], b[TN];
#pragma unroll
        for (int i = 0; i < TM; ++i) a[i] = A[(m0 + i * MS) * a_m + kk * a_k];
#pragma unroll
        for (int j = 0; j < TN; ++j) b[j] = B[kk * b_k + (n0 + j * NS) * b_n];
        if constexpr (TN % 2 == 0) {
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < TN; j += 2) fma2(acc[i][j], acc[i][j + 1], a[i], a[i], b[j], b[j + 1]);
        } else if constexpr (TM % 2 == 0) {
#pragma unroll
            for (int i = 0; i < TM; i += 2)
#pragma unroll
                for (int j = 0; j < TN; ++j) fma2(acc[i][j], acc[i + 1][j], a[i], a[i + 1], b[j], b[j]);
        } else {
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
    }
}

// B row kk, columns n0 .. n0 + TN - 1 (contiguous, 8-byte aligned for TN = 2,
// 16-byte aligned for TN = 4 or 8) into b.
template <int TN>
__device__ __forceinline__ void ld_row(float (&b)[TN], const float* p)
{
    static_assert(TN == 2 || TN % 4 == 0, "row segment of 2, 4 or 8 floats");
    if constexpr (TN == 2) {
        const float2 x = *reinterpret_cast<const float2*>(p);
        b[0] = x.x;
        b[1] = x.y;
    } else {
#pragma unroll
        for (int j = 0; j < TN; j += 4) {
            const float4 x = *reinterpret_cast<const float4*>(p + j);
            b[j] = x.x;
            b[j + 1] = x.y;
            b[j + 2] = x.z;
            b[j + 3] = x.w;
        }
    }
}

// acc[i][j] += sum_kk A[(m0 + i) * lda + kk] * B[kk * ldb + n0 + j]: TM
// consecutive rows and TN consecutive columns per thread, A rows read four K
// values at a time.  K, lda and m0's row offsets are multiples of 4 (16-byte
// aligned A rows); B rows as for ld_row.  Each element is accumulated in K
// order with packed fp32x2 FMAs (the rounding of fmaf).
template <int TM, int TN>
__device__ __forceinline__ void mma_rk(float (&acc)[TM][TN], const float* A, int lda, const float* B, int ldb, int K,
                                       int m0, int n0)
{
    static_assert(TN % 2 == 0, "columns in pairs");
#pragma unroll 2
    for (int k0 = 0; k0 < K; k0 += 4) {
        float4 a[TM];
#pragma unroll
        for (int i = 0; i < TM; ++i) a[i] = *reinterpret_cast<const float4*>(A + (m0 + i) * lda + k0);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float b[TN];
            ld_row<TN>(b, B + (k0 + u) * ldb + n0);
#pragma unroll
            for (int i = 0; i < TM; ++i) {
                const float av = u == 0 ? a[i].x : u == 1 ? a[i].y : u == 2 ? a[i].z : a[i].w;
#pragma unroll
                for (int j = 0; j < TN; j += 2) fma2(acc[i][j], acc[i][j + 1], av, av, b[j], b[j + 1]);
            }
        }
    }
}

// acc[i][j] += sum_kk A[kk * lda + m0 + i] * B[kk * ldb + n0 + j]: the same
// with A stored transposed (K rows of M), read TM values at a time (TM = 2, 4
// or 8; A's row segments aligned as for ld_row).
template <int TM, int TN>
__device__ __forceinline__ void mma_tk(float (&acc)[TM][TN], const float* A, int lda, const float* B, int ldb, int K,
                                       int m0, int n0)
{
    static_assert(TN % 2 == 0 && (TM == 2 || TM % 4 == 0), "columns in pairs, rows in pairs or fours");
#pragma unroll 4
    for (int kk = 0; kk < K; ++kk) {
        float a[TM], b[TN];
        ld_row<TM>(a, A + kk * lda + m0);
        ld_row<TN>(b, B + kk * ldb + n0);
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; j += 2) fma2(acc[i][j], acc[i][j + 1], a[i], a[i], b[j], b[j + 1]);
    }
}

template <int DK>
struct Smem {
    static constexpr int LDK = DK + 1;   // padded row pitch of the [C][DK] tiles
    static constexpr int LDC = C + 1;    // padded pitch of the [C][C] tiles
    static constexpr int LDX = DK + 4;   // pitch of the 16-row blocks' operands (16-byte rows)
    static constexpr int XROWS = 56;     // 32 row-block operand rows + up to 24 column rows
    float qm[C * LDK];    // q * E (segmented chunks: q e^G)
    float km[C * LDK];    // k * E (segmented chunks: k e^G)
    float kf[C * LDK];    // cumulative gate G, then k * F (segmented chunks: k e^(G_last - G))
    float A[C * LDC];
    float P[C * LDC];
    float T[C * LDC];     // T, and with Sm the operands of the 16-row blocks (free until the UT transform)
    float Sm[DK * NV];    // exp(G_m) * S for the current chunk
    float S[DK * NV];     // state slice, fp32, carried across chunks
    float V[C * NV];      // values, then Y = beta (V - X)
    float Vp[C * NV];     // V' = T Y
    float gm[DK];         // exp(G_m) (segmented chunks: 1)
    float gam[DK];        // exp(G_last)
    float glm[DK];        // exp(G_last - G_m) (segmented chunks: 1)
    float gl[DK];         // G_last
    float beta[C];
};

// P, A of a chunk outside the middle-row split's range, by 16-row blocks, on
// the raw q, k and the cumulative gates G in qm, km, kf; then the state-side
// operands q e^G, k e^G and k e^(G_last - G) in their place, gm = glm = 1 and
// Sm = S.  Row block I against the columns s < r0 = 16 I: the decay split at
// row r0, the block operands in T and Sm (X rows 0..15 = q e^(G - G_r0), 16..31
// = k e^(G - G_r0) of rows r0 .. r0 + 15; 32.. = k e^(G_r0 - G) of up to 24
// columns at a time).  Diagonal 16 x 16 blocks with e^(G_r - G_s) per element.
static_assert(offsetof(Smem<128>, Sm) == offsetof(Smem<128>, T) + sizeof(float) * C * Smem<128>::LDC &&
              Smem<128>::XROWS * Smem<128>::LDX <= C * Smem<128>::LDC + 128 * NV &&
              Smem<64>::XROWS * Smem<64>::LDX <= C * Smem<64>::LDC + 64 * NV,
              "the 16-row blocks' operands fit in T and Sm");

template <int DK>
__device__ __forceinline__ void segmented_pa(Smem<DK>& sm, int tid, bool erase)
{
    constexpr int LDK = Smem<DK>::LDK, LDC = Smem<DK>::LDC, LDX = Smem<DK>::LDX;
    float* X = sm.T;
    for (int e = tid; e < C * C; e += NT) {
        sm.P[(e / C) * LDC + e % C] = 0.f;
        sm.A[(e / C) * LDC + e % C] = 0.f;
    }
    for (int I = 1; I < C / 16; ++I) {
        const int r0 = 16 * I;
        for (int e = tid; e < 32 * DK; e += NT) {
            const int row = e / DK, c = e % DK, r = r0 + (row & 15);
            const float f = __expf(sm.kf[r * LDK + c] - sm.kf[r0 * LDK + c]);
            X[row * LDX + c] = (row < 16 ? sm.qm[r * LDK + c] : sm.km[r * LDK + c]) * f;
        }
        for (int s0 = 0; s0 < r0; s0 += 24) {
            const int ns = min(24, r0 - s0);
            for (int e = tid; e < ns * DK; e += NT) {
                const int sr = s0 + e / DK, c = e % DK;
                X[(32 + e / DK) * LDX + c] = sm.km[sr * LDK + c] * __expf(sm.kf[r0 * LDK + c] - sm.kf[sr * LDK + c]);
            }
            __syncthreads();
            for (int ix = tid; ix < 16 * ns; ix += NT) {
                const int r = ix / ns, j = ix % ns;
                const float4* xq = reinterpret_cast<const float4*>(X + r * LDX);
                const float4* xk = reinterpret_cast<const float4*>(X + (16 + r) * LDX);
                const float4* xc = reinterpret_cast<const float4*>(X + (32 + j) * LDX);
                float p = 0.f, a = 0.f;
#pragma unroll 4
                for (int c4 = 0; c4 < DK / 4; ++c4) {
                    const float4 u = xq[c4], w = xk[c4], z = xc[c4];
                    p = fmaf(u.x, z.x, p); p = fmaf(u.y, z.y, p); p = fmaf(u.z, z.z, p); p = fmaf(u.w, z.w, p);
                    a = fmaf(w.x, z.x, a); a = fmaf(w.y, z.y, a); a = fmaf(w.z, z.z, a); a = fmaf(w.w, z.w, a);
                }
                sm.P[(r0 + r) * LDC + s0 + j] = p;
                sm.A[(r0 + r) * LDC + s0 + j] = erase ? sm.beta[r0 + r] * a : 0.f;
            }
            __syncthreads();
        }
    }
    for (int ix = tid; ix < (C / 16) * 136; ix += NT) {
        int t = ix % 136, r = 0;
        while (t > r) {   // (r, t): t-th entry of the lower-inclusive 16 x 16 triangle, row-major
            t -= r + 1;
            ++r;
        }
        const int R = 16 * (ix / 136) + r, Sc = R - r + t;
        float p = 0.f, a = 0.f;
        for (int c = 0; c < DK; ++c) {
            const float kd = sm.km[Sc * LDK + c] * __expf(sm.kf[R * LDK + c] - sm.kf[Sc * LDK + c]);
            p = fmaf(sm.qm[R * LDK + c], kd, p);
            a = fmaf(sm.km[R * LDK + c], kd, a);
        }
        sm.P[R * LDC + Sc] = p;
        sm.A[R * LDC + Sc] = (erase && t < r) ? sm.beta[R] * a : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < C * DK; e += NT) {
        const int r = e / DK, c = e % DK;
        const float g = sm.kf[r * LDK + c], kv = sm.km[r * LDK + c], eg = __expf(g);
        sm.qm[r * LDK + c] *= eg;
        sm.km[r * LDK + c] = kv * eg;
        sm.kf[r * LDK + c] = kv * __expf(sm.gl[c] - g);
    }
    for (int e = tid; e < DK * NV; e += NT) sm.Sm[e] = sm.S[e];
    if (tid < DK) {
        sm.gm[tid] = 1.f;
        sm.glm[tid] = 1.f;
    }
    __syncthreads();
}

// The chunk loop of one CTA from token t_begin of its sequence.  SEG = false:
// every chunk takes the middle-row split, and the loop returns the offset of
// the first chunk that the split cannot take (len if none) with that chunk's
// state untouched; SEG = true: chunks outside its range are segmented by
// 16-row blocks.  Two functions, so that the common loop is compiled alone.
template <bool SEG, typename TIn, typename TOut, int DK>
__device__ __noinline__ int chunk_loop(Smem<DK>& sm, const TIn* __restrict__ q, const TIn* __restrict__ k,
                                       const TIn* __restrict__ v, const float* __restrict__ beta,
                                       const float* __restrict__ log_alpha, TOut* __restrict__ o, int tok0,
                                       int len, int t_begin, int H, int h, int DV, int col0, int mode)
{
    const bool head_gate = (mode & KDA_MODE_HEAD_GATE) != 0;   // log_alpha [tokens, H]
    const bool erase = (mode & KDA_MODE_NO_ERASE) == 0;
    const bool logits = (mode & KDA_MODE_GATE_LOGITS) != 0;
    const bool norm_qk = (mode & KDA_MODE_NORM_QK) != 0;
    constexpr int LDK = Smem<DK>::LDK, LDC = Smem<DK>::LDC;
    const int tid = threadIdx.x;
    for (int t0 = t_begin; t0 < len; t0 += C) {
        const int L = min(C, len - t0);
        __syncthreads();
        // ---- load the chunk (rows >= L are zero: no key, no value, no decay)
        for (int e = tid; e < C * DK; e += NT) {
            const int r = e / DK, c = e % DK;
            float qv = 0.f, kv = 0.f, gv = 0.f;
            if (r < L) {
                const size_t off = ((size_t)(tok0 + t0 + r) * H + h) * DK + c;
                qv = Elem<TIn>::load(q + off);
                kv = Elem<TIn>::load(k + off);
                gv = head_gate ? log_alpha[(size_t)(tok0 + t0 + r) * H + h] : log_alpha[off];
                if (logits) gv = neg_softplus(gv);
            }
            sm.qm[r * LDK + c] = qv;
            sm.km[r * LDK + c] = kv;
            sm.kf[r * LDK + c] = gv;
        }
        for (int e = tid; e < C * NV; e += NT) {
            const int r = e / NV, j = e % NV;
            sm.V[e] = r < L ? Elem<TIn>::load(v + ((size_t)(tok0 + t0 + r) * H + h) * DV + col0 + j) : 0.f;
        }
        if (tid < C) sm.beta[tid] = tid < L ? beta[(size_t)(tok0 + t0 + tid) * H + h] : 0.f;
        __syncthreads();
        if (norm_qk) {   // raw q, k: each row divided by its L2 norm, one warp per row
            const int lane = tid & 31;
            for (int rw = tid >> 5; rw < 2 * C; rw += NT / 32) {
                float* row = (rw < C ? sm.qm : sm.km) + (rw % C) * LDK;
                float ss = 0.f;
                for (int c = lane; c < DK; c += 32) ss = fmaf(row[c], row[c], ss);
                const float inv = inv_norm(warp_sum(ss));
                for (int c = lane; c < DK; c += 32) row[c] *= inv;
            }
            __syncthreads();
        }

        // ---- gate cumsum per channel (fp32, log space); does the chunk fit the middle-row split?
        bool seg = false;
        if (tid < DK) {
            const int c = tid;
            float acc = 0.f;
            for (int r = 0; r < C; ++r) { acc += sm.kf[r * LDK + c]; sm.kf[r * LDK + c] = acc; }
            const float Gm = sm.kf[(C / 2 - 1) * LDK + c];
            const float Gl = acc;
            sm.gm[c] = expf(Gm);
            sm.gam[c] = expf(Gl);
            sm.glm[c] = expf(Gl - Gm);
            sm.gl[c] = Gl;
            seg = sm.kf[c] - Gm > kMidRange || Gm - Gl > kMidRange;
        }
        seg = __syncthreads_or(seg);

        if (SEG && seg) {
            segmented_pa<DK>(sm, tid, erase);
        } else {
            if (seg) return t0;   // first chunk the middle-row split cannot take
            // ---- the factor split at the middle row m: E = e^(G - G_m), F = e^(G_m - G)
            if (tid < DK) {
                const int c = tid;
                const float Gm = sm.kf[(C / 2 - 1) * LDK + c];
                for (int r = 0; r < C; ++r) {
                    const float G = sm.kf[r * LDK + c];
                    const float Er = expf(fminf(G - Gm, 80.f));
                    const float Fr = expf(fminf(Gm - G, 80.f));
                    sm.qm[r * LDK + c] *= Er;
                    const float kk = sm.km[r * LDK + c];
                    sm.km[r * LDK + c] = kk * Er;
                    sm.kf[r * LDK + c] = kk * Fr;
                }
            }
            __syncthreads();

            // ---- P = (q E)(k F)^T (lower incl.), A = beta (k E)(k F)^T (strictly lower)
            {
                const int tn = tid % 16, tm = tid / 16;
                float p[4][4] = {}, a[4][4] = {};
                mma_tile<4, 4>(p, sm.qm, LDK, 1, sm.kf, 1, LDK, DK, tm, 16, tn, 16);
                mma_tile<4, 4>(a, sm.km, LDK, 1, sm.kf, 1, LDK, DK, tm, 16, tn, 16);
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int r = tm + 16 * i, s = tn + 16 * j;
                        sm.P[r * LDC + s] = s <= r ? p[i][j] : 0.f;
                        sm.A[r * LDC + s] = (erase && s < r) ? sm.beta[r] * a[i][j] : 0.f;
                    }
                // Sm = exp(G_m) * S  (state rows scaled per key channel)
                for (int e = tid; e < DK * NV; e += NT) sm.Sm[e] = sm.gm[e / NV] * sm.S[e];
            }
            __syncthreads();
        }

        // ---- UT transform T = (I + A)^-1 by forward substitution: column j of T
        // depends only on column j of earlier rows; 4 lanes share one column.
        {
            const int j = tid >> 2, p = tid & 3;
            for (int r = 0; r < C; ++r) {
                float acc = 0.f;
                if (r > j)
                    for (int s = j + p; s < r; s += 4) acc = fmaf(sm.A[r * LDC + s], sm.T[s * LDC + j], acc);
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                if (p == 0) sm.T[r * LDC + j] = (r == j ? 1.f : 0.f) - (r > j ? acc : 0.f);
                __syncwarp();
            }
        }
        // ---- X = (k E) Sm ; Y = beta (V - X)   (into sm.V)
        {
            const int tn = tid % 16, tm = tid / 16;
            float x[4][2] = {};
            mma_tile<4, 2>(x, sm.km, LDK, 1, sm.Sm, NV, 1, DK, tm, 16, tn, 16);
            __syncthreads();
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int r = tm + 16 * i, cc = tn + 16 * j;
                    sm.V[r * NV + cc] = sm.beta[r] * (sm.V[r * NV + cc] - (erase ? x[i][j] : 0.f));
                }
        }
        __syncthreads();
        // ---- V' = T Y
        {
            const int tn = tid % 16, tm = tid / 16;
            float y[4][2] = {};
            mma_tile<4, 2>(y, sm.T, LDC, 1, sm.V, NV, 1, C, tm, 16, tn, 16);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j) sm.Vp[(tm + 16 * i) * NV + tn + 16 * j] = y[i][j];
        }
        __syncthreads();
        // ---- O = (q E) Sm + P V'  -> output rows < L
        {
            const int tn = tid % 16, tm = tid / 16;
            float ov[4][2] = {};
            mma_tile<4, 2>(ov, sm.qm, LDK, 1, sm.Sm, NV, 1, DK, tm, 16, tn, 16);
            mma_tile<4, 2>(ov, sm.P, LDC, 1, sm.Vp, NV, 1, C, tm, 16, tn, 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = tm + 16 * i;
                if (r < L)
#pragma unroll
                    for (int j = 0; j < 2; ++j)
                        Elem<TOut>::store(o + ((size_t)(tok0 + t0 + r) * H + h) * DV + col0 + tn + 16 * j,
                                         ov[i][j]);
            }
        }
        // ---- S <- gamma S + exp(G_last - G_m) (k F)^T V'
        {
            constexpr int TM = DK / 16;
            const int tn = tid % 16, tm = tid / 16;
            float ds[TM][2] = {};
            mma_tile<TM, 2>(ds, sm.kf, 1, LDK, sm.Vp, NV, 1, C, tm, 16, tn, 16);
#pragma unroll
            for (int i = 0; i < TM; ++i) {
                const int c = tm + 16 * i;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int e = c * NV + tn + 16 * j;
                    sm.S[e] = fmaf(sm.gam[c], sm.S[e], sm.glm[c] * ds[i][j]);
                }
            }
        }
    }
    return len;
}

template <typename TIn, typename TOut, int DK>
__global__ void __launch_bounds__(NT)
chunk_fwd_simt_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                      const TIn* __restrict__ v, const float* __restrict__ beta,
                      const float* __restrict__ log_alpha, const float* s0, TOut* __restrict__ o,
                      float* sT, const int32_t* __restrict__ cu, int nseq, int T, long long tokens, int H, int DV,
                      int mode)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem<DK>& sm = *reinterpret_cast<Smem<DK>*>(smem_raw);

    const int nslice = DV / NV;
    const int slice = blockIdx.x % nslice;
    const int h = (blockIdx.x / nslice) % H;
    const int rank = blockIdx.x / (nslice * H);
    int n, tok0, len;
    if (cu) {   // packed sequences in their own order; a range outside the token axis is skipped
        n = rank;
        tok0 = cu[n];
        len = max(0, cu[n + 1] - tok0);
        if (tok0 < 0 || (long long)tok0 + len > tokens) {   // no tokens read; final state = initial
            if (threadIdx.x == 0) flag_bad_input();
            tok0 = 0;
            len = 0;
        }
    } else {
        n = rank;
        tok0 = n * T;
        len = T;
    }
    const int col0 = slice * NV;
    const int tid = threadIdx.x;

    // initial state slice
    for (int e = tid; e < DK * NV; e += NT) {
        const int c = e / NV, j = e % NV;
        sm.S[e] = s0 ? s0[(((size_t)n * H + h) * DK + c) * DV + col0 + j] : 0.f;
    }

    const int t_seg = chunk_loop<false>(sm, q, k, v, beta, log_alpha, o, tok0, len, 0, H, h, DV, col0, mode);
    if (t_seg < len) chunk_loop<true>(sm, q, k, v, beta, log_alpha, o, tok0, len, t_seg, H, h, DV, col0, mode);
    __syncthreads();
    if (sT)
        for (int e = tid; e < DK * NV; e += NT) {
            const int c = e / NV, j = e % NV;
            sT[(((size_t)n * H + h) * DK + c) * DV + col0 + j] = sm.S[e];
        }
}

template <typename TIn, typename TOut, int DK>
cudaError_t launch(const void* q, const void* k, const void* v, const float* beta,
                   const float* log_alpha, const float* s0, void* o, float* sT, const int32_t* cu,
                   int nseq, int T, long long tokens, int H, int dv, int mode, cudaStream_t stream)
{
    const size_t smem = sizeof(Smem<DK>);
    auto kern = chunk_fwd_simt_kernel<TIn, TOut, DK>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const long long blocks = (long long)nseq * H * (dv / NV);
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    kern<<<(unsigned)blocks, NT, smem, stream>>>(
        static_cast<const TIn*>(q), static_cast<const TIn*>(k), static_cast<const TIn*>(v), beta,
        log_alpha, s0, static_cast<TOut*>(o), sT, cu, nseq, T, tokens, H, dv, mode);
    return cudaGetLastError();
}

template <typename TIn, typename TOut>
cudaError_t launch_dk(const void* q, const void* k, const void* v, const float* beta,
                      const float* log_alpha, const float* s0, void* o, float* sT,
                      const int32_t* cu, int nseq, int T, long long tokens, int H, int dk, int dv, int mode,
                      cudaStream_t s)
{
    if (dk == 128) return launch<TIn, TOut, 128>(q, k, v, beta, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dv, mode, s);
    if (dk == 64) return launch<TIn, TOut, 64>(q, k, v, beta, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dv, mode, s);
    return cudaErrorInvalidValue;
}

}  // namespace simt

cudaError_t chunk_fwd_simt(const void* q, const void* k, const void* v, const float* beta,
                           const float* log_alpha, const float* s0, void* o, float* sT,
                           const int32_t* cu, int nseq, int T, long long tokens, int H, int dk, int dv,
                           kda_dtype dtype, kda_dtype o_dtype, int mode, cudaStream_t s)
{
    using bf = __nv_bfloat16;
    if (dtype == KDA_BF16 && o_dtype == KDA_BF16)
        return simt::launch_dk<bf, bf>(q, k, v, beta, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dk, dv, mode, s);
    if (dtype == KDA_BF16 && o_dtype == KDA_F32)
        return simt::launch_dk<bf, float>(q, k, v, beta, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dk, dv, mode, s);
    if (dtype == KDA_F32 && o_dtype == KDA_BF16)
        return simt::launch_dk<float, bf>(q, k, v, beta, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dk, dv, mode, s);
    return simt::launch_dk<float, float>(q, k, v, beta, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dk, dv, mode, s);
}

}  // namespace kda
