// Chunkwise KDA backward on CUDA cores (fp32 arithmetic): gradients of
// L = sum(o * do) + sum(S_T * dS_T) with respect to q, k, v, beta, log alpha
// and the initial state.
//
// "Hybrid Linear Attention Architecture: Making LLM Training and Inference More
// Efficient", section IV, notes that backpropagation reuses the chunked
// structure of the forward pass.  This is the adjoint of the chunk recurrence
// of the CUDA-core forward (kda_chunk_simt.cu), with the same factors around
// the chunk's middle row m (E = exp(G - G_m), F = 1 / E, Q~ = q E, K~ = k E,
// K~n = k F, MA = K~ K~n^T, P = lower-incl(Q~ K~n^T), A = beta strictly-lower(MA),
// T = (I + A)^-1, Qh = e^G_m Q~, Kh = e^G_m K~, Kl = e^(G_last - G_m) K~n):
//
//   forward of one chunk:  X = Kh S, Y = beta (V - X), U = T Y,
//                          O = Qh S + P U,  S' = diag(gamma) S + Kl^T U
//   backward, given dO and dS' (the gradient reaching the state after it):
//     dU = P^T dO + Kl dS',  dY = T^T dU,  dV = beta dY,  dX = -beta dY
//     dP = lower-incl(dO U^T),  dT = dU Y^T,  dA = -strictly-lower(T^T dT T^T)
//     dbeta = rowsum((V - X) dY) + rowsum(MA dA),  dMA = beta dA
//     dS = diag(gamma) dS' + Qh^T dO + Kh^T dX
//   and through the factors, per element (r, c):
//     a_q = e^G_m dO S^T + dP K~n                        (dq = E a_q)
//     a_k = e^G_m dX S^T + dMA K~n                       (dk = E a_k + F a_n)
//     a_n = e^(G_last - G_m) U dS'^T + dP^T Q~ + dMA^T K~
//     dG  = Q~ a_q + K~ a_k - K~n a_n,  plus, on the last row, rowsum(dS' S')
//   (the derivative with respect to the reference G_m cancels: the products
//   depend on differences of G only), and dlog alpha is the reverse
//   cumulative sum of dG inside the chunk.
//
// One CTA (256 threads) per (sequence, head, 16 value columns).  A forward
// walk over the chunks stores the state entering every chunk in the
// workspace; a reverse walk then carries dS.  Gradients that sum over value
// columns (dq, dk, dbeta, dlog alpha) are added with atomics into outputs the
// launcher has zeroed; dv and the initial state's gradient belong to one
// slice each.
#include "kda_chunk.cuh"

namespace kda {

namespace bwd {

using simt::mma_tile;

constexpr int C = 64;       // chunk length
constexpr int NV = 16;      // value columns per CTA
constexpr int NT = 256;     // threads per CTA

template <int DK>
struct Smem {
    static constexpr int LDK = DK + 1;   // padded row pitch of the [C][DK] tiles
    static constexpr int LDC = C + 1;    // padded pitch of the [C][C] tiles
    float qm[C * LDK];    // q E, then dG
    float km[C * LDK];    // k E
    float kf[C * LDK];    // cumulative gate G, then k F
    float MA[C * LDC];    // strictly-lower (k E)(k F)^T
    float P[C * LDC];     // lower-incl (q E)(k F)^T, then T^T dT
    float T[C * LDC];     // (I + A)^-1
    float D[C * LDC];     // A, then dP, dT, dA, dMA
    float S[DK * NV];     // state entering the chunk (slice)
    float Sm[DK * NV];    // e^G_m S, then the state gradient entering the chunk
    float dS[DK * NV];    // gradient reaching the state after the chunk
    float dSg[DK * NV];   // e^(G_last - G_m) dS
    float V[C * NV];      // V, then V - X
    float Y[C * NV];      // beta (V - X)
    float U[C * NV];      // T Y
    float dO[C * NV];
    float dU[C * NV];
    float dY[C * NV];     // T^T dU, then dX = -beta dY
    float gm[DK];         // e^G_m
    float gam[DK];        // e^G_last
    float glm[DK];        // e^(G_last - G_m)
    float dgl[DK];        // rowsum(dS' S'): the last row's extra dG
    float beta[C];
};

struct Params {
    const float* beta;
    const float* log_alpha;
    const float* s0;         // [nseq, H, DK, DV] or nullptr
    const float* dout;       // [tokens, H, DV]
    const float* dsT;        // [nseq, H, DK, DV] or nullptr
    float* dq;               // [tokens, H, DK], zeroed
    float* dk;
    float* dv;               // [tokens, H, DV]
    float* dbeta;            // [tokens, H], zeroed
    float* dla;              // [tokens, H, DK], zeroed
    float* ds0;              // [nseq, H, DK, DV] or nullptr
    float* states;           // workspace: state entering every chunk, and the final one
    float* escr;             // workspace: E of the current chunk, per CTA [C][DK]
    const int32_t* cu;
    const int32_t* choff;    // varlen: first chunk of each sequence
    long long tokens;
    int nseq, T, H, DV;
};

// Loads chunk [t0, t0 + L) of one (sequence, head) and forms the gate
// factors, the intra-chunk products and T = (I + A)^-1 (all threads).
template <typename TIn, int DK>
__device__ void prepare(Smem<DK>& sm, const TIn* q, const TIn* k, const TIn* v, const Params& p, int tok,
                        int L, int h, int col0, float* escr)
{
    constexpr int LDK = Smem<DK>::LDK, LDC = Smem<DK>::LDC;
    const int tid = threadIdx.x, H = p.H;
    for (int e = tid; e < C * DK; e += NT) {
        const int r = e / DK, c = e % DK;
        float qv = 0.f, kv = 0.f, gv = 0.f;
        if (r < L) {
            const size_t off = ((size_t)(tok + r) * H + h) * DK + c;
            qv = Elem<TIn>::load(q + off);
            kv = Elem<TIn>::load(k + off);
            gv = p.log_alpha[off];
        }
        sm.qm[r * LDK + c] = qv;
        sm.km[r * LDK + c] = kv;
        sm.kf[r * LDK + c] = gv;
    }
    for (int e = tid; e < C * NV; e += NT) {
        const int r = e / NV, j = e % NV;
        sm.V[e] = r < L ? Elem<TIn>::load(v + ((size_t)(tok + r) * H + h) * p.DV + col0 + j) : 0.f;
    }
    if (tid < C) sm.beta[tid] = tid < L ? p.beta[(size_t)(tok + tid) * H + h] : 0.f;
    __syncthreads();
    if (tid < DK) {   // gate cumsum per channel (fp32, log space) and the factor split
        const int c = tid;
        float acc = 0.f;
        for (int r = 0; r < C; ++r) { acc += sm.kf[r * LDK + c]; sm.kf[r * LDK + c] = acc; }
        const float Gm = sm.kf[(C / 2 - 1) * LDK + c];
        sm.gm[c] = expf(Gm);
        sm.gam[c] = expf(acc);
        sm.glm[c] = expf(acc - Gm);
        for (int r = 0; r < C; ++r) {
            const float x = fminf(fmaxf(sm.kf[r * LDK + c] - Gm, -80.f), 80.f);
            const float E = expf(x), F = expf(-x);
            if (escr) escr[r * DK + c] = E;
            sm.qm[r * LDK + c] *= E;
            const float kk = sm.km[r * LDK + c];
            sm.km[r * LDK + c] = kk * E;
            sm.kf[r * LDK + c] = kk * F;
        }
    }
    __syncthreads();
    {   // MA (strictly lower), P (lower incl.), A = beta MA -> D
        const int tn = tid % 16, tm = tid / 16;
        float pp[4][4] = {}, a[4][4] = {};
        mma_tile<4, 4>(pp, sm.qm, LDK, 1, sm.kf, 1, LDK, DK, tm, 16, tn, 16);
        mma_tile<4, 4>(a, sm.km, LDK, 1, sm.kf, 1, LDK, DK, tm, 16, tn, 16);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = tm + 16 * i, s = tn + 16 * j;
                sm.P[r * LDC + s] = s <= r ? pp[i][j] : 0.f;
                sm.MA[r * LDC + s] = s < r ? a[i][j] : 0.f;
                sm.D[r * LDC + s] = s < r ? sm.beta[r] * a[i][j] : 0.f;
            }
    }
    __syncthreads();
    {   // T = (I + A)^-1 by forward substitution; 4 lanes share one column
        const int j = tid >> 2, pq = tid & 3;
        for (int r = 0; r < C; ++r) {
            float acc = 0.f;
            if (r > j)
                for (int s = j + pq; s < r; s += 4) acc = fmaf(sm.D[r * LDC + s], sm.T[s * LDC + j], acc);
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            if (pq == 0) sm.T[r * LDC + j] = (r == j ? 1.f : 0.f) - (r > j ? acc : 0.f);
            __syncwarp();
        }
    }
    __syncthreads();
}

// X = (k E)(e^G_m S), V <- V - X, Y = beta (V - X), U = T Y   (Sm must hold e^G_m S)
template <int DK>
__device__ void chunk_uy(Smem<DK>& sm)
{
    constexpr int LDK = Smem<DK>::LDK, LDC = Smem<DK>::LDC;
    const int tid = threadIdx.x, tn = tid % 16, tm = tid / 16;
    float x[4][1] = {};
    mma_tile<4, 1>(x, sm.km, LDK, 1, sm.Sm, NV, 1, DK, tm, 16, tn, 16);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = tm + 16 * i;
        const float d = sm.V[r * NV + tn] - x[i][0];
        sm.V[r * NV + tn] = d;
        sm.Y[r * NV + tn] = sm.beta[r] * d;
    }
    __syncthreads();
    float u[4][1] = {};
    mma_tile<4, 1>(u, sm.T, LDC, 1, sm.Y, NV, 1, C, tm, 16, tn, 16);
#pragma unroll
    for (int i = 0; i < 4; ++i) sm.U[(tm + 16 * i) * NV + tn] = u[i][0];
    __syncthreads();
}

// Sum over the 16 threads (consecutive lanes) that share tm.
__device__ __forceinline__ float sum16(float x)
{
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

template <typename TIn, int DK>
__global__ void __launch_bounds__(NT, 1)
chunk_bwd_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v, const Params p)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem<DK>& sm = *reinterpret_cast<Smem<DK>*>(smem_raw);
    constexpr int LDK = Smem<DK>::LDK, LDC = Smem<DK>::LDC;
    constexpr int TK = DK / 16;
    const int DV = p.DV, H = p.H;
    const int nslice = DV / NV;
    const int slice = blockIdx.x % nslice;
    const int h = (blockIdx.x / nslice) % H;
    const int n = blockIdx.x / (nslice * H);
    const int col0 = slice * NV;
    const int tid = threadIdx.x, tn = tid % 16, tm = tid / 16;
    float* escr = p.escr + (size_t)blockIdx.x * C * DK;

    int tok0, len;
    long long sbase;   // state slot of the sequence's first chunk
    if (p.cu) {
        tok0 = p.cu[n];
        len = max(0, p.cu[n + 1] - tok0);
        sbase = (long long)p.choff[n] + n;
        if (tok0 < 0 || (long long)tok0 + len > p.tokens) {   // no tokens read; the state passes through
            if (tid == 0) flag_bad_input();
            tok0 = 0;
            len = 0;
        }
    } else {
        tok0 = n * p.T;
        len = p.T;
        sbase = (long long)n * ((p.T + C - 1) / C + 1);
    }
    const int nch = (len + C - 1) / C;
    auto state_at = [&](int c) { return p.states + ((sbase + c) * H + h) * (size_t)DK * DV + col0; };

    // ---- forward walk: the state entering every chunk (and after the last)
    for (int e = tid; e < DK * NV; e += NT) {
        const int c = e / NV, j = e % NV;
        sm.S[e] = p.s0 ? p.s0[(((size_t)n * H + h) * DK + c) * DV + col0 + j] : 0.f;
    }
    __syncthreads();
    for (int ci = 0; ci < nch; ++ci) {
        const int L = min(C, len - ci * C);
        float* st = state_at(ci);
        for (int e = tid; e < DK * NV; e += NT) st[(e / NV) * DV + e % NV] = sm.S[e];
        prepare<TIn, DK>(sm, q, k, v, p, tok0 + ci * C, L, h, col0, nullptr);
        for (int e = tid; e < DK * NV; e += NT) sm.Sm[e] = sm.gm[e / NV] * sm.S[e];
        __syncthreads();
        chunk_uy<DK>(sm);
        {   // S <- gamma S + e^(G_last - G_m) (k F)^T U
            float ds[TK][1] = {};
            mma_tile<TK, 1>(ds, sm.kf, 1, LDK, sm.U, NV, 1, C, tm, 16, tn, 16);
#pragma unroll
            for (int i = 0; i < TK; ++i) {
                const int c = tm + 16 * i, e = c * NV + tn;
                sm.S[e] = fmaf(sm.gam[c], sm.S[e], sm.glm[c] * ds[i][0]);
            }
        }
        __syncthreads();
    }
    {
        float* st = state_at(nch);
        for (int e = tid; e < DK * NV; e += NT) st[(e / NV) * DV + e % NV] = sm.S[e];
    }

    // ---- reverse walk carrying dS
    for (int e = tid; e < DK * NV; e += NT) {
        const int c = e / NV, j = e % NV;
        sm.dS[e] = p.dsT ? p.dsT[(((size_t)n * H + h) * DK + c) * DV + col0 + j] : 0.f;
    }
    __threadfence_block();
    __syncthreads();
    for (int ci = nch - 1; ci >= 0; --ci) {
        const int L = min(C, len - ci * C), tok = tok0 + ci * C;
        prepare<TIn, DK>(sm, q, k, v, p, tok, L, h, col0, escr);
        {
            const float* st = state_at(ci);
            const float* st1 = state_at(ci + 1);
            for (int e = tid; e < DK * NV; e += NT) {
                const int c = e / NV, j = e % NV;
                const float s = st[c * DV + j];
                sm.S[e] = s;
                sm.Sm[e] = sm.gm[c] * s;
                sm.dSg[e] = sm.glm[c] * sm.dS[e];
            }
            for (int e = tid; e < C * NV; e += NT) {
                const int r = e / NV, j = e % NV;
                sm.dO[e] = r < L ? p.dout[((size_t)(tok + r) * H + h) * DV + col0 + j] : 0.f;
            }
            if (tid < DK) {   // rowsum(dS' S'), S' = the state after this chunk
                float a = 0.f;
                for (int j = 0; j < NV; ++j) a = fmaf(sm.dS[tid * NV + j], st1[tid * DV + j], a);
                sm.dgl[tid] = a;
            }
        }
        __syncthreads();
        chunk_uy<DK>(sm);

        float aq[4][TK] = {}, ak[4][TK] = {}, an[4][TK] = {};
        // a_q = e^G_m dO S^T, a_n = e^(G_last - G_m) U dS'^T
        mma_tile<4, TK>(aq, sm.dO, NV, 1, sm.Sm, 1, NV, NV, tm, 16, tn, 16);
        mma_tile<4, TK>(an, sm.U, NV, 1, sm.dSg, 1, NV, NV, tm, 16, tn, 16);
        {   // dU = P^T dO + Kl dS'
            float du[4][1] = {};
            mma_tile<4, 1>(du, sm.P, 1, LDC, sm.dO, NV, 1, C, tm, 16, tn, 16);
            mma_tile<4, 1>(du, sm.kf, LDK, 1, sm.dSg, NV, 1, DK, tm, 16, tn, 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) sm.dU[(tm + 16 * i) * NV + tn] = du[i][0];
        }
        __syncthreads();
        float db[4];
        {   // dY = T^T dU; dv = beta dY; dbeta = rowsum((V - X) dY)
            float dy[4][1] = {};
            mma_tile<4, 1>(dy, sm.T, 1, LDC, sm.dU, NV, 1, C, tm, 16, tn, 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = tm + 16 * i;
                sm.dY[r * NV + tn] = dy[i][0];
                if (r < L) p.dv[((size_t)(tok + r) * H + h) * DV + col0 + tn] = sm.beta[r] * dy[i][0];
                db[i] = sum16(sm.V[r * NV + tn] * dy[i][0]);
            }
        }
        {   // dP = lower-incl(dO U^T) -> D
            float dp[4][4] = {};
            mma_tile<4, 4>(dp, sm.dO, NV, 1, sm.U, 1, NV, NV, tm, 16, tn, 16);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int r = tm + 16 * i, s = tn + 16 * j;
                    sm.D[r * LDC + s] = s <= r ? dp[i][j] : 0.f;
                }
        }
        __syncthreads();
        // a_k = e^G_m dX S^T (dX = -beta dY); a_q += dP K~n; a_n += dP^T Q~
        {
            float t[4][TK] = {};
            mma_tile<4, TK>(t, sm.dY, NV, 1, sm.Sm, 1, NV, NV, tm, 16, tn, 16);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < TK; ++j) ak[i][j] = -sm.beta[tm + 16 * i] * t[i][j];
        }
        mma_tile<4, TK>(aq, sm.D, LDC, 1, sm.kf, LDK, 1, C, tm, 16, tn, 16);
        mma_tile<4, TK>(an, sm.D, 1, LDC, sm.qm, LDK, 1, C, tm, 16, tn, 16);
        __syncthreads();
        {   // dT = dU Y^T -> D
            float dt[4][4] = {};
            mma_tile<4, 4>(dt, sm.dU, NV, 1, sm.Y, 1, NV, NV, tm, 16, tn, 16);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) sm.D[(tm + 16 * i) * LDC + tn + 16 * j] = dt[i][j];
        }
        __syncthreads();
        {   // T^T dT -> P
            float z[4][4] = {};
            mma_tile<4, 4>(z, sm.T, 1, LDC, sm.D, LDC, 1, C, tm, 16, tn, 16);
            __syncthreads();
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) sm.P[(tm + 16 * i) * LDC + tn + 16 * j] = z[i][j];
        }
        __syncthreads();
        {   // dA = -strictly-lower((T^T dT) T^T); dbeta += rowsum(MA dA); dMA = beta dA -> D
            float da[4][4] = {};
            mma_tile<4, 4>(da, sm.P, LDC, 1, sm.T, 1, LDC, C, tm, 16, tn, 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = tm + 16 * i;
                float part = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int s = tn + 16 * j;
                    const float a = s < r ? -da[i][j] : 0.f;
                    part = fmaf(sm.MA[r * LDC + s], a, part);
                    sm.D[r * LDC + s] = sm.beta[r] * a;
                }
                db[i] += sum16(part);
            }
        }
        __syncthreads();
        // a_k += dMA K~n; a_n += dMA^T K~
        mma_tile<4, TK>(ak, sm.D, LDC, 1, sm.kf, LDK, 1, C, tm, 16, tn, 16);
        mma_tile<4, TK>(an, sm.D, 1, LDC, sm.km, LDK, 1, C, tm, 16, tn, 16);
        {   // dX = -beta dY (in dY); then dS = diag(gamma) dS' + e^G_m ((q E)^T dO + (k E)^T dX) -> Sm
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = tm + 16 * i;
                sm.dY[r * NV + tn] *= -sm.beta[r];
            }
            __syncthreads();
            float ds[TK][1] = {};
            mma_tile<TK, 1>(ds, sm.qm, 1, LDK, sm.dO, NV, 1, C, tm, 16, tn, 16);
            mma_tile<TK, 1>(ds, sm.km, 1, LDK, sm.dY, NV, 1, C, tm, 16, tn, 16);
#pragma unroll
            for (int i = 0; i < TK; ++i) {
                const int c = tm + 16 * i, e = c * NV + tn;
                sm.Sm[e] = fmaf(sm.gam[c], sm.dS[e], sm.gm[c] * ds[i][0]);
            }
        }
        __syncthreads();
        // dG = Q~ a_q + K~ a_k - K~n a_n (into qm); dq = E a_q, dk = E a_k + a_n / E
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = tm + 16 * i;
#pragma unroll
            for (int j = 0; j < TK; ++j) {
                const int c = tn + 16 * j;
                const float g = sm.qm[r * LDK + c] * aq[i][j] + sm.km[r * LDK + c] * ak[i][j] -
                                sm.kf[r * LDK + c] * an[i][j];
                sm.qm[r * LDK + c] = g;
                if (r < L) {
                    const float E = escr[r * DK + c];
                    const size_t off = ((size_t)(tok + r) * H + h) * DK + c;
                    atomicAdd(p.dq + off, E * aq[i][j]);
                    atomicAdd(p.dk + off, E * ak[i][j] + an[i][j] / E);
                }
            }
            if (tn == 0 && r < L) atomicAdd(p.dbeta + (size_t)(tok + r) * H + h, db[i]);
        }
        __syncthreads();
        if (tid < DK) {   // dlog alpha: reverse cumulative sum of dG inside the chunk
            const int c = tid;
            float acc = sm.dgl[c];
            for (int r = L - 1; r >= 0; --r) {
                acc += sm.qm[r * LDK + c];
                atomicAdd(p.dla + ((size_t)(tok + r) * H + h) * DK + c, acc);
            }
        }
        for (int e = tid; e < DK * NV; e += NT) sm.dS[e] = sm.Sm[e];
        __syncthreads();
    }
    if (p.ds0)
        for (int e = tid; e < DK * NV; e += NT) {
            const int c = e / NV, j = e % NV;
            p.ds0[(((size_t)n * H + h) * DK + c) * DV + col0 + j] = sm.dS[e];
        }
}

// First chunk of every packed sequence: choff[i] = sum_{j<i} ceil(len_j / 64)
// (negative lengths count as empty).  One CTA; each thread sums a contiguous
// range of sequences, then a block-wide scan.
__global__ void __launch_bounds__(1024) chunk_offsets_kernel(const int32_t* cu, int nseq, int32_t* choff)
{
    __shared__ int warp_tot[32];
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int per = (nseq + 1023) / 1024;
    const int a = min(nseq, tid * per), b = min(nseq, a + per);
    int local = 0;
    for (int i = a; i < b; ++i) local += (max(0, cu[i + 1] - cu[i]) + C - 1) / C;
    int x = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[w] = x;
    __syncthreads();
    if (w == 0) {
        int t = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        warp_tot[lane] = t;
    }
    __syncthreads();
    int base = x - local + (w ? warp_tot[w - 1] : 0);
    for (int i = a; i < b; ++i) {
        choff[i] = base;
        base += (max(0, cu[i + 1] - cu[i]) + C - 1) / C;
    }
}

// Bytes of workspace: states (chunks + 1 per sequence), the E scratch of
// every CTA, and for packed batches the chunk offsets.
size_t workspace(int nseq, int T, long long tokens, int H, int dk, int dv, bool varlen)
{
    const long long slots = varlen ? tokens / C + 2LL * nseq : (long long)nseq * ((T + C - 1) / C + 1);
    const long long ctas = (long long)nseq * H * (dv / NV);
    auto al = [](size_t x) { return (x + 1023) & ~(size_t)1023; };
    return al((size_t)slots * H * dk * dv * 4) + al((size_t)ctas * C * dk * 4) +
           (varlen ? al(((size_t)nseq + 1) * 4) : 0);
}

template <typename TIn, int DK>
cudaError_t launch(const void* q, const void* k, const void* v, Params p, int dv, unsigned char* ws,
                   cudaStream_t stream)
{
    const long long ctas = (long long)p.nseq * p.H * (dv / NV);
    if (ctas > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    auto kern = chunk_bwd_kernel<TIn, DK>;
    const size_t smem = sizeof(Smem<DK>);
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    if (ctas == 0) return cudaSuccess;
    kern<<<(unsigned)ctas, NT, smem, stream>>>(static_cast<const TIn*>(q), static_cast<const TIn*>(k),
                                               static_cast<const TIn*>(v), p);
    return cudaGetLastError();
}

}  // namespace bwd

size_t chunk_bwd_workspace(int nseq, int T, long long tokens, int H, int dk, int dv, bool varlen)
{
    return bwd::workspace(nseq, T, tokens, H, dk, dv, varlen);
}

cudaError_t chunk_bwd(const void* q, const void* k, const void* v, const float* beta, const float* log_alpha,
                      const float* s0, const float* dout, const float* dsT, float* dq, float* dk, float* dv,
                      float* dbeta, float* dla, float* ds0, const int32_t* cu, int nseq, int T, long long tokens,
                      int H, int dkd, int dvd, kda_dtype dtype, void* ws, size_t ws_bytes, cudaStream_t stream)
{
    const bool varlen = cu != nullptr;
    if (!ws || ws_bytes < bwd::workspace(nseq, T, tokens, H, dkd, dvd, varlen)) return cudaErrorInvalidValue;
    auto al = [](size_t x) { return (x + 1023) & ~(size_t)1023; };
    const long long slots = varlen ? tokens / bwd::C + 2LL * nseq : (long long)nseq * ((T + bwd::C - 1) / bwd::C + 1);
    const long long ctas = (long long)nseq * H * (dvd / bwd::NV);
    unsigned char* w = static_cast<unsigned char*>(ws);
    bwd::Params p{};
    p.beta = beta;
    p.log_alpha = log_alpha;
    p.s0 = s0;
    p.dout = dout;
    p.dsT = dsT;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.dbeta = dbeta;
    p.dla = dla;
    p.ds0 = ds0;
    p.states = reinterpret_cast<float*>(w);
    p.escr = reinterpret_cast<float*>(w + al((size_t)slots * H * dkd * dvd * 4));
    int32_t* choff = reinterpret_cast<int32_t*>(w + al((size_t)slots * H * dkd * dvd * 4) +
                                                al((size_t)ctas * bwd::C * dkd * 4));
    p.cu = cu;
    p.choff = varlen ? choff : nullptr;
    p.tokens = tokens;
    p.nseq = nseq;
    p.T = T;
    p.H = H;
    p.DV = dvd;
    const size_t th = (size_t)tokens * H;
    cudaError_t err = cudaMemsetAsync(dq, 0, th * dkd * 4, stream);
    if (err == cudaSuccess) err = cudaMemsetAsync(dk, 0, th * dkd * 4, stream);
    if (err == cudaSuccess) err = cudaMemsetAsync(dla, 0, th * dkd * 4, stream);
    if (err == cudaSuccess) err = cudaMemsetAsync(dbeta, 0, th * 4, stream);
    if (err == cudaSuccess && varlen) {
        bwd::chunk_offsets_kernel<<<1, 1024, 0, stream>>>(cu, nseq, choff);
        err = cudaGetLastError();
    }
    if (err != cudaSuccess) return err;
    using bf = __nv_bfloat16;
    if (dtype == KDA_BF16)
        return dkd == 128 ? bwd::launch<bf, 128>(q, k, v, p, dvd, w, stream) : bwd::launch<bf, 64>(q, k, v, p, dvd, w, stream);
    return dkd == 128 ? bwd::launch<float, 128>(q, k, v, p, dvd, w, stream)
                      : bwd::launch<float, 64>(q, k, v, p, dvd, w, stream);
}

}  // namespace kda
