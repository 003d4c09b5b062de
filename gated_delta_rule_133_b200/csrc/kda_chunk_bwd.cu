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
// Only the two walks over the chunks are sequential, and they carry nothing
// but [d_k x 32] slices of S and dS.  Four launches:
//   1. factors   one CTA per (chunk, head): the V-independent factors (Q~, K~,
//                K~n, G, P, T, MA and the channel vectors), once per chunk,
//                stored as a record;
//   2. forward   one CTA per (sequence, head, 32 value columns): the state
//                entering every chunk, and U = T Y;
//   3. reverse   the same CTAs carry dS back: the gradient reaching every
//                chunk's end state, dU and dY; dv and dS_0 are written here;
//   4. gradients one CTA per (chunk, head): every product that sums over
//                value columns (dP, dT, the a_* terms) over all columns at
//                once, then dA, and dq, dk, dbeta and dlog alpha of the
//                chunk's rows, written without atomics.
#include "kda_chunk.cuh"
#include "kda_packed.cuh"

namespace kda {

namespace bwd {

using simt::mma_rk;
using simt::mma_tk;
using simt::mma_tile;

constexpr int C = 64;       // chunk length
constexpr int NW = 32;      // value columns per walk CTA
constexpr int NV = 16;      // value columns per pass of the gradient kernel
constexpr int NT = 256;     // threads per CTA

// Factor record of one (chunk, head), in floats, laid out so that each walk
// streams two contiguous parts (the channel vectors are stored twice):
//   Q~, K~ [C][DK]; VEC;  P, T [C][C]; K~n [C][DK]; VEC again;  G [C][DK]; MA, T^T [C][C]
// with VEC = e^G_m, e^G_last, e^(G_last - G_m) [DK] and beta [C].
//   forward walk: part 0 = K~, VEC;          part 1 = T, K~n, VEC
//   reverse walk: part 0 = P, T, K~n, VEC;   part 1 = Q~, K~, VEC
template <int DK>
struct Rec {
    static constexpr int VECN = 3 * DK + C;
    static constexpr int QM = 0, KM = QM + C * DK, VEC = KM + C * DK;
    static constexpr int GM = VEC, GAM = VEC + DK, GLM = VEC + 2 * DK, BETA = VEC + 3 * DK;
    static constexpr int P = VEC + VECN, T = P + C * C, KF = T + C * C, VEC2 = KF + C * DK;
    static constexpr int G = VEC2 + VECN, MA = G + C * DK, TT = MA + C * C;
    static constexpr int FLOATS = (TT + C * C + 63) & ~63;
    // vector offsets inside a VEC block
    static constexpr int V_GM = 0, V_GAM = DK, V_GLM = 2 * DK, V_BETA = 3 * DK;
};

struct Params {
    const float* beta;
    const float* log_alpha;
    const float* s0;         // [nseq, H, DK, DV] or nullptr
    const float* dout;       // [tokens, H, DV]
    const float* dsT;        // [nseq, H, DK, DV] or nullptr
    float* dq;               // [tokens, H, DK]
    float* dk;
    float* dv;               // [tokens, H, DV]
    float* dbeta;            // [tokens, H]
    float* dla;              // [tokens, H, DK]
    float* ds0;              // [nseq, H, DK, DV] or nullptr
    float* states;           // state entering every chunk, and the final one: [slot][H][DK][DV]
    float* rec;              // factor records [record][H][Rec::FLOATS]
    float* U;                // [record][H][C][DV]
    float* dU;
    float* dY;
    float* VX;               // V - X of every chunk: [record][H][C][DV]
    float* dSn;              // gradient reaching the state after each chunk: [record][H][DK][DV]
    const int32_t* cu;
    const int32_t* choff;    // varlen: first record of each sequence, [nseq + 1]
    long long tokens;
    long long nrec;          // records per head the workspace holds
    int nseq, T, H, DV, nch; // nch: chunks per sequence (dense)
};

__device__ __forceinline__ packed::Layout layout_of(const Params& p)
{
    return packed::Layout{p.cu, p.choff, p.tokens, p.nrec, p.nseq, p.T, p.nch, p.H};
}

// Sum over the 16 threads (consecutive lanes) that share tm.
__device__ __forceinline__ float sum16(float x)
{
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Copies a [ROWS][COLS] row-major block from global memory into shared
// memory with row pitch ld, optionally scaling column c by sc[c].  Every load
// of a thread is issued before its first store (src 16-byte aligned, read-only
// for the kernel's lifetime).
template <int ROWS, int COLS>
__device__ __forceinline__ void stage(float* dst, int ld, const float* src, const float* sc = nullptr)
{
    constexpr int Q4 = COLS / 4, N = ROWS * Q4 / NT;
    static_assert(ROWS * Q4 % NT == 0, "tile not a multiple of the CTA");
    float4 x[N];
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const int e = threadIdx.x + i * NT;
        x[i] = __ldg(reinterpret_cast<const float4*>(src + (size_t)(e / Q4) * COLS + 4 * (e % Q4)));
    }
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const int e = threadIdx.x + i * NT;
        const int r = e / Q4, c = 4 * (e % Q4);
        if (sc) {
            x[i].x *= sc[c];
            x[i].y *= sc[c + 1];
            x[i].z *= sc[c + 2];
            x[i].w *= sc[c + 3];
        }
        float* d = dst + r * ld + c;
        d[0] = x[i].x;
        d[1] = x[i].y;
        d[2] = x[i].z;
        d[3] = x[i].w;
    }
}

// ================================================================ 1. factors

template <int DK>
struct FacSmem {
    // A and T take the place of q E and k E once the products have read
    // them, so that two CTAs fit on an SM
    static constexpr int LDK = DK + 1, LDC = C + 1;
    union {
        struct {
            float qm[C * LDK];    // q, then q E
            float km[C * LDK];    // k, then k E
        };
        struct {
            float D[C * LDC];     // A = beta MA
            float T[C * LDC];     // (I + A)^-1
        };
    };
    float kf[C * LDK];    // log alpha, then G, then k F
    float beta[C];
    static_assert(LDC <= LDK, "A and T fit in the space of q E and k E");
};

template <typename TIn, int DK>
__global__ void __launch_bounds__(NT, 2)
bwd_factor_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const Params p)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    FacSmem<DK>& sm = *reinterpret_cast<FacSmem<DK>*>(smem_raw);
    using R = Rec<DK>;
    constexpr int LDK = FacSmem<DK>::LDK, LDC = FacSmem<DK>::LDC;
    const packed::Pos x = packed::locate(layout_of(p), blockIdx.x);
    if (!x.ok) return;
    const int tid = threadIdx.x, H = p.H, L = x.L, h = x.h;
    float* rec = p.rec + (size_t)blockIdx.x * R::FLOATS;

    {
        const size_t row0 = ((size_t)x.tok * H + h) * DK, stride = (size_t)H * DK;
        packed::load_rows<TIn, DK, NT>(sm.qm, LDK, q + row0, stride, L);
        packed::load_rows<TIn, DK, NT>(sm.km, LDK, k + row0, stride, L);
        packed::load_rows<float, DK, NT>(sm.kf, LDK, p.log_alpha + row0, stride, L);
    }
    if (tid < C) {
        const float b = tid < L ? p.beta[(size_t)(x.tok + tid) * H + h] : 0.f;
        sm.beta[tid] = b;
        rec[R::VEC + R::V_BETA + tid] = b;
        rec[R::VEC2 + R::V_BETA + tid] = b;
    }
    __syncthreads();
    if (tid < DK) {   // gate cumsum per channel (fp32, log space) and the factor split
        const int c = tid;
        float acc = 0.f;
        for (int r = 0; r < C; ++r) {
            acc += sm.kf[r * LDK + c];
            sm.kf[r * LDK + c] = acc;
            rec[R::G + r * DK + c] = acc;
        }
        const float Gm = sm.kf[(C / 2 - 1) * LDK + c];
        check_domain(sm.kf[c], Gm, acc);
        const float vg[3] = {expf(Gm), expf(acc), expf(acc - Gm)};
#pragma unroll
        for (int u = 0; u < 3; ++u) {
            rec[R::VEC + u * DK + c] = vg[u];
            rec[R::VEC2 + u * DK + c] = vg[u];
        }
        for (int r = 0; r < C; ++r) {
            const float e = fminf(fmaxf(sm.kf[r * LDK + c] - Gm, -80.f), 80.f);
            const float E = expf(e), F = expf(-e);
            const float qe = sm.qm[r * LDK + c] * E;
            const float kk = sm.km[r * LDK + c];
            sm.qm[r * LDK + c] = qe;
            sm.km[r * LDK + c] = kk * E;
            sm.kf[r * LDK + c] = kk * F;
            rec[R::QM + r * DK + c] = qe;
            rec[R::KM + r * DK + c] = kk * E;
            rec[R::KF + r * DK + c] = kk * F;
        }
    }
    __syncthreads();
    {   // MA (strictly lower), P (lower incl.) to the record; A = beta MA -> D
        const int tn = tid % 16, tm = tid / 16;
        float pp[4][4] = {}, a[4][4] = {};
        mma_tile<4, 4>(pp, sm.qm, LDK, 1, sm.kf, 1, LDK, DK, tm, 16, tn, 16);
        mma_tile<4, 4>(a, sm.km, LDK, 1, sm.kf, 1, LDK, DK, tm, 16, tn, 16);
        __syncthreads();   // q E and k E are read: A takes their place
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = tm + 16 * i, s = tn + 16 * j;
                rec[R::P + r * C + s] = s <= r ? pp[i][j] : 0.f;
                rec[R::MA + r * C + s] = s < r ? a[i][j] : 0.f;
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
    for (int e = tid; e < C * C; e += NT) {
        rec[R::T + e] = sm.T[(e / C) * LDC + e % C];
        rec[R::TT + e] = sm.T[(e % C) * LDC + e / C];
    }
}

// ================================================================ 2. forward walk

// Shared memory of the forward walk: the two streamed record parts
// (unpadded, as stored), the state slice, e^G_m S, V, Y and U.
template <int DK>
struct FwdSmem {
    using R = Rec<DK>;
    float p0[C * DK + R::VECN];            // K~, VEC
    float p1[C * C + C * DK + R::VECN];    // T, K~n, VEC
    float S[DK * NW];     // state slice entering the chunk
    float Sm[DK * NW];    // e^G_m S
    float V[C * NW];
    float Y[C * NW];
    float U[C * NW];
    packed::Stream st;
};

// Per chunk: wait for part 0; X = K~ (e^G_m S), Y = beta (V - X); part 0 of
// the next chunk is fetched; wait for part 1; U = T Y; S <- gamma S +
// e^(G_last - G_m) (K~n^T U); part 1 of the next chunk is fetched.
template <typename TIn, int DK>
__global__ void __launch_bounds__(NT, 1)
bwd_forward_kernel(const TIn* __restrict__ v, const Params p)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    FwdSmem<DK>& sm = *reinterpret_cast<FwdSmem<DK>*>(smem_raw);
    using R = Rec<DK>;
    constexpr int TK = DK / 16;
    constexpr int NVR = C * NW / NT;   // V elements per thread
    constexpr uint32_t B0 = (C * DK + R::VECN) * 4, B1 = (C * C + C * DK + R::VECN) * 4;
    const float* KM = sm.p0;
    const float* vec = sm.p0 + C * DK;
    const float* T = sm.p1;
    const float* KF = sm.p1 + C * C;
    const float* vec2 = KF + C * DK;
    const int DV = p.DV, H = p.H;
    const int nslice = DV / NW;
    const int slice = blockIdx.x % nslice;
    const int h = (blockIdx.x / nslice) % H;
    const int n = blockIdx.x / (nslice * H);
    const int col0 = slice * NW;
    const int tid = threadIdx.x, tn = tid % 16, tm = tid / 16;

    const packed::Walk wk = packed::walk_of(layout_of(p), n, true);
    if (!wk.has_slots) return;   // nothing of this sequence is read again
    const int nch = (wk.len + C - 1) / C;
    auto rec_of = [&](int ci) { return p.rec + ((size_t)(wk.rbase + ci) * H + h) * R::FLOATS; };
    auto v_at = [&](int ci, int e) {
        const int r = e / NW, j = e % NW;
        return ci * C + r < wk.len ? Elem<TIn>::load(v + ((size_t)(wk.tok0 + ci * C + r) * H + h) * DV + col0 + j)
                                   : 0.f;
    };

    packed::stream_init(sm.st);
    if (tid == 0 && nch > 0) {
        packed::stream_fetch(sm.st, 0, sm.p0, rec_of(0) + R::KM, B0);
        packed::stream_fetch(sm.st, 1, sm.p1, rec_of(0) + R::T, B1);
    }
    for (int e = tid; e < DK * NW; e += NT) {
        const int c = e / NW, j = e % NW;
        sm.S[e] = p.s0 ? p.s0[(((size_t)n * H + h) * DK + c) * DV + col0 + j] : 0.f;
    }
    if (nch > 0)
#pragma unroll
        for (int i = 0; i < NVR; ++i) sm.V[tid + i * NT] = v_at(0, tid + i * NT);
    __syncthreads();
    for (int ci = 0; ci < nch; ++ci) {
        const size_t item = (size_t)(wk.rbase + ci) * H + h;
        float* st = p.states + ((wk.sbase + ci) * H + h) * (size_t)DK * DV + col0;
        for (int e = tid; e < DK * NW; e += NT) st[(e / NW) * DV + e % NW] = sm.S[e];
        if (!packed::stream_wait(sm.st, 0, ci)) goto drain;
        for (int e = tid; e < DK * NW; e += NT) sm.Sm[e] = vec[R::V_GM + e / NW] * sm.S[e];
        __syncthreads();
        {   // X = K~ Sm, Y = beta (V - X); V - X is kept for the gradient kernel
            float xx[4][2] = {};
            mma_rk<4, 2>(xx, KM, DK, sm.Sm, NW, DK, 4 * tm, 2 * tn);
            float* vxg = p.VX + item * (size_t)C * DV + col0;
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int r = 4 * tm + i, cc = 2 * tn + j, e = r * NW + cc;
                    const float vx = sm.V[e] - xx[i][j];
                    sm.Y[e] = vec[R::V_BETA + r] * vx;
                    vxg[(size_t)r * DV + cc] = vx;
                }
        }
        __syncthreads();   // part 0 is read
        if (tid == 0 && ci + 1 < nch) packed::stream_fetch(sm.st, 0, sm.p0, rec_of(ci + 1) + R::KM, B0);
        if (!packed::stream_wait(sm.st, 1, ci)) goto drain;
        float vn[NVR];   // next chunk's V, in flight during the arithmetic below
#pragma unroll
        for (int i = 0; i < NVR; ++i) vn[i] = ci + 1 < nch ? v_at(ci + 1, tid + i * NT) : 0.f;
        {   // U = T Y
            float u[4][2] = {};
            mma_rk<4, 2>(u, T, C, sm.Y, NW, C, 4 * tm, 2 * tn);
            float* ug = p.U + item * (size_t)C * DV + col0;
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int r = 4 * tm + i, cc = 2 * tn + j;
                    sm.U[r * NW + cc] = u[i][j];
                    ug[(size_t)r * DV + cc] = u[i][j];
                }
        }
        __syncthreads();
        {   // S <- gamma S + e^(G_last - G_m) (K~n^T U)
            float ds[TK][2] = {};
            mma_tk<TK, 2>(ds, KF, DK, sm.U, NW, C, TK * tm, 2 * tn);
#pragma unroll
            for (int i = 0; i < TK; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int c = TK * tm + i, e = c * NW + 2 * tn + j;
                    sm.S[e] = fmaf(vec2[R::V_GAM + c], sm.S[e], vec2[R::V_GLM + c] * ds[i][j]);
                }
        }
        __syncthreads();   // part 1, V and U are read
        if (tid == 0 && ci + 1 < nch) packed::stream_fetch(sm.st, 1, sm.p1, rec_of(ci + 1) + R::T, B1);
#pragma unroll
        for (int i = 0; i < NVR; ++i) sm.V[tid + i * NT] = vn[i];
        __syncthreads();
    }
    {
        float* st = p.states + ((wk.sbase + nch) * H + h) * (size_t)DK * DV + col0;
        for (int e = tid; e < DK * NW; e += NT) st[(e / NW) * DV + e % NW] = sm.S[e];
    }
    return;
drain:
    packed::stream_drain(sm.st);
}

// ================================================================ 3. reverse walk

template <int DK>
struct RevSmem {
    using R = Rec<DK>;
    float p0[2 * C * C + C * DK + R::VECN];   // P, T, K~n, VEC
    float p1[2 * C * DK + R::VECN];           // Q~, K~, VEC
    float dS[DK * NW];    // gradient reaching the state after the chunk, then before it
    float dSg[DK * NW];   // e^(G_last - G_m) dS'
    float dO[C * NW];
    float dU[C * NW];
    float dX[C * NW];     // -beta dY
    packed::Stream st;
};

// Per chunk (last to first): wait for part 0; dU = P^T dO + K~n dSg, dY =
// T^T dU (dv and dX); part 0 of the previous chunk is fetched; wait for part
// 1; dS <- gamma dS' + e^G_m (Q~^T dO + K~^T dX); part 1 is fetched.
template <int DK>
__global__ void __launch_bounds__(NT, 1)
bwd_reverse_kernel(const Params p)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    RevSmem<DK>& sm = *reinterpret_cast<RevSmem<DK>*>(smem_raw);
    using R = Rec<DK>;
    constexpr int TK = DK / 16;
    constexpr int NVR = C * NW / NT;
    constexpr uint32_t B0 = (2 * C * C + C * DK + R::VECN) * 4, B1 = (2 * C * DK + R::VECN) * 4;
    const float* P = sm.p0;
    const float* T = sm.p0 + C * C;
    const float* KF = sm.p0 + 2 * C * C;
    const float* vec2 = KF + C * DK;
    const float* QM = sm.p1;
    const float* KM = sm.p1 + C * DK;
    const float* vec = sm.p1 + 2 * C * DK;
    const int DV = p.DV, H = p.H;
    const int nslice = DV / NW;
    const int slice = blockIdx.x % nslice;
    const int h = (blockIdx.x / nslice) % H;
    const int n = blockIdx.x / (nslice * H);
    const int col0 = slice * NW;
    const int tid = threadIdx.x, tn = tid % 16, tm = tid / 16;

    // a skipped sequence was reported by the forward walk
    const packed::Walk wk = packed::walk_of(layout_of(p), n, false);
    const int nch = (wk.len + C - 1) / C;
    auto rec_of = [&](int ci) { return p.rec + ((size_t)(wk.rbase + ci) * H + h) * R::FLOATS; };
    auto do_at = [&](int ci, int e) {
        const int r = e / NW, j = e % NW;
        return ci * C + r < wk.len ? p.dout[((size_t)(wk.tok0 + ci * C + r) * H + h) * DV + col0 + j] : 0.f;
    };

    packed::stream_init(sm.st);
    if (tid == 0 && nch > 0) {
        packed::stream_fetch(sm.st, 0, sm.p0, rec_of(nch - 1) + R::P, B0);
        packed::stream_fetch(sm.st, 1, sm.p1, rec_of(nch - 1) + R::QM, B1);
    }
    for (int e = tid; e < DK * NW; e += NT) {
        const int c = e / NW, j = e % NW;
        sm.dS[e] = p.dsT ? p.dsT[(((size_t)n * H + h) * DK + c) * DV + col0 + j] : 0.f;
    }
    if (nch > 0)
#pragma unroll
        for (int i = 0; i < NVR; ++i) sm.dO[tid + i * NT] = do_at(nch - 1, tid + i * NT);
    __syncthreads();
    for (int ci = nch - 1, k = 0; ci >= 0; --ci, ++k) {
        const int L = min(C, wk.len - ci * C), tok = wk.tok0 + ci * C;
        const size_t item = (size_t)(wk.rbase + ci) * H + h;
        float* dsn = p.dSn + item * (size_t)DK * DV + col0;
        for (int e = tid; e < DK * NW; e += NT) dsn[(e / NW) * DV + e % NW] = sm.dS[e];
        if (!packed::stream_wait(sm.st, 0, k)) goto drain;
        for (int e = tid; e < DK * NW; e += NT) sm.dSg[e] = vec2[R::V_GLM + e / NW] * sm.dS[e];
        __syncthreads();
        {   // dU = P^T dO + K~n dSg
            float du[4][2] = {};
            mma_tk<4, 2>(du, P, C, sm.dO, NW, C, 4 * tm, 2 * tn);
            mma_rk<4, 2>(du, KF, DK, sm.dSg, NW, DK, 4 * tm, 2 * tn);
            float* g = p.dU + item * (size_t)C * DV + col0;
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int r = 4 * tm + i, cc = 2 * tn + j;
                    sm.dU[r * NW + cc] = du[i][j];
                    g[(size_t)r * DV + cc] = du[i][j];
                }
        }
        __syncthreads();
        {   // dY = T^T dU; dv = beta dY; dX = -beta dY
            float dy[4][2] = {};
            mma_tk<4, 2>(dy, T, C, sm.dU, NW, C, 4 * tm, 2 * tn);
            float* g = p.dY + item * (size_t)C * DV + col0;
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int r = 4 * tm + i, cc = 2 * tn + j;
                    const float b = vec2[R::V_BETA + r];
                    g[(size_t)r * DV + cc] = dy[i][j];
                    sm.dX[r * NW + cc] = -b * dy[i][j];
                    if (r < L) p.dv[((size_t)(tok + r) * H + h) * DV + col0 + cc] = b * dy[i][j];
                }
        }
        __syncthreads();   // part 0 is read
        if (tid == 0 && ci > 0) packed::stream_fetch(sm.st, 0, sm.p0, rec_of(ci - 1) + R::P, B0);
        if (!packed::stream_wait(sm.st, 1, k)) goto drain;
        float dn[NVR];   // previous chunk's dO, in flight during the arithmetic below
#pragma unroll
        for (int i = 0; i < NVR; ++i) dn[i] = ci > 0 ? do_at(ci - 1, tid + i * NT) : 0.f;
        {   // dS = gamma dS' + e^G_m (Q~^T dO + K~^T dX)
            float ds[TK][2] = {};
            mma_tk<TK, 2>(ds, QM, DK, sm.dO, NW, C, TK * tm, 2 * tn);
            mma_tk<TK, 2>(ds, KM, DK, sm.dX, NW, C, TK * tm, 2 * tn);
#pragma unroll
            for (int i = 0; i < TK; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int c = TK * tm + i, e = c * NW + 2 * tn + j;
                    sm.dS[e] = fmaf(vec[R::V_GAM + c], sm.dS[e], vec[R::V_GM + c] * ds[i][j]);
                }
        }
        __syncthreads();   // part 1 and dO are read
        if (tid == 0 && ci > 0) packed::stream_fetch(sm.st, 1, sm.p1, rec_of(ci - 1) + R::QM, B1);
#pragma unroll
        for (int i = 0; i < NVR; ++i) sm.dO[tid + i * NT] = dn[i];
        __syncthreads();
    }
    if (p.ds0)
        for (int e = tid; e < DK * NW; e += NT) {
            const int c = e / NW, j = e % NW;
            p.ds0[(((size_t)n * H + h) * DK + c) * DV + col0 + j] = sm.dS[e];
        }
    return;
drain:
    packed::stream_drain(sm.st);
}

// ================================================================ 4. gradients

// Every operand tile is laid out so that the products read it along rows:
// the record tiles unpadded, the pass tiles that serve as B operands
// transposed ([16][*]).  A thread owns rows 4 tm .. 4 tm + 3 and a run of
// consecutive columns of every accumulator.
template <int DK>
struct GradSmem {
    float qm[C * DK];     // Q~, then dG
    float km[C * DK];     // K~
    float kf[C * DK];     // K~n
    float MA[C * C];
    float T[C * C];
    float TT[C * C];      // T^T
    float D1[C * C];      // dP, then T^T dT
    float D2[C * C];      // dT, then dMA
    float dO[C * NV];     // pass tiles, [C][16]
    float dX[C * NV];     // -beta dY
    float U[C * NV];
    float dU[C * NV];
    float SmT[NV * DK];   // (e^G_m S)^T, [16][DK]
    float dSgT[NV * DK];  // (e^(G_last - G_m) dS')^T
    float UT[NV * C];     // U^T, [16][C]
    float YT[NV * C];     // (beta (V - X))^T
    float gm[DK];
    float glm[DK];
    float dgl[DK];        // rowsum(dS' S'): the last row's extra dG
    float beta[C];
    float db[C];
};

template <int DK>
__global__ void __launch_bounds__(NT, 1)
bwd_grad_kernel(const Params p)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    GradSmem<DK>& sm = *reinterpret_cast<GradSmem<DK>*>(smem_raw);
    using R = Rec<DK>;
    constexpr int TK = DK / 16;   // accumulator columns per thread: TK tn .. TK tn + TK - 1
    const packed::Pos x = packed::locate(layout_of(p), blockIdx.x);
    if (!x.ok) return;
    const int tid = threadIdx.x, tn = tid % 16, tm = tid / 16;
    const int DV = p.DV, H = p.H, L = x.L, h = x.h;
    const int m0 = 4 * tm, n0 = TK * tn, s0c = 4 * tn;
    const size_t item = blockIdx.x;
    const float* rec = p.rec + item * R::FLOATS;
    const float* S0 = p.states + ((size_t)x.slot * H + h) * (size_t)DK * DV;          // entering the chunk
    const float* S1 = p.states + ((size_t)(x.slot + 1) * H + h) * (size_t)DK * DV;    // after it
    const float* dS1 = p.dSn + item * (size_t)DK * DV;
    const float* Ug = p.U + item * (size_t)C * DV;
    const float* dUg = p.dU + item * (size_t)C * DV;
    const float* dYg = p.dY + item * (size_t)C * DV;
    const float* VXg = p.VX + item * (size_t)C * DV;

    if (tid < DK) {
        sm.gm[tid] = rec[R::GM + tid];
        sm.glm[tid] = rec[R::GLM + tid];
    }
    if (tid < C) sm.beta[tid] = rec[R::BETA + tid];
    stage<C, DK>(sm.qm, DK, rec + R::QM);
    stage<C, DK>(sm.km, DK, rec + R::KM);
    stage<C, DK>(sm.kf, DK, rec + R::KF);
    stage<C, C>(sm.MA, C, rec + R::MA);
    stage<C, C>(sm.T, C, rec + R::T);
    stage<C, C>(sm.TT, C, rec + R::TT);

    float aq[4][TK] = {}, ak[4][TK] = {}, an[4][TK] = {};
    float dp[4][4] = {}, dt[4][4] = {};
    float db1 = 0.f;      // rowsum((V - X) dY) of row tid / 4 over this thread's columns
    // pass loads: thread tid holds float4 number tid + i NT of each [DK][16]
    // slice (channel (tid + i NT) / 4) and float4 number tid of each [C][16]
    // slice (row tid / 4); all are issued before the first store
    constexpr int NS = DK * NV / 4 / NT;              // float4 per thread of a [DK][16] slice
    static_assert(C * NV / 4 == NT, "one float4 of a [C][16] slice per thread");
    float dgl[NS] = {};   // channel (tid + i NT) / 4, summed over this thread's columns
    const int rr = tid / 4, c4 = 4 * (tid % 4);
    const bool rin = rr < L;
    const size_t rowg = ((size_t)(x.tok + rr) * H + h) * DV;
    for (int j0 = 0; j0 < DV; j0 += NV) {
        float4 sa[NS], d1[NS], s1[NS];
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            const int e = tid + i * NT;
            const size_t g = (size_t)(e / 4) * DV + j0 + 4 * (e % 4);
            sa[i] = __ldg(reinterpret_cast<const float4*>(S0 + g));
            d1[i] = __ldg(reinterpret_cast<const float4*>(dS1 + g));
            s1[i] = __ldg(reinterpret_cast<const float4*>(S1 + g));
        }
        const size_t g = (size_t)rr * DV + j0 + c4;
        const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 o4 = rin ? __ldg(reinterpret_cast<const float4*>(p.dout + rowg + j0 + c4)) : z4;
        const float4 u4 = __ldg(reinterpret_cast<const float4*>(Ug + g));
        const float4 du4 = __ldg(reinterpret_cast<const float4*>(dUg + g));
        const float4 dy4 = __ldg(reinterpret_cast<const float4*>(dYg + g));
        const float4 vx4 = __ldg(reinterpret_cast<const float4*>(VXg + g));
        __syncthreads();   // the previous pass has read its tiles (first pass: the vectors are in place)
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            const int e = tid + i * NT, c = e / 4, q = 4 * (e % 4);
            const float gmc = sm.gm[c], glc = sm.glm[c];
            sm.SmT[(q + 0) * DK + c] = gmc * sa[i].x;
            sm.SmT[(q + 1) * DK + c] = gmc * sa[i].y;
            sm.SmT[(q + 2) * DK + c] = gmc * sa[i].z;
            sm.SmT[(q + 3) * DK + c] = gmc * sa[i].w;
            sm.dSgT[(q + 0) * DK + c] = glc * d1[i].x;
            sm.dSgT[(q + 1) * DK + c] = glc * d1[i].y;
            sm.dSgT[(q + 2) * DK + c] = glc * d1[i].z;
            sm.dSgT[(q + 3) * DK + c] = glc * d1[i].w;
            dgl[i] += d1[i].x * s1[i].x + d1[i].y * s1[i].y + d1[i].z * s1[i].z + d1[i].w * s1[i].w;
        }
        {
            const int e = rr * NV + c4;
            const float b = sm.beta[rr];
            *reinterpret_cast<float4*>(sm.dO + e) = o4;
            *reinterpret_cast<float4*>(sm.U + e) = u4;
            *reinterpret_cast<float4*>(sm.dU + e) = du4;
            *reinterpret_cast<float4*>(sm.dX + e) = make_float4(-b * dy4.x, -b * dy4.y, -b * dy4.z, -b * dy4.w);
            sm.UT[(c4 + 0) * C + rr] = u4.x;
            sm.UT[(c4 + 1) * C + rr] = u4.y;
            sm.UT[(c4 + 2) * C + rr] = u4.z;
            sm.UT[(c4 + 3) * C + rr] = u4.w;
            sm.YT[(c4 + 0) * C + rr] = b * vx4.x;
            sm.YT[(c4 + 1) * C + rr] = b * vx4.y;
            sm.YT[(c4 + 2) * C + rr] = b * vx4.z;
            sm.YT[(c4 + 3) * C + rr] = b * vx4.w;
            db1 += vx4.x * dy4.x + vx4.y * dy4.y + vx4.z * dy4.z + vx4.w * dy4.w;
        }
        __syncthreads();
        // a_q += dO Sm^T, a_k += dX Sm^T, a_n += U dSg^T; dP += dO U^T, dT += dU Y^T
        mma_rk<4, TK>(aq, sm.dO, NV, sm.SmT, DK, NV, m0, n0);
        mma_rk<4, TK>(ak, sm.dX, NV, sm.SmT, DK, NV, m0, n0);
        mma_rk<4, TK>(an, sm.U, NV, sm.dSgT, DK, NV, m0, n0);
        mma_rk<4, 4>(dp, sm.dO, NV, sm.UT, C, NV, m0, s0c);
        mma_rk<4, 4>(dt, sm.dU, NV, sm.YT, C, NV, m0, s0c);
    }
    // dP (lower incl.) -> D1, dT -> D2; dgl and the first part of dbeta
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = m0 + i;
        float4 a4, b4;
        a4.x = s0c + 0 <= r ? dp[i][0] : 0.f;
        a4.y = s0c + 1 <= r ? dp[i][1] : 0.f;
        a4.z = s0c + 2 <= r ? dp[i][2] : 0.f;
        a4.w = s0c + 3 <= r ? dp[i][3] : 0.f;
        b4 = make_float4(dt[i][0], dt[i][1], dt[i][2], dt[i][3]);
        *reinterpret_cast<float4*>(sm.D1 + r * C + s0c) = a4;
        *reinterpret_cast<float4*>(sm.D2 + r * C + s0c) = b4;
    }
    {   // the 4 threads of a row are consecutive lanes
        float b = db1;
        b += __shfl_xor_sync(0xffffffffu, b, 1);
        b += __shfl_xor_sync(0xffffffffu, b, 2);
        if ((tid & 3) == 0) sm.db[tid / 4] = b;
    }
#pragma unroll
    for (int i = 0; i < NS; ++i) {   // the 4 threads of a channel are consecutive lanes
        float g = dgl[i];
        g += __shfl_xor_sync(0xffffffffu, g, 1);
        g += __shfl_xor_sync(0xffffffffu, g, 2);
        if ((tid & 3) == 0) sm.dgl[(tid + i * NT) / 4] = g;
    }
    __syncthreads();
    // a_q += dP K~n; a_n += dP^T Q~; T^T dT
    mma_rk<4, TK>(aq, sm.D1, C, sm.kf, DK, C, m0, n0);
    mma_tk<4, TK>(an, sm.D1, C, sm.qm, DK, C, m0, n0);
    {
        float z[4][4] = {};
        mma_tk<4, 4>(z, sm.T, C, sm.D2, C, C, m0, s0c);
        __syncthreads();   // dP and dT are read
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<float4*>(sm.D1 + (m0 + i) * C + s0c) = make_float4(z[i][0], z[i][1], z[i][2], z[i][3]);
    }
    __syncthreads();
    {   // dA = -strictly-lower((T^T dT) T^T); dbeta += rowsum(MA dA); dMA = beta dA -> D2
        float da[4][4] = {};
        mma_rk<4, 4>(da, sm.D1, C, sm.TT, C, C, m0, s0c);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = m0 + i;
            const float4 ma = *reinterpret_cast<const float4*>(sm.MA + r * C + s0c);
            float a[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) a[j] = s0c + j < r ? -da[i][j] : 0.f;
            const float part = ma.x * a[0] + ma.y * a[1] + ma.z * a[2] + ma.w * a[3];
            const float br = sm.beta[r];
            *reinterpret_cast<float4*>(sm.D2 + r * C + s0c) = make_float4(br * a[0], br * a[1], br * a[2], br * a[3]);
            const float b = sum16(part);
            if (tn == 0) sm.db[r] += b;
        }
    }
    __syncthreads();
    // a_k += dMA K~n; a_n += dMA^T K~
    mma_rk<4, TK>(ak, sm.D2, C, sm.kf, DK, C, m0, n0);
    mma_tk<4, TK>(an, sm.D2, C, sm.km, DK, C, m0, n0);
    // dG = Q~ a_q + K~ a_k - K~n a_n into qm (each thread rewrites only the
    // elements it reads; no product reads Q~ any more); dq = E a_q,
    // dk = E a_k + a_n / E
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = m0 + i;
        float qv[TK], kv[TK], fv[TK];
        simt::ld_row<TK>(qv, sm.qm + r * DK + n0);
        simt::ld_row<TK>(kv, sm.km + r * DK + n0);
        simt::ld_row<TK>(fv, sm.kf + r * DK + n0);
        float g[TK];
#pragma unroll
        for (int j = 0; j < TK; ++j) g[j] = qv[j] * aq[i][j] + kv[j] * ak[i][j] - fv[j] * an[i][j];
#pragma unroll
        for (int j = 0; j < TK; j += 4)
            *reinterpret_cast<float4*>(sm.qm + r * DK + n0 + j) = make_float4(g[j], g[j + 1], g[j + 2], g[j + 3]);
        if (r < L) {
            float gr[TK], gmid[TK];
            simt::ld_row<TK>(gr, rec + R::G + r * DK + n0);
            simt::ld_row<TK>(gmid, rec + R::G + (C / 2 - 1) * DK + n0);
            float dqv[TK], dkv[TK];
#pragma unroll
            for (int j = 0; j < TK; ++j) {
                const float E = expf(fminf(fmaxf(gr[j] - gmid[j], -80.f), 80.f));
                dqv[j] = E * aq[i][j];
                dkv[j] = E * ak[i][j] + an[i][j] / E;
            }
            const size_t off = ((size_t)(x.tok + r) * H + h) * DK + n0;
#pragma unroll
            for (int j = 0; j < TK; j += 4) {
                *reinterpret_cast<float4*>(p.dq + off + j) = make_float4(dqv[j], dqv[j + 1], dqv[j + 2], dqv[j + 3]);
                *reinterpret_cast<float4*>(p.dk + off + j) = make_float4(dkv[j], dkv[j + 1], dkv[j + 2], dkv[j + 3]);
            }
        }
    }
    __syncthreads();
    if (tid < DK) {   // dlog alpha: reverse cumulative sum of dG inside the chunk
        const int c = tid;
        float acc = sm.dgl[c];
        for (int r = L - 1; r >= 0; --r) {
            acc += sm.qm[r * DK + c];
            p.dla[((size_t)(x.tok + r) * H + h) * DK + c] = acc;
        }
    }
    if (tid < L) p.dbeta[(size_t)(x.tok + tid) * H + h] = sm.db[tid];
}

// ================================================================ host side

// Parts of a call's workspace (byte offsets).
struct Ws {
    size_t states, rec, U, dU, dY, VX, dSn, choff, bytes;
    long long nrec;   // records per head (an upper bound for packed batches)
};

static size_t al1k(size_t x) { return (x + 1023) & ~(size_t)1023; }

static Ws ws_layout(int nseq, int T, long long tokens, int H, int dk, int dv, bool varlen)
{
    Ws w{};
    w.nrec = packed::records(nseq, T, tokens, varlen);
    const long long slots = packed::state_slots(nseq, T, tokens, varlen);
    const size_t recf = dk == 128 ? Rec<128>::FLOATS : Rec<64>::FLOATS;
    size_t off = 0;
    w.states = off;
    off += al1k((size_t)slots * H * dk * dv * 4);
    w.rec = off;
    off += al1k((size_t)w.nrec * H * recf * 4);
    w.U = off;
    off += al1k((size_t)w.nrec * H * C * dv * 4);
    w.dU = off;
    off += al1k((size_t)w.nrec * H * C * dv * 4);
    w.dY = off;
    off += al1k((size_t)w.nrec * H * C * dv * 4);
    w.VX = off;
    off += al1k((size_t)w.nrec * H * C * dv * 4);
    w.dSn = off;
    off += al1k((size_t)w.nrec * H * dk * dv * 4);
    w.choff = off;
    off += varlen ? al1k(((size_t)nseq + 1) * 4) : 0;
    w.bytes = off;
    return w;
}

size_t workspace(int nseq, int T, long long tokens, int H, int dk, int dv, bool varlen)
{
    return ws_layout(nseq, T, tokens, H, dk, dv, varlen).bytes;
}

template <typename TIn, int DK>
cudaError_t launch(const void* q, const void* k, const void* v, const Params& p, long long nrec, cudaStream_t stream)
{
    const long long walk_ctas = (long long)p.nseq * p.H * (p.DV / NW);
    const long long items = nrec * p.H;
    if (walk_ctas > 0x7fffffffLL || items > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    auto kf = bwd_factor_kernel<TIn, DK>;
    auto kw = bwd_forward_kernel<TIn, DK>;
    auto kr = bwd_reverse_kernel<DK>;
    auto kg = bwd_grad_kernel<DK>;
    cudaError_t err = cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(FacSmem<DK>));
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(kw, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(FwdSmem<DK>));
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(kr, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(RevSmem<DK>));
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(kg, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(GradSmem<DK>));
    if (err != cudaSuccess) return err;
    if (walk_ctas == 0) return cudaSuccess;
    const TIn* qq = static_cast<const TIn*>(q);
    const TIn* kk = static_cast<const TIn*>(k);
    const TIn* vv = static_cast<const TIn*>(v);
    if (items > 0) {
        kf<<<(unsigned)items, NT, sizeof(FacSmem<DK>), stream>>>(qq, kk, p);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    kw<<<(unsigned)walk_ctas, NT, sizeof(FwdSmem<DK>), stream>>>(vv, p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    kr<<<(unsigned)walk_ctas, NT, sizeof(RevSmem<DK>), stream>>>(p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    if (items > 0) {
        kg<<<(unsigned)items, NT, sizeof(GradSmem<DK>), stream>>>(p);
        err = cudaGetLastError();
    }
    return err;
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
    const bwd::Ws L = bwd::ws_layout(nseq, T, tokens, H, dkd, dvd, varlen);
    if (!ws || ws_bytes < L.bytes) return cudaErrorInvalidValue;
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
    p.states = reinterpret_cast<float*>(w + L.states);
    p.rec = reinterpret_cast<float*>(w + L.rec);
    p.U = reinterpret_cast<float*>(w + L.U);
    p.dU = reinterpret_cast<float*>(w + L.dU);
    p.dY = reinterpret_cast<float*>(w + L.dY);
    p.VX = reinterpret_cast<float*>(w + L.VX);
    p.dSn = reinterpret_cast<float*>(w + L.dSn);
    int32_t* choff = reinterpret_cast<int32_t*>(w + L.choff);
    p.cu = cu;
    p.choff = varlen ? choff : nullptr;
    p.tokens = tokens;
    p.nrec = L.nrec;
    p.nseq = nseq;
    p.T = T;
    p.H = H;
    p.DV = dvd;
    p.nch = varlen ? 0 : (T + bwd::C - 1) / bwd::C;
    cudaError_t err = cudaSuccess;
    if (varlen) {   // rows outside every sequence get zero gradients (dense batches write every row)
        const size_t th = (size_t)tokens * H;
        err = cudaMemsetAsync(dq, 0, th * dkd * 4, stream);
        if (err == cudaSuccess) err = cudaMemsetAsync(dk, 0, th * dkd * 4, stream);
        if (err == cudaSuccess) err = cudaMemsetAsync(dla, 0, th * dkd * 4, stream);
        if (err == cudaSuccess) err = cudaMemsetAsync(dbeta, 0, th * 4, stream);
        if (err == cudaSuccess) {
            packed::chunk_offsets_kernel<<<1, 1024, 0, stream>>>(cu, nseq, tokens, choff);
            err = cudaGetLastError();
        }
    }
    if (err != cudaSuccess) return err;
    using bf = __nv_bfloat16;
    if (dtype == KDA_BF16)
        return dkd == 128 ? bwd::launch<bf, 128>(q, k, v, p, L.nrec, stream)
                          : bwd::launch<bf, 64>(q, k, v, p, L.nrec, stream);
    return dkd == 128 ? bwd::launch<float, 128>(q, k, v, p, L.nrec, stream)
                      : bwd::launch<float, 64>(q, k, v, p, L.nrec, stream);
}

}  // namespace kda
