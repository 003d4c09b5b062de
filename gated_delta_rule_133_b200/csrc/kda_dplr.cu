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
// Two launches (plus, for packed batches, the chunk-offset kernel):
//   1. factors  one CTA per (chunk, head): the intra-chunk products, with the
//               relative decays factored around the chunk's middle row m so
//               that every factor is bounded by the decay of 32 tokens
//               (a e^{Gx - G_m}, q e^{G - G_m}, b e^{G_m - G}, k e^{G_m - G}),
//               the inverse (I - A_ab)^-1 by forward substitution, and the
//               state-side factors e^{Gx} a, e^G q, e^{G_last - G} b,
//               e^{G_last - G} k, stored as one record;
//   2. walk     one CTA per (sequence, head, 32 value columns; the columns of
//               S evolve independently, the transition acts on the d_k side)
//               carries the state through the chunks from the records.
#include "kda_chunk.cuh"
#include "kda_packed.cuh"

namespace kda {

namespace dplr {

using simt::mma_rk;
using simt::mma_tk;
using simt::mma_tile;

constexpr int C = 64;
constexpr int NW = 32;      // value columns per walk CTA
constexpr int NT = 256;

// Record of one (chunk, head), in floats, as two parts that the walk streams
// separately: part 1 e^{Gx} a, e^G q [C][DK], (I - A_ab)^-1, A_ak [C][C];
// part 2 e^{G_last - G} b, e^{G_last - G} k [C][DK], P_qb, P_qk [C][C],
// e^{G_last} [DK].
template <int DK>
struct Rec {
    static constexpr int AX = 0, QX = AX + C * DK, TI = QX + C * DK, AAK = TI + C * C;
    static constexpr int PART2 = AAK + C * C;
    static constexpr int BL = PART2, KL = BL + C * DK, PQB = KL + C * DK, PQK = PQB + C * C;
    static constexpr int GAM = PQK + C * C;
    static constexpr int FLOATS = (GAM + DK + 63) & ~63;
    static constexpr uint32_t PART1_BYTES = PART2 * 4u, PART2_BYTES = (GAM + DK - PART2) * 4u;
};

struct Params {
    const float* log_alpha;
    const float* s0;
    float* sT;
    float* rec;
    packed::Layout lay;
    int DV;
};

// ================================================================ 1. factors

template <int DK>
struct FacSmem {
    static constexpr int LDK = DK + 1, LDC = C + 1;
    float ax[C * LDK];    // a e^{Gx - G_m}
    float bf[C * LDK];    // b e^{G_m - G}
    float kf[C * LDK];    // k e^{G_m - G}
    float qx[C * LDK];    // q e^{G - G_m}
    float M[C * LDC];     // A_ab
    float T[C * LDC];     // (I - A_ab)^-1
    float part[NT];       // per-part gate sums of the cumsum
    float gmid[DK];       // G of the middle row
    float glast[DK];      // G of the last row
};

template <typename TIn, int DK>
__global__ void __launch_bounds__(NT, 1)
dplr_factor_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ a,
                   const TIn* __restrict__ b, const Params p)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    FacSmem<DK>& sm = *reinterpret_cast<FacSmem<DK>*>(smem_raw);
    using R = Rec<DK>;
    constexpr int LDK = FacSmem<DK>::LDK, LDC = FacSmem<DK>::LDC;
    const packed::Pos x = packed::locate(p.lay, blockIdx.x);
    if (!x.ok) return;
    const int tid = threadIdx.x, H = p.lay.H, L = x.L, h = x.h;
    float* rec = p.rec + (size_t)blockIdx.x * R::FLOATS;

    // rows >= L are zero: no key, no value, no decay
    {
        const size_t row0 = ((size_t)x.tok * H + h) * DK, stride = (size_t)H * DK;
        packed::load_rows<TIn, DK, NT>(sm.ax, LDK, a + row0, stride, L);
        packed::load_rows<TIn, DK, NT>(sm.bf, LDK, b + row0, stride, L);
        packed::load_rows<TIn, DK, NT>(sm.kf, LDK, k + row0, stride, L);
        packed::load_rows<TIn, DK, NT>(sm.qx, LDK, q + row0, stride, L);
    }
    __syncthreads();
    {   // gate cumsum per channel (fp32, log space), factors and the record's
        // scaled rows: thread (part, c) takes rows [part RP, (part + 1) RP) of
        // channel c; the part sums are added in part order
        constexpr int NP = NT / DK, RP = C / NP;
        const int c = tid % DK, part = tid / DK, r0 = part * RP;
        float G[RP];
        float acc = 0.f;
#pragma unroll
        for (int rr = 0; rr < RP; ++rr) {
            acc += r0 + rr < L ? p.log_alpha[((size_t)(x.tok + r0 + rr) * H + h) * DK + c] : 0.f;
            G[rr] = acc;
        }
        sm.part[tid] = acc;
        __syncthreads();
        float off = 0.f;   // G of the row before this part
        for (int q2 = 0; q2 < part; ++q2) off += sm.part[q2 * DK + c];
#pragma unroll
        for (int rr = 0; rr < RP; ++rr) G[rr] += off;
#pragma unroll
        for (int rr = 0; rr < RP; ++rr) {
            if (r0 + rr == C / 2 - 1) sm.gmid[c] = G[rr];
            if (r0 + rr == C - 1) sm.glast[c] = G[rr];
        }
        __syncthreads();
        const float Gm = sm.gmid[c], Gl = sm.glast[c];
        if (part == 0) {
            rec[R::GAM + c] = expf(Gl);
            check_domain(G[0], Gm, Gl);
        }
#pragma unroll
        for (int rr = 0; rr < RP; ++rr) {
            const int r = r0 + rr;
            const float g = G[rr], gx = rr ? G[rr - 1] : off;
            const float f = expf(fminf(Gm - g, 80.f));
            const float av = sm.ax[r * LDK + c], bv = sm.bf[r * LDK + c], kv = sm.kf[r * LDK + c];
            const float qv = sm.qx[r * LDK + c];
            sm.ax[r * LDK + c] = av * expf(fminf(gx - Gm, 80.f));
            sm.bf[r * LDK + c] = bv * f;
            sm.kf[r * LDK + c] = kv * f;
            sm.qx[r * LDK + c] = qv * expf(fminf(g - Gm, 80.f));
            const float el = expf(Gl - g);
            rec[R::AX + r * DK + c] = av * expf(gx);
            rec[R::QX + r * DK + c] = qv * expf(g);
            rec[R::BL + r * DK + c] = bv * el;
            rec[R::KL + r * DK + c] = kv * el;
        }
    }
    __syncthreads();
    const int tn = tid % 16, tm = tid / 16;
    {   // A_ab (strictly lower) -> M; A_ak (strictly lower) -> the record
        float p1[4][4] = {}, p2[4][4] = {};
        mma_tile<4, 4>(p1, sm.ax, LDK, 1, sm.bf, 1, LDK, DK, tm, 16, tn, 16);
        mma_tile<4, 4>(p2, sm.ax, LDK, 1, sm.kf, 1, LDK, DK, tm, 16, tn, 16);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = tm + 16 * i, s = tn + 16 * j;
                sm.M[r * LDC + s] = s < r ? p1[i][j] : 0.f;
                rec[R::AAK + r * C + s] = s < r ? p2[i][j] : 0.f;
            }
    }
    {   // P_qb, P_qk (lower incl.) -> the record
        float p1[4][4] = {}, p2[4][4] = {};
        mma_tile<4, 4>(p1, sm.qx, LDK, 1, sm.bf, 1, LDK, DK, tm, 16, tn, 16);
        mma_tile<4, 4>(p2, sm.qx, LDK, 1, sm.kf, 1, LDK, DK, tm, 16, tn, 16);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = tm + 16 * i, s = tn + 16 * j;
                rec[R::PQB + r * C + s] = s <= r ? p1[i][j] : 0.f;
                rec[R::PQK + r * C + s] = s <= r ? p2[i][j] : 0.f;
            }
    }
    __syncthreads();
    {   // T = (I - A_ab)^-1 by forward substitution; 4 lanes share one column
        const int j = tid >> 2, pq = tid & 3;
        for (int r = 0; r < C; ++r) {
            float acc = 0.f;
            if (r > j)
                for (int s = j + pq; s < r; s += 4) acc = fmaf(sm.M[r * LDC + s], sm.T[s * LDC + j], acc);
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            if (pq == 0) sm.T[r * LDC + j] = (r == j ? 1.f : 0.f) + (r > j ? acc : 0.f);
            __syncwarp();
        }
    }
    __syncthreads();
    for (int e = tid; e < C * C; e += NT) rec[R::TI + e] = sm.T[(e / C) * LDC + e % C];
}

// ================================================================ 2. walk

// Shared memory of the walk: the two record parts (unpadded, as stored),
// the state slice, V and W.
template <int DK>
struct WalkSmem {
    float part1[Rec<DK>::PART2];                       // AX, QX, TI, AAK
    float part2[Rec<DK>::GAM + DK - Rec<DK>::PART2];   // BL, KL, PQB, PQK, e^{G_last}
    float S[DK * NW];     // state slice
    float V[C * NW];
    float W[C * NW];      // (e^{Gx} a) S + A_ak V, then U
    packed::Stream st;
};

// Per chunk: wait for part 1; W = (e^{Gx} a) S + A_ak V and (e^G q) S;
// U = (I - A_ab)^-1 W; part 1 of the next chunk is fetched; wait for part 2;
// the output rows and the state update; part 2 of the next chunk is fetched.
// Each part's copy overlaps the other part's arithmetic.
template <typename TIn, typename TOut, int DK>
__global__ void __launch_bounds__(NT, 1)
dplr_walk_kernel(const TIn* __restrict__ v, TOut* __restrict__ o, const Params p)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    WalkSmem<DK>& sm = *reinterpret_cast<WalkSmem<DK>*>(smem_raw);
    using R = Rec<DK>;
    constexpr int TK = DK / 16;
    constexpr int NVR = C * NW / NT;   // V elements per thread
    const float* AX = sm.part1 + R::AX;
    const float* QX = sm.part1 + R::QX;
    const float* TI = sm.part1 + R::TI;
    const float* AAK = sm.part1 + R::AAK;
    const float* BL = sm.part2 + (R::BL - R::PART2);
    const float* KL = sm.part2 + (R::KL - R::PART2);
    const float* PQB = sm.part2 + (R::PQB - R::PART2);
    const float* PQK = sm.part2 + (R::PQK - R::PART2);
    const float* gam = sm.part2 + (R::GAM - R::PART2);
    const int DV = p.DV, H = p.lay.H;
    const int nslice = DV / NW;
    const int slice = blockIdx.x % nslice;
    const int h = (blockIdx.x / nslice) % H;
    const int n = blockIdx.x / (nslice * H);
    const int col0 = slice * NW;
    const int tid = threadIdx.x, tn = tid % 16, tm = tid / 16;
    const packed::Walk wk = packed::walk_of(p.lay, n, true);   // a skipped sequence keeps its initial state
    const int nch = (wk.len + C - 1) / C;
    auto rec_of = [&](int ci) { return p.rec + ((size_t)(wk.rbase + ci) * H + h) * R::FLOATS; };
    auto v_at = [&](int ci, int e) {   // element e of chunk ci's V slice (0 past the sequence)
        const int r = e / NW, j = e % NW;
        return ci * C + r < wk.len ? Elem<TIn>::load(v + ((size_t)(wk.tok0 + ci * C + r) * H + h) * DV + col0 + j)
                                   : 0.f;
    };

    packed::stream_init(sm.st);
    if (tid == 0 && nch > 0) {
        packed::stream_fetch(sm.st, 0, sm.part1, rec_of(0), R::PART1_BYTES);
        packed::stream_fetch(sm.st, 1, sm.part2, rec_of(0) + R::PART2, R::PART2_BYTES);
    }
    for (int e = tid; e < DK * NW; e += NT) {
        const int c = e / NW, j = e % NW;
        sm.S[e] = p.s0 ? p.s0[(((size_t)n * H + h) * DK + c) * DV + col0 + j] : 0.f;
    }
    if (nch > 0)
#pragma unroll
        for (int i = 0; i < NVR; ++i) sm.V[tid + i * NT] = v_at(0, tid + i * NT);
    for (int ci = 0; ci < nch; ++ci) {
        const int L = min(C, wk.len - ci * C), tok = wk.tok0 + ci * C;
        if (!packed::stream_wait(sm.st, 0, ci)) goto drain;   // also orders S and V
        // W = (e^{Gx} a) S + A_ak V;  OQ = (e^G q) S
        float w[4][2] = {}, oq[4][2] = {};
        mma_rk<4, 2>(w, AX, DK, sm.S, NW, DK, 4 * tm, 2 * tn);
        mma_rk<4, 2>(w, AAK, C, sm.V, NW, C, 4 * tm, 2 * tn);
        mma_rk<4, 2>(oq, QX, DK, sm.S, NW, DK, 4 * tm, 2 * tn);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 2; ++j) sm.W[(4 * tm + i) * NW + 2 * tn + j] = w[i][j];
        __syncthreads();
        // U = (I - A_ab)^-1 W
        float u[4][2] = {};
        mma_rk<4, 2>(u, TI, C, sm.W, NW, C, 4 * tm, 2 * tn);
        __syncthreads();   // part 1 and W are read
        if (tid == 0 && ci + 1 < nch) packed::stream_fetch(sm.st, 0, sm.part1, rec_of(ci + 1), R::PART1_BYTES);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 2; ++j) sm.W[(4 * tm + i) * NW + 2 * tn + j] = u[i][j];
        if (!packed::stream_wait(sm.st, 1, ci)) goto drain;   // also orders U
        float vn[NVR];   // next chunk's V, in flight during the arithmetic below
#pragma unroll
        for (int i = 0; i < NVR; ++i) vn[i] = ci + 1 < nch ? v_at(ci + 1, tid + i * NT) : 0.f;
        // O = OQ + P_qb U + P_qk V -> rows < L
        mma_rk<4, 2>(oq, PQB, C, sm.W, NW, C, 4 * tm, 2 * tn);
        mma_rk<4, 2>(oq, PQK, C, sm.V, NW, C, 4 * tm, 2 * tn);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = 4 * tm + i;
            if (r < L)
#pragma unroll
                for (int j = 0; j < 2; ++j)
                    Elem<TOut>::store(o + ((size_t)(tok + r) * H + h) * DV + col0 + 2 * tn + j, oq[i][j]);
        }
        // S <- e^{G_last} S + (e^{G_last - G} b)^T U + (e^{G_last - G} k)^T V
        {
            float ds[TK][2] = {};
            mma_tk<TK, 2>(ds, BL, DK, sm.W, NW, C, TK * tm, 2 * tn);
            mma_tk<TK, 2>(ds, KL, DK, sm.V, NW, C, TK * tm, 2 * tn);
#pragma unroll
            for (int i = 0; i < TK; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int c = TK * tm + i, e = c * NW + 2 * tn + j;
                    sm.S[e] = fmaf(gam[c], sm.S[e], ds[i][j]);
                }
        }
        __syncthreads();   // part 2, V and U are read
        if (tid == 0 && ci + 1 < nch)
            packed::stream_fetch(sm.st, 1, sm.part2, rec_of(ci + 1) + R::PART2, R::PART2_BYTES);
#pragma unroll
        for (int i = 0; i < NVR; ++i) sm.V[tid + i * NT] = vn[i];
    }
    __syncthreads();
    if (p.sT)
        for (int e = tid; e < DK * NW; e += NT) {
            const int c = e / NW, j = e % NW;
            p.sT[(((size_t)n * H + h) * DK + c) * DV + col0 + j] = sm.S[e];
        }
    return;
drain:
    packed::stream_drain(sm.st);
}

// ================================================================ host side

struct Ws {
    size_t rec, choff, bytes;
    long long nrec;
};

static size_t al1k(size_t x) { return (x + 1023) & ~(size_t)1023; }

static Ws ws_layout(int nseq, int T, long long tokens, int H, int dk, bool varlen)
{
    Ws w{};
    w.nrec = packed::records(nseq, T, tokens, varlen);
    const size_t recf = dk == 128 ? Rec<128>::FLOATS : Rec<64>::FLOATS;
    w.rec = 0;
    w.choff = al1k((size_t)w.nrec * H * recf * 4);
    w.bytes = w.choff + (varlen ? al1k(((size_t)nseq + 1) * 4) : 0);
    return w;
}

template <typename TIn, typename TOut, int DK>
cudaError_t launch(const void* q, const void* k, const void* v, const void* a, const void* b, void* o, const Params& p,
                   long long nrec, cudaStream_t stream)
{
    const long long walk_ctas = (long long)p.lay.nseq * p.lay.H * (p.DV / NW);
    const long long items = nrec * p.lay.H;
    if (walk_ctas > 0x7fffffffLL || items > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    auto kf = dplr_factor_kernel<TIn, DK>;
    auto kw = dplr_walk_kernel<TIn, TOut, DK>;
    cudaError_t err = cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(FacSmem<DK>));
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(kw, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(WalkSmem<DK>));
    if (err != cudaSuccess) return err;
    if (walk_ctas == 0) return cudaSuccess;
    if (items > 0) {
        kf<<<(unsigned)items, NT, sizeof(FacSmem<DK>), stream>>>(
            static_cast<const TIn*>(q), static_cast<const TIn*>(k), static_cast<const TIn*>(a),
            static_cast<const TIn*>(b), p);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    kw<<<(unsigned)walk_ctas, NT, sizeof(WalkSmem<DK>), stream>>>(static_cast<const TIn*>(v),
                                                                   static_cast<TOut*>(o), p);
    return cudaGetLastError();
}

template <typename TIn, typename TOut>
cudaError_t launch_dk(const void* q, const void* k, const void* v, const void* a, const void* b, void* o,
                      const Params& p, int dk, long long nrec, cudaStream_t s)
{
    if (dk == 128) return launch<TIn, TOut, 128>(q, k, v, a, b, o, p, nrec, s);
    if (dk == 64) return launch<TIn, TOut, 64>(q, k, v, a, b, o, p, nrec, s);
    return cudaErrorInvalidValue;
}

}  // namespace dplr

size_t dplr_fwd_workspace(int nseq, int T, long long tokens, int H, int dk, int dv, bool varlen)
{
    (void)dv;
    return dplr::ws_layout(nseq, T, tokens, H, dk, varlen).bytes;
}

cudaError_t dplr_fwd(const void* q, const void* k, const void* v, const void* a, const void* b, const float* log_alpha,
                     const float* s0, void* o, float* sT, const int32_t* cu, int nseq, int T, long long tokens, int H,
                     int dk, int dv, kda_dtype dtype, kda_dtype o_dtype, void* ws, size_t ws_bytes, cudaStream_t s)
{
    const bool varlen = cu != nullptr;
    const dplr::Ws L = dplr::ws_layout(nseq, T, tokens, H, dk, varlen);
    if (!ws || ws_bytes < L.bytes) return cudaErrorInvalidValue;
    unsigned char* w = static_cast<unsigned char*>(ws);
    int32_t* choff = reinterpret_cast<int32_t*>(w + L.choff);
    dplr::Params p{};
    p.log_alpha = log_alpha;
    p.s0 = s0;
    p.sT = sT;
    p.rec = reinterpret_cast<float*>(w + L.rec);
    p.lay = packed::Layout{cu, varlen ? choff : nullptr, tokens, L.nrec, nseq, T,
                           varlen ? 0 : (T + dplr::C - 1) / dplr::C, H};
    p.DV = dv;
    if (varlen) {
        packed::chunk_offsets_kernel<<<1, 1024, 0, s>>>(cu, nseq, tokens, choff);
        const cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    using bf = __nv_bfloat16;
    if (dtype == KDA_BF16 && o_dtype == KDA_BF16) return dplr::launch_dk<bf, bf>(q, k, v, a, b, o, p, dk, L.nrec, s);
    if (dtype == KDA_BF16) return dplr::launch_dk<bf, float>(q, k, v, a, b, o, p, dk, L.nrec, s);
    if (o_dtype == KDA_BF16) return dplr::launch_dk<float, bf>(q, k, v, a, b, o, p, dk, L.nrec, s);
    return dplr::launch_dk<float, float>(q, k, v, a, b, o, p, dk, L.nrec, s);
}

}  // namespace kda
