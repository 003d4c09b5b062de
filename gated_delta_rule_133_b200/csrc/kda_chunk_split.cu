// Chunkwise-parallel KDA forward in two passes on the sm_100a tensor cores
// (bf16 q/k/v; fp32 gates, state and accumulation).
//
// The chunk algebra is that of the CUDA-core path ("Hybrid Linear Attention
// Architecture: Making LLM Training and Inference More Efficient", section IV;
// "... Technical Deep Dive ...", section 4; "Linear Attention Architecture Deep
// Dive", section 5).  Per chunk of 64 tokens, G = cumsum(log alpha):
//
//   P  = lower-incl((q e^G)(k e^-G)^T)        A = beta strictly-lower((k e^G)(k e^-G)^T)
//   T  = (I + A)^-1                           (UT transform)
//   Z  = (e^(G_last - G) k)^T T   (d_k x 64)  PT = P T   (64 x 64)
//   Qh = e^G q,  Kh = e^G k
//   [O ; X] = [Qh ; Kh] S,   Y = diag(beta) (V - X)
//   S <- diag(e^G_last) S + Z Y,   O += PT Y
//
// Everything above the last two lines depends on the chunk alone, so pass 1
// (chunk_prep_kernel) computes it for every (chunk, head) pair at once, over
// the whole GPU, and stores one operand record per pair.  Pass 2
// (chunk_scan_kernel) is the only sequential part: one CTA per (sequence,
// head, 64 value columns) walks its chunks with two MMA rounds per chunk.
//
// Precision.  The intra-chunk products P and A use the middle row m of the
// chunk as reference, E = exp(G - G_m) and 1/E (each bounded by 32 tokens of
// decay), and run as kind::tf32 MMAs with operands rounded to nearest; T is
// fp32.  Z and PT are kind::f16 MMAs: T, P and k e^(G_last - G) are rounded to
// fp16, which has the tf32 mantissa and holds them (every factor is at most 1).
// The record's operands are fp16 too: every
// factor e^G, e^(G_last - G) is at most 1, so Qh, Kh, Z and PT stay in range,
// and S and Y are rounded to fp16 as the scan's MMA operands (|S|, |Y| must
// stay below 65504).  The scan accumulates in fp32 in TMEM.
#include "kda_chunk.cuh"
#include "kda_tc_util.cuh"

#include <algorithm>
#include <cstring>
#include <mutex>

namespace kda {
namespace split {

using namespace sm100;
using namespace tcu;
using namespace tcu_host;

constexpr int NT = 512;     // threads per CTA (both kernels): four warpgroups
constexpr int NV = 64;      // value columns per scan CTA

// One operand record per (chunk, head), chunk-major (record index = chunk * H
// + head).  Tiles are fp16 in the K-major 128-byte-swizzled layout, so a scan
// CTA copies the record into shared memory with one bulk copy and feeds the
// tiles to the tensor cores as they are.
template <int DK>
struct Rec {
    static constexpr int QK = 0;                  // [128][DK]: rows 0..63 Qh, 64..127 Kh
    static constexpr int Z = DK * 256;            // [DK][64]
    static constexpr int PT = Z + DK * 128;       // [64][64]
    static constexpr int EGL = PT + 8192;         // fp32 [DK]: exp(G_last)
    static constexpr int BETA = EGL + DK * 4;     // fp32 [64]: beta (0 past the chunk end)
    static constexpr int BYTES = BETA + 256;
};
static_assert(Rec<128>::BYTES % 16 == 0 && Rec<64>::BYTES % 16 == 0, "record size must allow bulk copies");
static_assert(Rec<128>::BYTES <= 65536, "record must fit a 64 KB slot");

// Stores 16 consecutive values of one row of a 16-bit SW128 tile as fp16
// (col0 a multiple of 8: two 16-byte chunks).
__device__ __forceinline__ void st_row_h16(unsigned char* tile, int row, int col0, int rows, const float* x)
{
#pragma unroll
    for (int u = 0; u < 2; ++u)
        *reinterpret_cast<uint4*>(tile + swh_off(row, col0 + 8 * u, rows)) =
            make_uint4(pack_f16(x[8 * u], x[8 * u + 1]), pack_f16(x[8 * u + 2], x[8 * u + 3]),
                       pack_f16(x[8 * u + 4], x[8 * u + 5]), pack_f16(x[8 * u + 6], x[8 * u + 7]));
}


// Every thread polls (measured faster than one poller per warp); a CTA-wide
// vote turns any timeout into a common exit.
#define KDA_WAIT_OR_EXIT(bar, bit, parity)                                                   \
    do {                                                                                     \
        const bool ok_ = mbar_wait((bar), (uint32_t)(parity), abort_flag, p.timeout_cycles); \
        if (__syncthreads_or(!ok_)) goto finish;                                             \
        pend &= ~(bit);                                                                      \
    } while (0)

// Cooperative schedule: a prep CTA publishes a finished record (its generic
// stores ordered by a CTA barrier, its bulk stores completed) with a release
// store; a scan CTA's copy thread acquires the flag, with a bounded wait,
// before its bulk copies read the record.
__device__ __forceinline__ void publish(unsigned* flag)
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __threadfence();
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(flag), "r"(1u) : "memory");
}

__device__ __forceinline__ bool wait_ready(const unsigned* flag, volatile int* abort, long long limit_cycles)
{
    const long long t0 = clock64();
    for (uint32_t i = 0;; ++i) {
        unsigned v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
        if (v) {
            asm volatile("fence.proxy.async.global;" ::: "memory");
            return true;
        }
        __nanosleep(32);
        if ((i & 15u) == 15u) {
            if (*abort) return false;
            if (clock64() - t0 > limit_cycles) break;
        }
    }
    *abort = 1;
    flag_timeout();
    return false;
}

// ============================================================== pass 1: prep

// Layer-variant instantiations of the kernels: the plain layer, the two gate
// tiers alone (each with the work it no longer needs removed), and one
// instantiation for every other combination of KDA_MODE_* flags (runtime
// branches).
constexpr int kVarPlain = 0, kVarHeadGate = 1, kVarNoErase = 2, kVarAny = 3;

struct PrepParams {
    const float* beta;
    const int32_t* cu;       // varlen boundaries, or nullptr (dense)
    const int32_t* choff;    // varlen: first chunk of each sequence, [nseq + 1]
    unsigned char* rec;
    int nseq, T, H, nch;     // dense: nch chunks per sequence
    int c_begin, cbs;        // dense: this launch covers chunks [c_begin, c_begin + cbs) of every sequence
    int rs, rc0;             // dense: record of (n, c, h) = (n * rs + c - rc0) * H + h
    long long nitems;        // (chunk, head) items of this launch
    long long tokens;
    long long timeout_cycles;
    unsigned* ready;         // cooperative schedule: ready[record] = 1 once the record is complete
    const float* gh;         // one gate per (token, head), [tokens, H] (KDA_MODE_HEAD_GATE), or nullptr
    int no_erase;            // KDA_MODE_NO_ERASE: A = 0, so T = I
    int norm_qk;             // KDA_MODE_NORM_QK: q, k rows divided by their L2 norms in the build
    int logits;              // KDA_MODE_GATE_LOGITS: gates are logits z, log alpha = -softplus(z)
};

struct Item {
    long long rec;           // record index: global chunk * H + head
    int tok0, L, h;
    bool ok;
};

__device__ __forceinline__ Item resolve(const PrepParams& p, long long item)
{
    Item it{0, 0, 0, 0, false};
    if (item >= p.nitems) return it;
    long long j;
    if (p.nitems <= 0xffffffffll) {   // 32-bit divisions (a fraction of the 64-bit routine's cost)
        const uint32_t i32 = (uint32_t)item, q = i32 / (uint32_t)p.H;
        it.h = (int)(i32 - q * (uint32_t)p.H);
        j = q;
    } else {
        it.h = (int)(item % p.H);
        j = item / p.H;
    }
    it.rec = item;
    if (p.cu) {
        if (j >= p.choff[p.nseq]) return it;
        int lo = 0, hi = p.nseq - 1;           // last sequence whose first chunk is <= j
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.choff[mid] <= j) lo = mid;
            else hi = mid - 1;
        }
        it.tok0 = p.cu[lo] + (int)(j - p.choff[lo]) * C;
        it.L = min(C, p.cu[lo + 1] - it.tok0);
    } else {   // chunk outermost, then sequence: the scans of all sequences advance together
        int n, c;
        if (p.nitems <= 0xffffffffll) {
            const uint32_t j32 = (uint32_t)j, jq = j32 / (uint32_t)p.nseq;
            n = (int)(j32 - jq * (uint32_t)p.nseq);
            c = p.c_begin + (int)jq;
        } else {
            n = (int)(j % p.nseq);
            c = p.c_begin + (int)(j / p.nseq);
        }
        it.tok0 = n * p.T + c * C;
        it.L = min(C, p.T - c * C);
        it.rec = ((long long)n * p.rs + c - p.rc0) * p.H + it.h;
    }
    it.ok = it.L > 0 && it.tok0 >= 0 && it.tok0 + it.L <= p.tokens;
    return it;
}

constexpr int LDT = 68;     // row stride (floats) of the UT matrix: 16-byte rows, conflict-free quads

// Shared memory of the prep kernel (byte offsets from a 1024-aligned base).
//   A1: [q E; k E] (tf32, [128][d_k]) of the item being built.
//   B1: k / E (tf32, [64][d_k]).
//   STG: TMA staging of q, k (bf16) and log alpha (fp32 -> G in place).
//   TOP: T^T [64][64] (fp16 B operand of MMAs Z, PT; entries below its
//        diagonal stay zero), then the UT product scratch XS.
//   AS: A, then T in place (fp32, row-major, row stride LDT).
//   VEC: per item (double-buffered): G_m, e^G_m, e^(G_last - G_m), e^G_last,
//        partial sums, beta.
//   TST: staging of the previous item's record tail (Z, PT, e^G_last, beta),
//        which one bulk store copies out.
struct PrepPlan {
    static constexpr int A1 = 0;
    static constexpr int B1 = 65536;
    static constexpr int STG = 98304;
    static constexpr int TOP = 163840;
    static constexpr int XS = TOP + 8192;
    static constexpr int AS = TOP + 16384;
    static constexpr int VEC = AS + C * LDT * 4;
    static constexpr int VECN = 7 * 128 + 64;
    static constexpr int TST = VEC + 2 * VECN * 4;
    static constexpr int TST_BYTES = 25344;
    static constexpr int BAR = TST + TST_BYTES;
    static constexpr int END = BAR + 128;
    static constexpr int BYTES = END + 1024;
};
static_assert(PrepPlan::BYTES <= 232448, "prep shared memory exceeds the per-CTA limit");
static_assert(Rec<128>::BYTES - Rec<128>::Z <= PrepPlan::TST_BYTES, "record tail staging too small");
static_assert(32 * 36 * 4 <= 8192, "UT scratch must fit behind the T^T tile");

template <int DK>
struct PrepCtx {
    const __nv_bfloat16* qs;
    const __nv_bfloat16* ks;
    float* gs;
    unsigned char* A1;
    unsigned char* B1;
};

// Channel vectors of one item buffer.
struct Vec {
    float* gml;    // G_m
    float* gm;     // e^G_m
    float* glm;    // e^(G_last - G_m)
    float* egl;    // e^G_last
    float* qtot;   // partial sums [3][128]
    float* beta;   // [64]
};
__device__ __forceinline__ Vec vec_at(unsigned char* base, int buf)
{
    float* f = reinterpret_cast<float*>(base) + buf * PrepPlan::VECN;
    return Vec{f, f + 128, f + 256, f + 384, f + 512, f + 896};
}

// Gate cumsum of the staged chunk in place, by 384 threads (t = 0..383:
// key channel t % 128, rows [21 p, 21 p + 21) of part p = t / 128, the last
// part 22 rows), and the item's channel vectors.  Named barrier 2.
//
// gate_v is the gate of row t (t < 64) when gates are per (token, head), read
// by the caller ahead of the wait for the tile.
template <int DK>
__device__ __forceinline__ void cumsum384(float* gs, const Vec& v, int L, int t, float beta_v,
                                          bool gh, float gate_v, bool logits)
{
    const int ch = t & 127, part = t >> 7;
    const int r0 = 21 * part, nr = part == 2 ? 22 : 21;
    if (gh) {   // one gate per (token, head): column 0 of the staging holds the chunk's 64 gates
        if (t < C) gs[t * DK] = (logits && t < L) ? neg_softplus(gate_v) : gate_v;
        bar_sync(2, 384);
    }
    float G[22];
    if (ch < DK) {
#pragma unroll
        for (int rr = 0; rr < 22; ++rr) {
            const int row = r0 + rr;
            G[rr] = (rr < nr && row < L) ? gs[row * DK + (gh ? 0 : ch)] : 0.f;
            if (logits && !gh && rr < nr && row < L) G[rr] = neg_softplus(G[rr]);
        }
#pragma unroll
        for (int rr = 1; rr < 22; ++rr) G[rr] += G[rr - 1];
        v.qtot[part * 128 + ch] = G[nr - 1];
    }
    if (t < C) v.beta[t] = beta_v;
    bar_sync(2, 384);
    if (ch < DK) {
        float off = 0.f;
        for (int q = 0; q < part; ++q) off += v.qtot[q * 128 + ch];
#pragma unroll
        for (int rr = 0; rr < 22; ++rr)
            if (rr < nr) gs[(r0 + rr) * DK + ch] = G[rr] + off;
        if (part == 1) {
            const float Gm = off + G[31 - 21];
            const float Gl = v.qtot[ch] + v.qtot[128 + ch] + v.qtot[256 + ch];
            v.gml[ch] = Gm;
            v.gm[ch] = expf(Gm);
            v.glm[ch] = expf(Gl - Gm);
            v.egl[ch] = expf(Gl);
        }
    }
    bar_sync(2, 384);
    if (part == 0 && ch < DK) check_domain(gs[ch], v.gml[ch], gs[(C - 1) * DK + ch]);
}

// Gate cumsum of one gate per (token, head), by 384 threads (named barrier 2):
// column 0 of the staging receives G and every key channel gets the same
// channel vectors.  Three lanes run the three row parts of cumsum384 for one
// channel, additions in the same order, so the result is bit-identical to the
// per-channel path fed the same gate on every channel.
template <int DK>
__device__ __forceinline__ void cumsum_head384(float* gs, const Vec& v, int L, int t, float beta_v, float gate_v)
{
    if (t < C) {
        gs[t * DK] = t < L ? gate_v : 0.f;
        v.beta[t] = beta_v;
    }
    bar_sync(2, 384);
    float G[22];
    const int r0 = 21 * t, nr = t == 2 ? 22 : 21;
    if (t < 3) {
#pragma unroll
        for (int rr = 0; rr < 22; ++rr) G[rr] = rr < nr ? gs[(r0 + rr) * DK] : 0.f;
#pragma unroll
        for (int rr = 1; rr < 22; ++rr) G[rr] += G[rr - 1];
        v.qtot[t * 128] = G[nr - 1];
    }
    bar_sync(2, 384);
    if (t < 3) {
        float off = 0.f;
        for (int q = 0; q < t; ++q) off += v.qtot[q * 128];
#pragma unroll
        for (int rr = 0; rr < 22; ++rr)
            if (rr < nr) gs[(r0 + rr) * DK] = G[rr] + off;
        if (t == 1) v.qtot[1] = off + G[31 - 21];   // G_m (slot 1 of part 0 is free)
    }
    bar_sync(2, 384);
    if (t < DK) {
        const float Gm = v.qtot[1];
        const float Gl = v.qtot[0] + v.qtot[128] + v.qtot[256];
        v.gml[t] = Gm;
        v.gm[t] = expf(Gm);
        v.glm[t] = expf(Gl - Gm);
        v.egl[t] = expf(Gl);
        if (t == 0) check_domain(gs[0], Gm, Gl);
    }
    bar_sync(2, 384);
}

// Operands of rows [row_lo, row_hi) of one item, by `nthr` threads (t = 0..nthr-1): A1 = [q E; k E]
// and B1 = k / E (tf32, smem) for the intra-chunk products; Qh = q e^G and
// Kh = k e^G (fp16) straight into the record.
//
// HG: one gate per (token, head): G is read from column 0 and every channel of
// a row shares one exponential and one reciprocal.
template <int DK, bool HG = false>
__device__ __forceinline__ void build_operands(const PrepCtx<DK>& x, const Vec& v, unsigned char* rec, int L, int t,
                                               int nthr, int row_lo, int row_hi, bool norm_qk = false)
{
    using R = Rec<DK>;
    constexpr int NG = DK / 4;
    const int rpp = nthr / NG;
    const int r0 = t / NG, c0 = (t % NG) * 4;
    const float4 m4 = *reinterpret_cast<const float4*>(v.gml + c0);
    const float4 gm4 = *reinterpret_cast<const float4*>(v.gm + c0);
#pragma unroll 2
    for (int r = row_lo + r0; r < row_hi; r += rpp) {
        const float4 g4 = HG ? make_float4(x.gs[r * DK], 0.f, 0.f, 0.f)
                             : *reinterpret_cast<const float4*>(x.gs + r * DK + c0);
        float4 q4 = make_float4(0.f, 0.f, 0.f, 0.f), k4 = q4;
        if (r < L) {
            q4 = bf16x4(x.qs + r * DK + c0);
            k4 = bf16x4(x.ks + r * DK + c0);
        }
        if (norm_qk) {   // the NG lanes holding row r are consecutive, and every lane runs the same rows
            float sq = q4.x * q4.x + q4.y * q4.y + q4.z * q4.z + q4.w * q4.w;
            float sk = k4.x * k4.x + k4.y * k4.y + k4.z * k4.z + k4.w * k4.w;
#pragma unroll
            for (int o = NG / 2; o > 0; o >>= 1) {
                sq += __shfl_xor_sync(0xffffffffu, sq, o);
                sk += __shfl_xor_sync(0xffffffffu, sk, o);
            }
            const float iq = inv_norm(sq), ik = inv_norm(sk);
            q4 = make_float4(q4.x * iq, q4.y * iq, q4.z * iq, q4.w * iq);
            k4 = make_float4(k4.x * ik, k4.y * ik, k4.z * ik, k4.w * ik);
        }
        float e0, e1, e2, e3, i0, i1, i2, i3;
        if (HG) {
            e0 = e1 = e2 = e3 = __expf(fminf(fmaxf(g4.x - m4.x, -80.f), 80.f));
            i0 = i1 = i2 = i3 = rcp_approx(e0);
        } else {
            e0 = __expf(fminf(fmaxf(g4.x - m4.x, -80.f), 80.f));
            e1 = __expf(fminf(fmaxf(g4.y - m4.y, -80.f), 80.f));
            e2 = __expf(fminf(fmaxf(g4.z - m4.z, -80.f), 80.f));
            e3 = __expf(fminf(fmaxf(g4.w - m4.w, -80.f), 80.f));
            i0 = rcp_approx(e0);
            i1 = rcp_approx(e1);
            i2 = rcp_approx(e2);
            i3 = rcp_approx(e3);
        }
        *reinterpret_cast<float4*>(x.A1 + swf_off(r, c0, 128)) = tf32r4(q4.x * e0, q4.y * e1, q4.z * e2, q4.w * e3);
        *reinterpret_cast<float4*>(x.A1 + swf_off(C + r, c0, 128)) = tf32r4(k4.x * e0, k4.y * e1, k4.z * e2, k4.w * e3);
        *reinterpret_cast<float4*>(x.B1 + swf_off(r, c0, 64)) =
            tf32r4(k4.x * i0, k4.y * i1, k4.z * i2, k4.w * i3);
        const float f0 = e0 * gm4.x, f1 = e1 * gm4.y, f2 = e2 * gm4.z, f3 = e3 * gm4.w;
        *reinterpret_cast<uint2*>(rec + R::QK + swh_off(r, c0, 128)) =
            make_uint2(pack_f16(q4.x * f0, q4.y * f1), pack_f16(q4.z * f2, q4.w * f3));
        *reinterpret_cast<uint2*>(rec + R::QK + swh_off(C + r, c0, 128)) =
            make_uint2(pack_f16(k4.x * f0, k4.y * f1), pack_f16(k4.z * f2, k4.w * f3));
    }
}

// d += s * b for two float4 accumulators, as four packed fp32x2 FMAs (each
// lane rounds exactly as fmaf does).
__device__ __forceinline__ void fma_s8(float4& d0, float4& d1, float s, const float4& b0, const float4& b1)
{
    asm("{\n\t.reg .b64 ss, bb, dd;\n\t"
        "mov.b64 ss, {%8, %8};\n\t"
        "mov.b64 bb, {%9, %10};\n\tmov.b64 dd, {%0, %1};\n\tfma.rn.f32x2 dd, ss, bb, dd;\n\tmov.b64 {%0, %1}, dd;\n\t"
        "mov.b64 bb, {%11, %12};\n\tmov.b64 dd, {%2, %3};\n\tfma.rn.f32x2 dd, ss, bb, dd;\n\tmov.b64 {%2, %3}, dd;\n\t"
        "mov.b64 bb, {%13, %14};\n\tmov.b64 dd, {%4, %5};\n\tfma.rn.f32x2 dd, ss, bb, dd;\n\tmov.b64 {%4, %5}, dd;\n\t"
        "mov.b64 bb, {%15, %16};\n\tmov.b64 dd, {%6, %7};\n\tfma.rn.f32x2 dd, ss, bb, dd;\n\tmov.b64 {%6, %7}, dd;\n\t}"
        : "+f"(d0.x), "+f"(d0.y), "+f"(d0.z), "+f"(d0.w), "+f"(d1.x), "+f"(d1.y), "+f"(d1.z), "+f"(d1.w)
        : "f"(s), "f"(b0.x), "f"(b0.y), "f"(b0.z), "f"(b0.w), "f"(b1.x), "f"(b1.y), "f"(b1.z), "f"(b1.w));
}
__device__ __forceinline__ void fma_s4(float4& d, float s, const float4& b)
{
    asm("{\n\t.reg .b64 ss, bb, dd;\n\t"
        "mov.b64 ss, {%4, %4};\n\t"
        "mov.b64 bb, {%5, %6};\n\tmov.b64 dd, {%0, %1};\n\tfma.rn.f32x2 dd, ss, bb, dd;\n\tmov.b64 {%0, %1}, dd;\n\t"
        "mov.b64 bb, {%7, %8};\n\tmov.b64 dd, {%2, %3};\n\tfma.rn.f32x2 dd, ss, bb, dd;\n\tmov.b64 {%2, %3}, dd;\n\t}"
        : "+f"(d.x), "+f"(d.y), "+f"(d.z), "+f"(d.w)
        : "f"(s), "f"(b.x), "f"(b.y), "f"(b.z), "f"(b.w));
}
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 neg4(const float4& a) { return make_float4(-a.x, -a.y, -a.z, -a.w); }
__device__ __forceinline__ float f4at(const float4& a, int u) { return u == 0 ? a.x : u == 1 ? a.y : u == 2 ? a.z : a.w; }

// UT transform T = (I + A)^-1 of the strictly lower 64 x 64 A, by the first
// 128 threads (named barrier 1).  On entry As[r * LDT + s] holds A[r][s] (zero
// for s >= r).  T^T goes to Top (fp16, K-major 128-byte swizzle: row j =
// column j of T) as each block of T is final; the entries of Top below its
// diagonal are never written (they hold zeros).  As keeps the blocks of T that
// later steps read (T[r][r] = 1, zero above the diagonal).  Diagonal 16 x 16 blocks by forward substitution (one lane per
// column), then T10 = -T11 A10 T00 and T32 = -T33 A32 T22, then the lower-left
// 32 x 32 block -T_BB A_BA T_AA.  Every sum runs in ascending index order
// (terms that the triangular factors make zero are skipped where a whole warp
// can skip them); X is the product scratch.
__device__ __forceinline__ void ut_rows(float* As, float* X, unsigned char* Top)
{
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid < 64) {
        const int b0 = 16 * (tid >> 4), j = tid & 15;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = 0.f;
        x[0] = j == 0 ? 1.f : 0.f;
#pragma unroll
        for (int r = 1; r < 16; ++r) {
            float acc = (r == j) ? 1.f : 0.f;
#pragma unroll
            for (int q = 0; 4 * q < r; ++q) {   // A[r][s] = 0 and x[s] = 0 for s >= r
                const float4 a = ld4(As + (b0 + r) * LDT + b0 + 4 * q);
                acc = fmaf(-a.x, x[4 * q], acc);
                acc = fmaf(-a.y, x[4 * q + 1], acc);
                acc = fmaf(-a.z, x[4 * q + 2], acc);
                acc = fmaf(-a.w, x[4 * q + 3], acc);
            }
            x[r] = acc;
        }
        __syncwarp();   // every lane has read its A block before T overwrites it
#pragma unroll
        for (int r = 0; r < 16; ++r)
            if (r >= j) As[(b0 + r) * LDT + b0 + j] = x[r];
        st_row_h16(Top, b0 + j, b0, C, x);   // x[r] = 0 for r < j
    }
    bar_sync(1, 128);
    {   // T10 (warps 0, 1) and T32 (warps 2, 3): lane -> row i, columns j0 .. j0 + 3
        const int pr = warp >> 1, half = warp & 1;
        const int rb = 16 + 32 * pr, cb = 32 * pr;
        const int i = lane & 15, j0 = 8 * half + 4 * (lane >> 4);
        float* Xp = X + pr * 16 * 20;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int q = 2 * half; q < 4; ++q) {   // T_cc[t][j] = 0 for t < j
            const float4 a = ld4(As + (rb + i) * LDT + cb + 4 * q);
#pragma unroll
            for (int u = 0; u < 4; ++u) fma_s4(acc, f4at(a, u), ld4(As + (cb + 4 * q + u) * LDT + cb + j0));
        }
        *reinterpret_cast<float4*>(Xp + i * 20 + j0) = acc;
        bar_sync(1, 128);
        acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 t = ld4(As + (rb + i) * LDT + rb + 4 * q);
#pragma unroll
            for (int u = 0; u < 4; ++u) fma_s4(acc, f4at(t, u), ld4(Xp + (4 * q + u) * 20 + j0));
        }
        const float4 t4 = neg4(acc);
        *reinterpret_cast<float4*>(As + (rb + i) * LDT + cb + j0) = t4;
#pragma unroll
        for (int u = 0; u < 4; ++u) *reinterpret_cast<__half*>(Top + swh_off(cb + j0 + u, rb + i, C)) = __float2half_rn(f4at(t4, u));
    }
    bar_sync(1, 128);
    {   // lower-left 32 x 32: lane -> row i (0..31), warp -> columns c0 .. c0 + 7
        const int i = lane, c0 = 8 * warp;
        float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
        for (int q = 2 * warp; q < 8; ++q) {   // T_AA[t][c] = 0 for t < c0 <= c
            const float4 a = ld4(As + (32 + i) * LDT + 4 * q);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float* tr = As + (4 * q + u) * LDT + c0;
                fma_s8(a0, a1, f4at(a, u), ld4(tr), ld4(tr + 4));
            }
        }
        *reinterpret_cast<float4*>(X + i * 36 + c0) = a0;
        *reinterpret_cast<float4*>(X + i * 36 + c0 + 4) = a1;
        bar_sync(1, 128);
        a0 = make_float4(0.f, 0.f, 0.f, 0.f);
        a1 = a0;
#pragma unroll 2
        for (int q = 0; q < 8; ++q) {
            const float4 t = ld4(As + (32 + i) * LDT + 32 + 4 * q);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float* xr = X + (4 * q + u) * 36 + c0;
                fma_s8(a0, a1, f4at(t, u), ld4(xr), ld4(xr + 4));
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            *reinterpret_cast<__half*>(Top + swh_off(c0 + u, 32 + i, C)) = __float2half_rn(-f4at(a0, u));
            *reinterpret_cast<__half*>(Top + swh_off(c0 + 4 + u, 32 + i, C)) = __float2half_rn(-f4at(a1, u));
        }
    }
}

// One persistent CTA per SM walks items blockIdx.x, + gridDim.x, ...  The
// UT transform of item k (warpgroup 0) overlaps the gate cumsum and operand
// build of item k + 1 (warpgroups 1-3); one MMA round then forms Z, PT of
// item k and [P ; A~] of item k + 1.
//
//   prologue: load, cumsum, build, MMA PA of item 0; P/A split of item 0
//   loop k:   WG0: UT(k), T^T tile      | WG1-3: cumsum + build of item k + 1
//             MMA Z(k), PT(k) (kind::f16), PA(k + 1) (kind::tf32)
//             record tail of item k (staged in TST, one bulk store); P/A split of k + 1
//
// Without the erase term A = 0 and T = I: the T^T tile is the identity from
// the start, no UT transform runs, and warpgroup 0 joins the build.
//
// TMEM: [P ; A~] double-buffered (0, 64); the fp16 A operands of Z and PT,
// k e^(G_last - G) transposed (128) and masked P (160), two per 32-bit column;
// Z 192, PT 256.
template <int DK, int VK>
__device__ __forceinline__ void prep_body(const CUtensorMap& tmq, const CUtensorMap& tmk, const CUtensorMap& tmg,
                                          const PrepParams& p, int bid, int nblk)
{
    // layer variants: kVarHeadGate and kVarNoErase fix one flag at compile
    // time; kVarAny reads every flag at run time
    constexpr bool kHG = VK == kVarHeadGate;   // per-head gates only
    constexpr bool kNE = VK == kVarNoErase;    // no erase term only
    const float* const gh = (kHG || VK == kVarAny) ? p.gh : nullptr;
    const bool no_erase = kNE || (VK == kVarAny && p.no_erase);
    const bool norm_qk = VK == kVarAny && p.norm_qk;
    const bool logits = VK == kVarAny && p.logits;
    using PL = PrepPlan;
    using R = Rec<DK>;
    extern __shared__ unsigned char smem_raw[];
    KDA_PHASE_DECL(0)
    unsigned char* sm = align1024(smem_raw);
    PrepCtx<DK> x;
    x.A1 = sm + PL::A1;
    x.B1 = sm + PL::B1;
    x.qs = reinterpret_cast<const __nv_bfloat16*>(sm + PL::STG);
    x.ks = x.qs + C * DK;
    x.gs = reinterpret_cast<float*>(sm + PL::STG + 2 * C * DK * 2);
    unsigned char* Top = sm + PL::TOP;
    float* As = reinterpret_cast<float*>(sm + PL::AS);
    float* Xs = reinterpret_cast<float*>(sm + PL::XS);
    unsigned char* vbase = sm + PL::VEC;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + PL::BAR);
    uint64_t* mb_tma = bars + 0;
    uint64_t* mb_mma = bars + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int lt = tid & 127;
    const int wg = tid >> 7;
    const int H = p.H;
    constexpr int kStoreIssuer = 128;   // first thread of warpgroup 1

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) mbar_init(bars + i, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async();
        prefetch_tmap(&tmq);
        prefetch_tmap(&tmk);
        if (!gh) prefetch_tmap(&tmg);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_off = ((uint32_t)(warp & 3) * 32) << 16;
    const uint32_t q_off = (uint32_t)wg * 16;
    const uint32_t t_K16 = tmem + 128, t_P16 = tmem + 160, t_Z = tmem + 192, t_PT = tmem + 256;
    constexpr uint32_t kH64 = idesc_f16(128, 64);

    constexpr uint32_t kStageBytes = (uint32_t)C * DK * (2 + 2 + 4);
    constexpr uint32_t kI64 = idesc_tf32(128, 64, 0, 0);
    constexpr int kR128 = 128 * 128, kR64 = 64 * 128;

    unsigned pend = 0;                 // bit 0: TMA load outstanding, bit 1: MMA commit outstanding
    int tpar = 0;                      // parity of the outstanding TMA load
    int nload = 0, nmma = 0;           // loads / commits issued so far
    bool stored = false;               // the store issuer has bulk stores in flight
    bool unpublished = false;
    long long stored_rec = 0;

    auto load_item = [&](const Item& it) {   // one thread; per-head gates are read by the cumsum
        mbar_expect_tx(mb_tma, gh ? (uint32_t)C * DK * 4 : kStageBytes);
        tma_load_3d((void*)x.qs, &tmq, mb_tma, 0, it.h, it.tok0);
        tma_load_3d((void*)x.ks, &tmk, mb_tma, 0, it.h, it.tok0);
        if (!gh) tma_load_3d((void*)x.gs, &tmg, mb_tma, 0, it.h, it.tok0);
    };
    auto beta_of = [&](const Item& it, int t) {
        return (it.ok && t < C && t < it.L) ? p.beta[(size_t)(it.tok0 + t) * H + it.h] : 0.f;
    };
    auto gate_of = [&](const Item& it, int t) {   // per-head gate of row t (0 past the chunk)
        return (gh && it.ok && t < C && t < it.L) ? gh[(size_t)(it.tok0 + t) * H + it.h] : 0.f;
    };
    auto cumsum = [&](const Vec& v, const Item& it, int t, float beta_v, float gate_v) {
        if (kHG) cumsum_head384<DK>(x.gs, v, it.L, t, beta_v, gate_v);
        else cumsum384<DK>(x.gs, v, it.L, t, beta_v, gh != nullptr, gate_v, logits);
    };
    // P masked (lanes 0..63, lower incl.) into the fp16 operand of PT; A = beta
    // A~ (lanes 64..127, strictly lower) to the UT scratch; (k / E)^T
    // e^(G_last - G_m) = (k e^(G_last - G))^T into the fp16 operand of Z
    auto split_pa = [&](uint32_t t_PA, const Vec& v) {
        float pa[16];
        tmem_ld16(t_PA + lane_off + q_off, pa);
        tmem_wait_ld();
        if (lt < C) {   // P, lower incl., packed fp16 (warps of lanes 0..63)
            uint32_t p16[8];
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2)
                p16[s2] = pack_f16((16 * wg + 2 * s2 <= lt) ? pa[2 * s2] : 0.f, (16 * wg + 2 * s2 + 1 <= lt) ? pa[2 * s2 + 1] : 0.f);
            tmem_st8(t_P16 + lane_off + wg * 8, p16);
        } else if (!kNE) {
            const int r = lt - C;
            const float b = v.beta[r];
            float a[16];
#pragma unroll
            for (int s2 = 0; s2 < 16; ++s2) a[s2] = (!no_erase && 16 * wg + s2 < r) ? b * pa[s2] : 0.f;
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4)
                *reinterpret_cast<float4*>(As + r * LDT + 16 * wg + 4 * s4) =
                    make_float4(a[4 * s4], a[4 * s4 + 1], a[4 * s4 + 2], a[4 * s4 + 3]);
        }
        const float gl = lt < DK ? v.glm[lt] : 0.f;   // k e^(G_last - G) = (k / E) e^(G_last - G_m)
        uint32_t kb[8];
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2)
            kb[s2] = lt < DK ? pack_f16(swf(x.B1, 16 * wg + 2 * s2, lt, 64) * gl, swf(x.B1, 16 * wg + 2 * s2 + 1, lt, 64) * gl) : 0u;
        tmem_st8(t_K16 + lane_off + wg * 8, kb);
        tmem_wait_st();
    };

    long long item = bid;
    Item cur = resolve(p, item);
    Item nxt{0, 0, 0, 0, false};
    int k = 0;
    if (!cur.ok) goto finish;

    // ---- prologue: item 0 by all threads
    for (int i = tid; i < C * C * 2 / 16; i += NT) reinterpret_cast<uint4*>(Top)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (kNE) {   // T = I for good
        __syncthreads();
        if (tid < C) *reinterpret_cast<__half*>(Top + swh_off(tid, tid, C)) = __float2half_rn(1.f);
    }
    if (tid == 0) load_item(cur);
    ++nload;
    pend |= 1u;
    tpar = 0;
    {
        const float beta_v = tid >= 128 ? beta_of(cur, tid - 128) : 0.f;
        const float gate_v = tid >= 128 ? gate_of(cur, tid - 128) : 0.f;
        KDA_WAIT_OR_EXIT(mb_tma, 1u, 0);
        if (tid >= 128) cumsum(vec_at(vbase, 0), cur, tid - 128, beta_v, gate_v);
        __syncthreads();
        build_operands<DK, kHG>(x, vec_at(vbase, 0), p.rec + (size_t)cur.rec * R::BYTES, cur.L, tid, NT, 0, C, norm_qk);
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    nxt = resolve(p, item + nblk);
    if (tid == 32 && nxt.ok) load_item(nxt);
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < DK / 8; ++kk)
            umma_tf32(tmem, kdesc(x.A1, kk, kR128), kdesc(x.B1, kk, kR64), kI64, kk > 0);
        umma_commit(mb_mma);
    }
    if (nxt.ok) {
        pend |= 1u;
        tpar = nload & 1;
        ++nload;
    }
    pend |= 2u;
    KDA_WAIT_OR_EXIT(mb_mma, 2u, 0);
    ++nmma;
    tc_fence_after();
    split_pa(tmem, vec_at(vbase, 0));
    tc_fence_before();
    __syncthreads();

    for (k = 0;; ++k) {
        const int vb = k & 1, nb = vb ^ 1;
        const Vec vcur = vec_at(vbase, vb), vnxt = vec_at(vbase, nb);
        const uint32_t t_PAn = tmem + 64 * nb;
        const long long nitem = item + nblk;
        KDA_PHASE(0);

        // ---- UT transform of item k (WG0) | cumsum + operands of item k + 1 (WG1-3)
        if (kNE) {   // no UT transform: all four warpgroups build
            if (nxt.ok) {
                const int t = tid - 128;
                const float beta_v = wg ? beta_of(nxt, t) : 0.f;
                const bool ok = mbar_wait(mb_tma, (uint32_t)tpar, abort_flag, p.timeout_cycles);
                if (!__syncthreads_or(!ok)) {
                    if (wg) cumsum(vnxt, nxt, t, beta_v, 0.f);
                    __syncthreads();
                    build_operands<DK>(x, vnxt, p.rec + (size_t)nxt.rec * R::BYTES, nxt.L, tid, NT, 0, C, false);
                }
            }
        } else if (wg == 0) {
            ut_rows(As, Xs, Top);
        } else {
            if (nxt.ok) {
                const int t = tid - 128;
                const float beta_v = beta_of(nxt, t);
                const float gate_v = gate_of(nxt, t);
                const bool ok = mbar_wait(mb_tma, (uint32_t)tpar, abort_flag, p.timeout_cycles);
                if (!bar_or(3, 384, !ok)) {
                    cumsum(vnxt, nxt, t, beta_v, gate_v);
                    build_operands<DK, kHG>(x, vnxt, p.rec + (size_t)nxt.rec * R::BYTES, nxt.L, t, 384, 0, C, norm_qk);
                }
            }
        }
        fence_proxy_async();
        tc_fence_before();
        if (__syncthreads_or(*abort_flag)) goto finish;
        if (nxt.ok) pend &= ~1u;
        if (p.ready && tid == kStoreIssuer && unpublished) {
            bulk_wait_all();
            publish(p.ready + stored_rec);
            unpublished = false;
        }
        KDA_PHASE(1);

        // ---- MMA round: Z(k) = (k e^(G_last - G))^T T, PT(k) = P T; [P ; A~](k + 1) = A1 B1^T
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                umma_f16_ts(t_Z, t_K16 + 8 * kk, kdesc(Top, kk, kR64), kH64, kk > 0);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                umma_f16_ts(t_PT, t_P16 + 8 * kk, kdesc(Top, kk, kR64), kH64, kk > 0);
            if (nxt.ok) {
#pragma unroll
                for (int kk = 0; kk < DK / 8; ++kk)
                    umma_tf32(t_PAn, kdesc(x.A1, kk, kR128), kdesc(x.B1, kk, kR64), kI64, kk > 0);
            }
            umma_commit(mb_mma);
        }
        const Item nn = nxt.ok ? resolve(p, nitem + nblk) : Item{0, 0, 0, 0, false};
        pend |= 2u;
        // the staging area is rewritten below: the previous tail's bulk store
        // (issued an iteration ago) must have read it
        if (tid == kStoreIssuer && stored) bulk_wait_read();
        KDA_WAIT_OR_EXIT(mb_mma, 2u, nmma & 1);
        // the next load lands in shared memory only now: a TMA copy arriving
        // while the MMAs read their operands slows the round by ~30 %
        if (tid == 32 && nn.ok) load_item(nn);
        if (nn.ok) {
            pend |= 1u;
            tpar = nload & 1;
            ++nload;
        }
        ++nmma;
        tc_fence_after();
        KDA_PHASE(2);

        // ---- record tail of item k, staged in TST: Z, PT, e^G_last, beta
        {
            unsigned char* stg = sm + PL::TST;
            float z[16];
            tmem_ld16(t_Z + lane_off + q_off, z);
            float pt[16];
            tmem_ld16(t_PT + lane_off + q_off, pt);
            tmem_wait_ld();
            if (lt < DK) st_row_h16(stg, lt, 16 * wg, DK, z);
            if (lt < C) st_row_h16(stg + (R::PT - R::Z), lt, 16 * wg, C, pt);
            if (tid < DK) reinterpret_cast<float*>(stg + (R::EGL - R::Z))[tid] = vcur.egl[tid];
            else if (tid >= 256 && tid < 256 + C) reinterpret_cast<float*>(stg + (R::BETA - R::Z))[tid - 256] = vcur.beta[tid - 256];
        }
        // ---- P/A split of item k + 1
        if (nxt.ok) split_pa(t_PAn, vnxt);
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == kStoreIssuer) {
            bulk_store(p.rec + (size_t)cur.rec * R::BYTES + R::Z, sm + PL::TST, (uint32_t)(R::BYTES - R::Z));
            bulk_commit();
            stored = true;
            unpublished = true;
            stored_rec = cur.rec;
        }
        KDA_PHASE(3);
        if (!nxt.ok) break;
        item = nitem;
        cur = nxt;
        nxt = nn;
    }

finish:
    KDA_PHASE_FLUSH
    if (*abort_flag) {
        volatile int never = 0;
        if (pend & 1u) (void)mbar_wait(mb_tma, (uint32_t)tpar, &never, p.timeout_cycles);
        if (pend & 2u) (void)mbar_wait(mb_mma, (uint32_t)(nmma & 1), &never, p.timeout_cycles);
    }
    if (tid == kStoreIssuer && stored) {
        bulk_wait_all();
        if (p.ready && unpublished && !*abort_flag) publish(p.ready + stored_rec);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ============================================================== pass 2: scan

struct ScanParams {
    const __nv_bfloat16* v;
    const float* s_in;       // state before chunk c_begin (nullptr: zeros)
    void* o;
    float* s_out;            // state after this launch's last chunk (nullptr: not stored)
    int c_begin, c_end;      // chunk range of this launch (per sequence)
    const int32_t* cu;
    const int32_t* choff;
    const int32_t* order;    // varlen: sequence of each scan rank (longest first)
    const unsigned char* rec;
    int nseq, T, H, DV, nch;
    int rs, rc0;             // dense: record of (n, c, h) = (n * rs + c - rc0) * H + h
    long long max_chunks;    // records available per head
    long long tokens;
    long long timeout_cycles;
    const unsigned* ready;   // cooperative schedule: wait for ready[record] before loading it
    int no_erase;            // KDA_MODE_NO_ERASE: Y = beta V (no X term)
    int items;               // scan kernel: (sequence, head, value slice) items over its CTAs
    int* next_item;          // packed batches: items past the first gridDim.x are claimed from this
                             // counter (zero before the launch); else strided over the CTAs
};

// Shared memory of the scan kernel: two 72 KB slots, each holding one record
// (the M = 128 reads of the 64-row PT tile, and for d_k = 64 of the Z tile,
// run on into the rest of the record's 64 KB, into rows whose products are
// discarded) and the chunk's V tile [64][NV] (bf16, 128-byte swizzle) at
// +64 KB; the state operand S [d_k][NV] and Y [64][NV] (fp16, MN-major B
// operands: value columns contiguous, 128-byte swizzle); the o staging tile
// [64][NV] (output type, 16-byte chunks XOR-swizzled by row).
template <int DK>
struct ScanPlan {
    static constexpr int SLOT = 73728, VOFF = 65536;
    static constexpr int SOP = 2 * SLOT;
    static constexpr int YB = SOP + NV * DK * 2;
    static constexpr int OST = YB + NV * C * 2;
    static constexpr int BAR = OST + C * NV * 4;
    static constexpr int END = BAR + 128;
    static constexpr int BYTES = END + 1024;
};

// MN-major SW128 B operand (16-bit, NV = 64 columns = one 128-byte row per K
// index): K-step kk (16 K rows = two 1 KB groups) starts 2 KB further on.
__device__ __forceinline__ uint64_t mn_desc(const unsigned char* tile, int kk, int k_rows)
{
    return sdesc_sw128(smem_u32(tile) + kk * 2048, (uint32_t)(k_rows * 128), 1024);
}

// Output rows [0, L) of one chunk from the TMEM accumulator (lane = row, 16
// columns per warpgroup), run by the 256 threads of lanes 0..63.  Rows are
// staged in the layout of the output tensor map's boxes (64 rows x 128 bytes,
// 128-byte swizzle; two boxes for fp32 output); a full chunk leaves with TMA
// stores issued by one thread, a partial one (the end of a sequence) with
// coalesced 16-byte row-segment stores.
template <typename TO>
__device__ __forceinline__ void store_o_tile(uint32_t t_acc, unsigned char* ost, const CUtensorMap* tmo, void* o,
                                             int tok, int h, int col0, size_t row0_off, size_t row_stride, int L,
                                             int lt, int wg, bool issuer)
{
    constexpr int EB = (int)sizeof(TO);
    constexpr int CPB = 8;                 // 16-byte chunks per 128-byte box row
    constexpr int CPT = EB;                // chunks per thread: 16 values
    constexpr int NBOX = NV * EB / 128;
    constexpr int CPR = NV * EB / 16;      // chunks per output row segment
    float acc[16];
    tmem_ld16(t_acc, acc);
    if (issuer) bulk_wait_read();          // the previous chunk's stores have read the tile
    tmem_wait_ld();
    bar_sync(1, 256);
#pragma unroll
    for (int u = 0; u < CPT; ++u) {
        const int k = wg * CPT + u, box = k / CPB, ci = k % CPB;
        uint4 val;
        if constexpr (EB == 4)
            val = make_uint4(__float_as_uint(acc[4 * u]), __float_as_uint(acc[4 * u + 1]),
                             __float_as_uint(acc[4 * u + 2]), __float_as_uint(acc[4 * u + 3]));
        else
            val = make_uint4(pack_bf16(acc[8 * u], acc[8 * u + 1]), pack_bf16(acc[8 * u + 2], acc[8 * u + 3]),
                             pack_bf16(acc[8 * u + 4], acc[8 * u + 5]), pack_bf16(acc[8 * u + 6], acc[8 * u + 7]));
        *reinterpret_cast<uint4*>(ost + box * 8192 + lt * 128 + ((ci ^ (lt & 7)) << 4)) = val;
    }
    fence_proxy_async();
    bar_sync(1, 256);
    if (L == C) {
        if (issuer) {
#pragma unroll
            for (int bx = 0; bx < NBOX; ++bx) tma_store_3d(tmo, ost + bx * 8192, col0 + bx * (128 / EB), h, tok);
            bulk_commit();
        }
    } else {
        const int t = wg * 64 + lt;
#pragma unroll
        for (int pss = 0; pss < C * CPR / 256; ++pss) {
            const int idx = pss * 256 + t, row = idx / CPR, k = idx % CPR;
            if (row < L) {
                const int box = k / CPB, ci = k % CPB;
                const uint4 val = *reinterpret_cast<const uint4*>(ost + box * 8192 + row * 128 + ((ci ^ (row & 7)) << 4));
                *reinterpret_cast<uint4*>(static_cast<unsigned char*>(o) + (row0_off + (size_t)row * row_stride) * EB + k * 16) = val;
            }
        }
    }
}

// One (sequence, head, NV value columns) item at a time: items bid0,
// bid0 + bid_step, ... (or claimed from p.next_item).  Thread (lane lt < d_k,
// warpgroup wg) keeps S[lt][16 wg .. 16 wg + 16) of the state in registers.
// Per chunk c (slot c % 2, c counted over all of the CTA's items):
//   S <- diag(e^G_last(c-1)) S + W(c-1)      W = Z Y of the chunk before, from TMEM
//   S operand (fp16) -> smem;  MMA [O ; X] = [Qh ; Kh] S  -> TMEM buffer c % 2
//   Y = diag(beta) (V - X) -> smem (lanes 64..127), while lanes 0..63 store
//   the o rows of chunk c - 1
//   MMA W = Z Y (commit), MMA O += PT Y
// A slot is refilled in two parts as soon as the MMAs reading each part have
// completed: the [Qh ; Kh] tile and V after chunk c's X MMA and Y phase, the
// Z, PT, e^G_last and beta part after chunk c + 1's X MMA (tcgen05 MMAs of
// one thread complete in issue order).
template <typename TO, int DK, int VK>
__device__ __forceinline__ void scan_body(const CUtensorMap& tmv, const CUtensorMap& tmo, const ScanParams& p,
                                          int bid0, int bid_step, int n_items)
{
    const bool no_erase = VK == kVarNoErase || (VK == kVarAny && p.no_erase);   // layer variant
    using PL = ScanPlan<DK>;
    using R = Rec<DK>;
    extern __shared__ unsigned char smem_raw[];
    KDA_PHASE_DECL(1)
    unsigned char* sm = align1024(smem_raw);
    unsigned char* Sop = sm + PL::SOP;
    unsigned char* Yb = sm + PL::YB;
    unsigned char* Ost = sm + PL::OST;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + PL::BAR);
    uint64_t* mb_a = bars + 0;     // [2]: [Qh ; Kh] and V of a slot
    uint64_t* mb_b = bars + 2;     // [2]: Z, PT, e^G_last and beta of a slot
    uint64_t* mb_x = bars + 4;
    uint64_t* mb_w = bars + 5;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int lt = tid & 127;
    const int wg = tid >> 7;
    const int nslice = p.DV / NV;
    const int H = p.H, DV = p.DV;
    const float* s_src = p.s_in;

    if (tid == 0) {
        for (int i = 0; i < 6; ++i) mbar_init(bars + i, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async();
        prefetch_tmap(&tmv);
        prefetch_tmap(&tmo);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_off = ((uint32_t)(warp & 3) * 32) << 16;
    const uint32_t q_off = (uint32_t)wg * 16;
    const uint32_t t_W = tmem + 128;
    constexpr uint32_t kI = idesc_f16(128, NV, 1);
    constexpr uint32_t kBytesA = R::Z + C * NV * 2;     // [Qh ; Kh] tile + V tile
    constexpr uint32_t kBytesB = R::BYTES - R::Z;       // Z, PT, e^G_last, beta

    // items bid0, bid0 + bid_step, ... (one (sequence, head, value slice) each):
    // the barriers and TMEM carry over, their phases counted across items
    int gbase = 0;                     // chunks this CTA ran before the current item
    int xbase = 0;                     // mb_x completions before the current item
    int slice = 0, h = 0, n = 0, tok0 = 0, len = 0, col0 = 0, nchunks = 0;
    long long j0 = 0;

    auto rec_of = [&](int cc) { return p.rec + ((size_t)(j0 + cc) * H + h) * R::BYTES; };
    // chunk cc of the current item is chunk gbase + cc of this CTA: its slot
    // and the parities of the slot's barriers follow that count
    auto issue_a = [&](int cc) {
        const int sl = (gbase + cc) & 1;
        unsigned char* slot = sm + sl * PL::SLOT;
        if (p.ready && !wait_ready(p.ready + (size_t)(j0 + cc) * H + h, abort_flag, p.timeout_cycles)) return;
        mbar_expect_tx(mb_a + sl, kBytesA);
        bulk_load(slot, rec_of(cc), R::Z, mb_a + sl);
        tma_load_3d(slot + PL::VOFF, &tmv, mb_a + sl, col0, h, tok0 + cc * C);
    };
    auto issue_b = [&](int cc) {
        const int sl = (gbase + cc) & 1;
        unsigned char* slot = sm + sl * PL::SLOT;
        mbar_expect_tx(mb_b + sl, kBytesB);
        bulk_load(slot + R::Z, rec_of(cc) + R::Z, kBytesB, mb_b + sl);
    };

    // thread 0 issues the MMAs; thread kIssuer every copy (record refills, V
    // tiles, output stores)
    constexpr int kIssuer = 32;
    const bool issuer = tid == kIssuer;
    unsigned pend = 0;                 // bits: 0-1 mb_a[slot], 2-3 mb_b[slot], 4 mb_x, 5 mb_w
    uint32_t apar = 0u, bpar = 0u;     // bit i: phase parity of the pending load of slot i
    int xph = 0, wph = 0;              // commits issued to mb_x / mb_w
    // packed batches: thread 0 claims the item after the current one when the
    // current one starts (the atomic's latency overlaps the item) and hands it
    // to the CTA after it
    int* const claim_sh = reinterpret_cast<int*>(tmem_slot + 2);
    int claimed = 0;
    auto advance = [&](int cur) {   // by every thread, after an item
        if (!p.next_item) return cur + bid_step;
        if (tid == 0) *claim_sh = claimed;
        __syncthreads();
        const int nb = *claim_sh;
        __syncthreads();   // every thread has read the claim before thread 0 writes the next
        return nb;
    };
    for (int bid = bid0; bid < n_items; bid = advance(bid)) {
        if (p.next_item && tid == 0) claimed = bid_step + atomicAdd(p.next_item, 1);
        slice = bid % nslice;
        h = (bid / nslice) % p.H;
        const int rank = bid / (nslice * p.H);
        if (p.cu) {
            n = p.order[rank];
            tok0 = p.cu[n];
            len = max(0, p.cu[n + 1] - tok0);
            j0 = p.choff[n];
        } else {
            n = rank;
            tok0 = n * p.T;
            len = p.T;
            j0 = (long long)n * p.rs - p.rc0;
        }
        col0 = slice * NV;
        nchunks = (len + C - 1) / C;
        if ((long long)tok0 + len > p.tokens || tok0 < 0) {
            if (tid == 0 && p.c_begin == 0) flag_bad_input();
            nchunks = 0;
            len = 0;
        }
        // this launch's part of the sequence: chunks [c_begin, c_end)
        if (p.c_begin > 0 && p.c_begin >= nchunks) continue;   // ended in an earlier launch; its state is final
        {
            const int lo = min(p.c_begin, nchunks), hi = min(p.c_end, nchunks);
            tok0 += lo * C;
            len = max(0, len - lo * C);
            j0 += lo;
            nchunks = max(0, hi - lo);
        }
        if (nchunks > 0 && (j0 < 0 || j0 + nchunks > p.max_chunks)) {   // records outside the buffer
            if (tid == 0) flag_bad_input();
            nchunks = 0;
            len = 0;
        }
        // records written earlier (not the cooperative hand-off): the first
        // two records and V tiles of item bid + bid_step, which some CTA takes
        // about one round of items later, into L2 (the address loads overlap
        // this item's first copies)
        if (!p.ready && tid == 64 && bid + bid_step < n_items) {
            const int nb = bid + bid_step;
            const int sl2 = nb % nslice, h2 = (nb / nslice) % p.H, r2 = nb / (nslice * p.H);
            int tk2, ln2;
            long long jj2;
            if (p.cu) {
                const int n2 = p.order[r2];
                tk2 = p.cu[n2];
                ln2 = max(0, p.cu[n2 + 1] - tk2);
                jj2 = p.choff[n2];
            } else {
                tk2 = r2 * p.T;
                ln2 = p.T;
                jj2 = (long long)r2 * p.rs - p.rc0;
            }
            const int lo2 = min(p.c_begin, (ln2 + C - 1) / C);
            const int nc2 = min(2, max(0, min(p.c_end, (ln2 + C - 1) / C) - lo2));
            if (tk2 >= 0 && (long long)tk2 + ln2 <= p.tokens && jj2 + lo2 >= 0 && jj2 + lo2 + nc2 <= p.max_chunks)
                for (int cc = 0; cc < nc2; ++cc) {
                    bulk_prefetch_l2(p.rec + ((size_t)(jj2 + lo2 + cc) * H + h2) * R::BYTES, (uint32_t)R::BYTES);
                    tma_prefetch_3d(&tmv, sl2 * NV, h2, tk2 + (lo2 + cc) * C);
                }
        }
        // state rows of this thread
        float S[16];
        {
            const bool own = lt < DK && s_src;
            const float* src = own ? s_src + (((size_t)n * H + h) * DK + lt) * DV + col0 + 16 * wg : nullptr;
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
                const float4 v4 = own ? *reinterpret_cast<const float4*>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
                S[j] = v4.x; S[j + 1] = v4.y; S[j + 2] = v4.z; S[j + 3] = v4.w;
            }
        }

        int c = 0;
        if (issuer)
            for (int cc = 0; cc < 2 && cc < nchunks; ++cc) {
                issue_a(cc);
                issue_b(cc);
            }
        for (int cc = 0; cc < 2 && cc < nchunks; ++cc) {
            const int sl = (gbase + cc) & 1;
            const uint32_t par = (uint32_t)(((gbase + cc) >> 1) & 1);
            pend |= (1u | 4u) << sl;
            apar = (apar & ~(1u << sl)) | (par << sl);
            bpar = (bpar & ~(1u << sl)) | (par << sl);
        }

        float eglp = 1.f;                  // e^G_last of the previous chunk, key channel lt
        int Lprev = 0;
        for (c = 0; c < nchunks; ++c) {
            const int g = gbase + c;   // this CTA's chunk count
            const int b = g & 1;
            unsigned char* slot = sm + b * PL::SLOT;
            const uint32_t t_XO = tmem + 64 * b;
            const int L = min(C, len - c * C);
            KDA_PHASE(0);

            // ---- state of chunk c - 1, then its fp16 operand (row = value column)
            if (c > 0) {
                KDA_WAIT_OR_EXIT(mb_w, 32u, (g - 1) & 1);
                tc_fence_after();
                float w[16];
                tmem_ld16(t_W + lane_off + q_off, w);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) S[j] = fmaf(eglp, S[j], w[j]);
            }
            if (lt < DK) st_row_h16(Sop, lt, 16 * wg, DK, S);
            fence_proxy_async();
            tc_fence_before();
            KDA_WAIT_OR_EXIT(mb_a + b, 1u << b, (apar >> b) & 1u);
            KDA_PHASE(1);

            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)    // [O ; X] = [Qh ; Kh] S
                    umma_f16(t_XO, kdesc(slot + R::QK, kk, 128 * 128), mn_desc(Sop, kk, DK), kI, kk > 0);
                umma_commit(mb_x);
            }
            ++xph;
            pend |= 16u;
            KDA_WAIT_OR_EXIT(mb_x, 16u, (xbase + c) & 1);
            tc_fence_after();
            // chunk c - 1's PT Y has completed as well: refill the other slot's
            // second part with chunk c + 1
            if (c >= 1 && c + 1 < nchunks) {
                if (issuer) {
                    fence_proxy_async();
                    issue_b(c + 1);
                }
                pend |= 4u << (b ^ 1);
                bpar = (bpar & ~(1u << (b ^ 1))) | ((uint32_t)(((g + 1) >> 1) & 1) << (b ^ 1));
            }
            KDA_WAIT_OR_EXIT(mb_b + b, 4u << b, (bpar >> b) & 1u);
            KDA_PHASE(2);

            // ---- Y = beta (V - X) (lanes 64..127) | o rows of chunk c - 1 (lanes 0..63)
            {
                const float* egl = reinterpret_cast<const float*>(slot + R::EGL);
                const float* beta = reinterpret_cast<const float*>(slot + R::BETA);
                eglp = lt < DK ? egl[lt] : 1.f;
                if (lt >= C) {
                    const int s = lt - C;
                    float x16[16];
                    tmem_ld16(t_XO + lane_off + q_off, x16);
                    tmem_wait_ld();
                    const float bs = beta[s];
                    const unsigned char* vt = slot + PL::VOFF;
                    uint4 vr[2];
                    vr[0] = *reinterpret_cast<const uint4*>(vt + swh_off(s, 16 * wg, C));
                    vr[1] = *reinterpret_cast<const uint4*>(vt + swh_off(s, 16 * wg + 8, C));
                    float y[16];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&vr[u]);
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            const float2 f2 = __bfloat1622float2(v2[w]);
                            const int jj = 8 * u + 2 * w;
                            y[jj] = bs * (f2.x - (no_erase ? 0.f : x16[jj]));
                            y[jj + 1] = bs * (f2.y - (no_erase ? 0.f : x16[jj + 1]));
                        }
                    }
                    st_row_h16(Yb, s, 16 * wg, C, y);
                } else if (c > 0) {
                    const int tk = tok0 + (c - 1) * C;
                    store_o_tile<TO>(tmem + 64 * (b ^ 1) + lane_off + q_off, Ost, &tmo, p.o, tk, h, col0,
                                     ((size_t)tk * H + h) * DV + col0, (size_t)H * DV, Lprev, lt, wg, issuer);
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncthreads();
            KDA_PHASE(3);
            if (issuer && c + 2 < nchunks) {            // X MMA done, V consumed: refill part one
                fence_proxy_async();
                issue_a(c + 2);
            }

            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)     // W = Z Y
                    umma_f16(t_W, kdesc(slot + R::Z, kk, DK * 128), mn_desc(Yb, kk, C), kI, kk > 0);
                umma_commit(mb_w);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)     // O += PT Y  (rows 64..127: discarded)
                    umma_f16(t_XO, kdesc(slot + R::PT, kk, C * 128), mn_desc(Yb, kk, C), kI, 1);
            }
            ++wph;
            pend |= 32u;
            if (c + 2 < nchunks) {
                pend |= 1u << b;
                apar = (apar & ~(1u << b)) | ((uint32_t)(((g + 2) >> 1) & 1) << b);
            }
            Lprev = L;
            KDA_PHASE(4);
        }

        if (nchunks > 0) {
            // W and O of the last chunk: one more commit covers every MMA issued
            if (tid == 0) umma_commit(mb_x);
            ++xph;
            pend |= 16u;
            KDA_WAIT_OR_EXIT(mb_x, 16u, (xbase + nchunks) & 1);
            pend &= ~32u;
            tc_fence_after();
            float w[16];
            tmem_ld16(t_W + lane_off + q_off, w);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) S[j] = fmaf(eglp, S[j], w[j]);
            if (lt < C) {
                const int tk = tok0 + (nchunks - 1) * C;
                store_o_tile<TO>(tmem + 64 * ((gbase + nchunks - 1) & 1) + lane_off + q_off, Ost, &tmo, p.o, tk, h, col0,
                                 ((size_t)tk * H + h) * DV + col0, (size_t)H * DV, Lprev, lt, wg, issuer);
            }
        }
        if (p.s_out && lt < DK) {
            float* dst = p.s_out + (((size_t)n * H + h) * DK + lt) * DV + col0 + 16 * wg;
#pragma unroll
            for (int j = 0; j < 16; j += 4)
                *reinterpret_cast<float4*>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }

        gbase += nchunks;
        xbase += nchunks > 0 ? nchunks + 1 : 0;
    }

finish:
    KDA_PHASE_FLUSH
    if (*abort_flag) {
        // let every copy and MMA in flight land before the TMEM is released
        volatile int never = 0;
        for (int i = 0; i < 2; ++i) {
            if (pend & (1u << i)) (void)mbar_wait(mb_a + i, (apar >> i) & 1u, &never, p.timeout_cycles);
            if (pend & (4u << i)) (void)mbar_wait(mb_b + i, (bpar >> i) & 1u, &never, p.timeout_cycles);
        }
        if (pend & 16u) (void)mbar_wait(mb_x, (uint32_t)((xph - 1) & 1), &never, p.timeout_cycles);
        if (pend & 32u) (void)mbar_wait(mb_w, (uint32_t)((wph - 1) & 1), &never, p.timeout_cycles);
        __syncthreads();
        if (tid == 0) umma_commit(mb_x);
        (void)mbar_wait(mb_x, (uint32_t)(xph & 1), &never, p.timeout_cycles);
    }
    if (issuer) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}
#undef KDA_WAIT_OR_EXIT

template <int DK, int VK>
__global__ void __launch_bounds__(NT, 1)
chunk_prep_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmg, const PrepParams p)
{
    prep_body<DK, VK>(tmq, tmk, tmg, p, blockIdx.x, gridDim.x);
}

template <typename TO, int DK, int VK>
__global__ void __launch_bounds__(NT, 1)
chunk_scan_kernel(const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
                  const ScanParams p)
{
    scan_body<TO, DK, VK>(tmv, tmo, p, blockIdx.x, gridDim.x, p.items);
}

// Cooperative schedule: CTAs [0, n_scan) scan, the others prep; the scan
// waits on the records' ready flags, the prep never waits on the scan, and a
// cooperative launch keeps every CTA resident, so the hand-off cannot stall.
template <typename TO, int DK, int VK>
__global__ void __launch_bounds__(NT, 1)
chunk_coop_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmg, const __grid_constant__ CUtensorMap tmv,
                  const __grid_constant__ CUtensorMap tmo, const PrepParams pp, const ScanParams sp, int n_scan)
{
    // the scan of a per-head-gate call is the plain layer's
    if ((int)blockIdx.x < n_scan)
        scan_body<TO, DK, VK == kVarHeadGate ? kVarPlain : VK>(tmv, tmo, sp, blockIdx.x, n_scan, n_scan);
    else prep_body<DK, VK>(tmq, tmk, tmg, pp, blockIdx.x - n_scan, gridDim.x - n_scan);
}

// Kernel entry points of one variant kind.
template <typename TO, int DK, int VK>
struct Kernels {
    static constexpr int kScanVK = VK == kVarHeadGate ? kVarPlain : VK;
    static constexpr auto prep = chunk_prep_kernel<DK, VK>;
    static constexpr auto scan = chunk_scan_kernel<TO, DK, kScanVK>;
    static constexpr auto coop = chunk_coop_kernel<TO, DK, VK>;
};

// ============================================================== host side

// Per-call index arrays of a packed (varlen) batch, one CTA of 1024 threads:
//   choff[i] = sum_{j<i} ceil(len_j / 64) (first record of sequence i),
//   choff[nseq] = total;
//   order[r] = the sequence the scan CTAs of rank r take: longest first, ties
//   by lower index (negative lengths count as empty).
// The order is a bitonic sort of 64-bit keys (complemented length, index) of
// the next power of two of nseq, in shared memory when it fits, else in the
// workspace `gkeys`.
constexpr int kIndexThreads = 1024;
constexpr int kSmemKeys = 16384;

__global__ void __launch_bounds__(kIndexThreads)
varlen_index_kernel(const int32_t* cu, int nseq, int32_t* choff, int32_t* order, unsigned long long* gkeys,
                    int* work)
{
    if (threadIdx.x == 0) *work = 0;
    __shared__ int warp_tot[32];
    extern __shared__ unsigned long long skeys[];
    const int tid = threadIdx.x;
    const int per = (nseq + kIndexThreads - 1) / kIndexThreads;
    const int a = min(nseq, tid * per), b = min(nseq, a + per);
    int local = 0;
    for (int i = a; i < b; ++i) local += (max(0, cu[i + 1] - cu[i]) + C - 1) / C;
    int x = local;
    const int lane = tid & 31, w = tid >> 5;
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
    if (tid == kIndexThreads - 1) choff[nseq] = base;

    int npad = 1;
    while (npad < nseq) npad <<= 1;
    unsigned long long* keys = npad <= kSmemKeys ? skeys : gkeys;
    for (int i = tid; i < npad; i += kIndexThreads) {
        const unsigned len = i < nseq ? (unsigned)max(0, cu[i + 1] - cu[i]) : 0u;
        // ascending keys: longer first, then lower index; padding sorts last
        keys[i] = i < nseq ? ((unsigned long long)(0x7fffffffu - len) << 32) | (unsigned)i : ~0ull;
    }
    __syncthreads();
    for (int size = 2; size <= npad; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = tid; t < npad / 2; t += kIndexThreads) {
                const int lo = 2 * t - (t & (stride - 1));    // index whose `stride` bit is clear
                const int hi = lo + stride;
                const bool up = (lo & size) == 0;
                const unsigned long long kl = keys[lo], kh = keys[hi];
                if ((kl > kh) == up) {
                    keys[lo] = kh;
                    keys[hi] = kl;
                }
            }
            __syncthreads();
        }
    }
    for (int r = tid; r < nseq; r += kIndexThreads) order[r] = (int32_t)(keys[r] & 0xffffffffu);
}

static int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return n > 0 ? n : 148;
}

// Second stream on which the parallel pass of the next block of chunks runs
// while the current block is scanned.  Cached per CUDA context (created on
// first use in that context), so a context that is destroyed and re-created
// gets a stream of its own.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

static CUcontext current_context()
{
    static CtxGetCurrentFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
    }
    CUcontext ctx = nullptr;
    if (cudaFree(nullptr) != cudaSuccess) return nullptr;   // makes the device's primary context current
    return fn(&ctx) == CUDA_SUCCESS ? ctx : nullptr;
}

static cudaStream_t side_stream()
{
    static std::mutex mu;
    static CUcontext ctxs[64] = {};
    static cudaStream_t streams[64] = {};
    const CUcontext ctx = current_context();
    if (!ctx) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    int slot = -1;
    for (int i = 0; i < 64; ++i) {
        if (ctxs[i] == ctx) return streams[i];
        if (!ctxs[i] && slot < 0) slot = i;
    }
    if (slot < 0) return nullptr;
    cudaStream_t st = nullptr;
    if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    ctxs[slot] = ctx;
    streams[slot] = st;
    return st;
}

constexpr int kMaxBlocks = 8;

// Offsets (bytes) of the parts of a call's workspace.
struct WsLayout {
    size_t choff, order, work, keys, carry, flags, rec, bytes;
    long long max_chunks;
};

static size_t align1k(size_t x) { return (x + 1023) & ~(size_t)1023; }

template <int DK>
static WsLayout ws_layout(int nseq, int T, long long tokens, int H, int dv, bool varlen)
{
    WsLayout w{};
    w.max_chunks = varlen ? tokens / C + nseq : (long long)nseq * ((T + C - 1) / C);
    int npad = 1;
    while (npad < nseq) npad <<= 1;
    size_t off = 0;
    w.choff = off;
    off += varlen ? align1k(((size_t)nseq + 1) * 4) : 0;
    w.order = off;
    off += varlen ? align1k((size_t)nseq * 4) : 0;
    w.work = off;                                          // the packed scan's next-item counter
    off += varlen ? 1024 : 0;
    w.keys = off;
    off += (varlen && npad > kSmemKeys) ? align1k((size_t)npad * 8) : 0;
    w.carry = off;                                         // state between blocks when no final state is kept
    off += varlen ? 0 : align1k((size_t)nseq * H * DK * dv * 4);
    w.flags = off;                                         // cooperative hand-off flags, one per record
    off += varlen ? 0 : align1k((size_t)w.max_chunks * H * 4);
    w.rec = off;
    off += (size_t)w.max_chunks * H * Rec<DK>::BYTES;
    w.bytes = off;
    return w;
}

template <typename TO, int DK>
static cudaError_t run(const void* q, const void* k, const void* v, const float* beta, const float* log_alpha,
                       const float* s0, void* o, float* sT, const int32_t* cu, int nseq, int T, long long tokens,
                       int H, int dv, long long timeout_cycles, int mode, unsigned char* ws, size_t ws_bytes,
                       cudaStream_t stream)
{
    const bool head_gate = (mode & KDA_MODE_HEAD_GATE) != 0;
    const int vflags = mode & (KDA_MODE_HEAD_GATE | KDA_MODE_NO_ERASE | KDA_MODE_NORM_QK | KDA_MODE_GATE_LOGITS);
    const int vk = vflags == 0 ? kVarPlain
                 : vflags == KDA_MODE_HEAD_GATE ? kVarHeadGate
                 : vflags == KDA_MODE_NO_ERASE ? kVarNoErase : kVarAny;
    const int req_blocks = (mode >> 8) & 0xff;     // KDA_MODE_BLOCKS(n), 0 = automatic
    const int nsm = sm_count();
    const int nch = cu ? 0 : (T + C - 1) / C;
    const WsLayout L = ws_layout<DK>(nseq, T, tokens, H, dv, cu != nullptr);
    if (!ws || ws_bytes < L.bytes) return cudaErrorInvalidValue;
    const long long max_chunks = L.max_chunks;
    const long long scan_ctas = (long long)nseq * H * (dv / NV);
    if (scan_ctas > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    // schedule: one cooperative launch (prep CTAs publish records, scan CTAs
    // consume them) when the scan grid leaves at least 32 SMs; otherwise prep
    // then scan.  KDA_MODE_BLOCKS(n) asks for n blocks of chunks on two
    // streams instead (dense inputs).
    const bool coop = !cu && req_blocks == 0 && scan_ctas > 0 && scan_ctas + 32 <= nsm;
    const int nb = (cu || coop || req_blocks == 0) ? 1 : std::max(1, std::min(std::min(req_blocks, nch), kMaxBlocks));
    cudaStream_t side = nb > 1 ? side_stream() : nullptr;

    CUtensorMap tq, tk, tg;
    memset(&tg, 0, sizeof(tg));   // per-head gates: no gate tile to load (the map is never used)
    if (!make_tmap(&tq, q, tokens, H, DK, false) || !make_tmap(&tk, k, tokens, H, DK, false) ||
        (!head_gate && !make_tmap(&tg, log_alpha, tokens, H, DK, true)))
        return cudaErrorInvalidValue;
    CUtensorMap tv, to;
    if (!make_tmap(&tv, v, tokens, H, dv, false, NV, true) ||
        !make_tmap(&to, o, tokens, H, dv, sizeof(TO) == 4, 128 / (int)sizeof(TO), true))
        return cudaErrorInvalidValue;
    using K0 = Kernels<TO, DK, kVarPlain>;
    using K1 = Kernels<TO, DK, kVarHeadGate>;
    using K2 = Kernels<TO, DK, kVarNoErase>;
    using K3 = Kernels<TO, DK, kVarAny>;
    auto pk = vk == kVarPlain ? K0::prep : vk == kVarHeadGate ? K1::prep : vk == kVarNoErase ? K2::prep : K3::prep;
    auto sk = vk == kVarPlain ? K0::scan : vk == kVarHeadGate ? K1::scan : vk == kVarNoErase ? K2::scan : K3::scan;
    cudaError_t err = cudaFuncSetAttribute(pk, cudaFuncAttributeMaxDynamicSharedMemorySize, PrepPlan::BYTES);
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(sk, cudaFuncAttributeMaxDynamicSharedMemorySize, ScanPlan<DK>::BYTES);
    if (err != cudaSuccess) return err;

    // events of the two-stream schedule (created last: no early return leaks them)
    cudaEvent_t ev[kMaxBlocks + 1];
    int nev = 0;
    if (side) {
        for (; nev <= nb; ++nev)
            if (cudaEventCreateWithFlags(&ev[nev], cudaEventDisableTiming) != cudaSuccess) break;
        if (nev <= nb) {   // fall back to one stream
            for (int i = 0; i < nev; ++i) cudaEventDestroy(ev[i]);
            nev = 0;
            side = nullptr;
        }
    }
    // without a second stream the blocks run one after the other (same results)
    const int nblocks = nb;
    const int cb = cu ? 0 : (nch + nblocks - 1) / nblocks;     // chunks per block (dense)
    int32_t* choff = reinterpret_cast<int32_t*>(ws + L.choff);
    int32_t* order = reinterpret_cast<int32_t*>(ws + L.order);
    float* carry = sT ? sT : reinterpret_cast<float*>(ws + L.carry);
    unsigned char* rec = ws + L.rec;

    if (cu) {
        int npad = 1;
        while (npad < nseq) npad <<= 1;
        const int smem = npad <= kSmemKeys ? npad * 8 : 0;
        err = cudaFuncSetAttribute(varlen_index_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemKeys * 8);
        if (err == cudaSuccess) {
            varlen_index_kernel<<<1, kIndexThreads, smem, stream>>>(cu, nseq, choff, order,
                                                                    reinterpret_cast<unsigned long long*>(ws + L.keys),
                                                                    reinterpret_cast<int*>(ws + L.work));
            err = cudaGetLastError();
        }
        if (err != cudaSuccess) {
            for (int i = 0; i < nev; ++i) cudaEventDestroy(ev[i]);
            return err;
        }
    }

    PrepParams pp{};
    pp.beta = beta;
    pp.cu = cu;
    pp.choff = choff;
    pp.rec = rec;
    pp.nseq = nseq;
    pp.T = T;
    pp.H = H;
    pp.nch = nch;
    pp.rs = nch;
    pp.rc0 = 0;
    pp.tokens = tokens;
    pp.timeout_cycles = timeout_cycles;
    pp.gh = head_gate ? log_alpha : nullptr;
    pp.no_erase = (mode & KDA_MODE_NO_ERASE) ? 1 : 0;
    pp.norm_qk = (mode & KDA_MODE_NORM_QK) ? 1 : 0;
    pp.logits = (mode & KDA_MODE_GATE_LOGITS) ? 1 : 0;
    ScanParams sp{};
    sp.no_erase = pp.no_erase;
    sp.v = static_cast<const __nv_bfloat16*>(v);
    sp.o = o;
    sp.cu = cu;
    sp.choff = choff;
    sp.order = order;
    sp.rec = rec;
    sp.nseq = nseq;
    sp.T = T;
    sp.H = H;
    sp.DV = dv;
    sp.nch = nch;
    sp.rs = nch;
    sp.rc0 = 0;
    sp.max_chunks = max_chunks;
    sp.tokens = tokens;
    sp.timeout_cycles = timeout_cycles;

    auto launch_prep = [&](int b, cudaStream_t st, long long grid_cap) {
        if (cu) {
            pp.c_begin = 0;
            pp.cbs = 0;
            pp.nitems = max_chunks * H;
        } else {
            pp.c_begin = b * cb;
            pp.cbs = std::max(0, std::min(cb, nch - b * cb));
            pp.nitems = (long long)nseq * pp.cbs * H;
        }
        if (pp.nitems <= 0) return cudaSuccess;
        const long long grid = std::max(1LL, std::min(pp.nitems, grid_cap));
        pk<<<(unsigned)grid, NT, PrepPlan::BYTES, st>>>(tq, tk, tg, pp);
        return cudaGetLastError();
    };
    auto launch_scan = [&](int b) {
        sp.c_begin = cu ? 0 : b * cb;
        sp.c_end = (cu || b == nblocks - 1) ? 0x7fffffff : (b + 1) * cb;
        sp.s_in = b == 0 ? s0 : carry;
        sp.s_out = (b == nblocks - 1) ? sT : carry;
        if (scan_ctas <= 0) return cudaSuccess;
        // one CTA per item; beyond 4 items per SM, one persistent CTA per SM
        // takes items in rank order (packed batches: claimed from a counter)
        const long long grid = scan_ctas > 4LL * nsm ? nsm : scan_ctas;
        sp.items = (int)scan_ctas;
        sp.next_item = (cu && grid < scan_ctas) ? reinterpret_cast<int*>(ws + L.work) : nullptr;
        sk<<<(unsigned)grid, NT, ScanPlan<DK>::BYTES, stream>>>(tv, to, sp);
        return cudaGetLastError();
    };

    bool done = false;
    if (coop) {
        unsigned* flags = reinterpret_cast<unsigned*>(ws + L.flags);
        err = cudaMemsetAsync(flags, 0, (size_t)max_chunks * H * 4, stream);
        auto ck = vk == kVarPlain ? K0::coop : vk == kVarHeadGate ? K1::coop : vk == kVarNoErase ? K2::coop : K3::coop;
        const int smem = std::max(PrepPlan::BYTES, ScanPlan<DK>::BYTES);
        if (err == cudaSuccess) err = cudaFuncSetAttribute(ck, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (err == cudaSuccess) {
            pp.ready = flags;
            pp.c_begin = 0;
            pp.cbs = nch;
            pp.nitems = max_chunks * H;
            sp.ready = flags;
            sp.c_begin = 0;
            sp.c_end = 0x7fffffff;
            sp.s_in = s0;
            sp.s_out = sT;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)nsm);
            cfg.blockDim = dim3(NT);
            cfg.dynamicSmemBytes = (size_t)smem;
            cfg.stream = stream;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeCooperative;
            attr[0].val.cooperative = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            const int n_scan = (int)scan_ctas;
            if (cudaLaunchKernelEx(&cfg, ck, tq, tk, tg, tv, to, pp, sp, n_scan) == cudaSuccess) done = true;
            else (void)cudaGetLastError();   // not co-residable here: fall back to prep then scan
            pp.ready = nullptr;
            sp.ready = nullptr;
        }
    }
    if (done) {
    } else if (nblocks == 1 || !side) {
        for (int b = 0; b < nblocks && err == cudaSuccess; ++b) {
            err = launch_prep(b, stream, nsm);
            if (err == cudaSuccess) err = launch_scan(b);
        }
    } else {
        // fork: the side stream starts after everything queued on `stream`;
        // the scan of block b waits for the prep of block b; the prep of
        // block b + 1 shares the GPU with that scan
        err = cudaEventRecord(ev[0], stream);
        if (err == cudaSuccess) err = cudaStreamWaitEvent(side, ev[0], 0);
        if (err == cudaSuccess) err = launch_prep(0, side, nsm);
        if (err == cudaSuccess) err = cudaEventRecord(ev[1], side);
        for (int b = 0; b < nblocks && err == cudaSuccess; ++b) {
            err = cudaStreamWaitEvent(stream, ev[b + 1], 0);
            if (err == cudaSuccess) err = launch_scan(b);
            if (err == cudaSuccess && b + 1 < nblocks) {
                err = launch_prep(b + 1, side, std::max(1LL, nsm - scan_ctas));
                if (err == cudaSuccess) err = cudaEventRecord(ev[b + 2], side);
            }
        }
        if (err != cudaSuccess) {   // join the side stream back whatever happened
            cudaEventRecord(ev[nblocks], side);
            cudaStreamWaitEvent(stream, ev[nblocks], 0);
        }
    }
    for (int i = 0; i < nev; ++i) cudaEventDestroy(ev[i]);
    return err;
}

// ============================================================== allocation-free variant

// Library-owned scratch of kda_chunk_fwd_noalloc: the operand records of two
// blocks of chunks used as a ring, and the carried state when the caller
// keeps no final state.  One area per device, so calls that use it must be
// ordered with respect to each other (one stream, or synchronised).
constexpr size_t kScratchBytes = size_t(64) << 20;
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Device address of this device's scratch area, looked up on every call
// (cheap), so that it always belongs to the current context.
static unsigned char* scratch_area()
{
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess) return nullptr;
    return static_cast<unsigned char*>(p);
}

static size_t carry_bytes(int nseq, int H, int dk, int dv, bool has_final)
{
    return has_final ? 0 : (((size_t)nseq * H * dk * dv * 4 + 1023) & ~(size_t)1023);
}

// Chunks per block of the ring: all nch in one block when their records fit
// (no carried state is needed then), else the most that fit twice over next
// to the carried state; 0 when not even one chunk fits that way.
template <int DK>
static long long noalloc_block(int nseq, int H, int dv, bool has_final, int nch)
{
    const size_t per_chunk = (size_t)nseq * H * Rec<DK>::BYTES;   // one chunk of every (sequence, head)
    if (per_chunk == 0) return 0;
    if ((size_t)nch * per_chunk <= kScratchBytes) return nch;
    const size_t carry = carry_bytes(nseq, H, DK, dv, has_final);
    if (carry + 2 * per_chunk > kScratchBytes) return 0;
    return std::min<long long>(nch, (long long)((kScratchBytes - carry) / (2 * per_chunk)));
}

template <typename TO, int DK>
static cudaError_t run_noalloc(const void* q, const void* k, const void* v, const float* beta,
                               const float* log_alpha, const float* s0, void* o, float* sT, int nseq, int T,
                               long long tokens, int H, int dv, long long timeout_cycles, cudaStream_t stream)
{
    using R = Rec<DK>;
    const int nsm = sm_count();
    const int nch = (T + C - 1) / C;
    const long long cb = noalloc_block<DK>(nseq, H, dv, sT != nullptr, nch);
    if (cb <= 0) return cudaErrorInvalidValue;
    const int nblocks = (int)((nch + cb - 1) / cb);
    const long long scan_ctas = (long long)nseq * H * (dv / NV);
    if (scan_ctas > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    unsigned char* area = scratch_area();
    if (!area) return cudaErrorInvalidSymbol;
    const size_t carry_sz = nblocks > 1 ? carry_bytes(nseq, H, DK, dv, sT != nullptr) : 0;
    float* carry = sT ? sT : reinterpret_cast<float*>(area);   // unused with one block
    unsigned char* ring[2] = {area + carry_sz, nullptr};
    if (nblocks > 1) ring[1] = area + carry_sz + (size_t)cb * nseq * H * R::BYTES;

    CUtensorMap tq, tk, tg, tv, to;
    if (!make_tmap(&tq, q, tokens, H, DK, false) || !make_tmap(&tk, k, tokens, H, DK, false) ||
        !make_tmap(&tg, log_alpha, tokens, H, DK, true) || !make_tmap(&tv, v, tokens, H, dv, false, NV, true) ||
        !make_tmap(&to, o, tokens, H, dv, sizeof(TO) == 4, 128 / (int)sizeof(TO), true))
        return cudaErrorInvalidValue;
    auto pk = chunk_prep_kernel<DK, kVarPlain>;
    auto sk = chunk_scan_kernel<TO, DK, kVarPlain>;
    cudaError_t err = cudaFuncSetAttribute(pk, cudaFuncAttributeMaxDynamicSharedMemorySize, PrepPlan::BYTES);
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(sk, cudaFuncAttributeMaxDynamicSharedMemorySize, ScanPlan<DK>::BYTES);
    if (err != cudaSuccess) return err;

    PrepParams pp{};
    pp.beta = beta;
    pp.nseq = nseq;
    pp.T = T;
    pp.H = H;
    pp.nch = nch;
    pp.rs = (int)cb;
    pp.tokens = tokens;
    pp.timeout_cycles = timeout_cycles;
    ScanParams sp{};
    sp.v = static_cast<const __nv_bfloat16*>(v);
    sp.o = o;
    sp.nseq = nseq;
    sp.T = T;
    sp.H = H;
    sp.DV = dv;
    sp.nch = nch;
    sp.rs = (int)cb;
    sp.max_chunks = (long long)nseq * cb;
    sp.tokens = tokens;
    sp.timeout_cycles = timeout_cycles;

    // block b: chunks [b cb, (b + 1) cb) of every sequence, records in ring[b % 2]
    auto launch_prep = [&](int b, cudaStream_t st, long long grid_cap) {
        pp.rec = ring[b & 1];
        pp.c_begin = (int)(b * cb);
        pp.rc0 = pp.c_begin;
        pp.cbs = (int)std::min<long long>(cb, nch - b * cb);
        pp.nitems = (long long)nseq * pp.cbs * H;
        if (pp.nitems <= 0) return cudaSuccess;
        const long long grid = std::max(1LL, std::min(pp.nitems, grid_cap));
        pk<<<(unsigned)grid, NT, PrepPlan::BYTES, st>>>(tq, tk, tg, pp);
        return cudaGetLastError();
    };
    auto launch_scan = [&](int b) {
        sp.rec = ring[b & 1];
        sp.c_begin = (int)(b * cb);
        sp.rc0 = sp.c_begin;
        sp.c_end = b == nblocks - 1 ? 0x7fffffff : (int)((b + 1) * cb);
        sp.s_in = b == 0 ? s0 : carry;
        sp.s_out = b == nblocks - 1 ? sT : carry;
        if (scan_ctas <= 0) return cudaSuccess;
        // one CTA per item; beyond 4 items per SM, one persistent CTA per SM
        // takes every gridDim.x-th item
        const long long grid = scan_ctas > 4LL * nsm ? nsm : scan_ctas;
        sp.items = (int)scan_ctas;
        sk<<<(unsigned)grid, NT, ScanPlan<DK>::BYTES, stream>>>(tv, to, sp);
        return cudaGetLastError();
    };

    cudaStream_t side = nblocks > 1 ? side_stream() : nullptr;
    cudaEvent_t ev[5];
    int nev = 0;
    if (side) {
        for (; nev < 5; ++nev)
            if (cudaEventCreateWithFlags(&ev[nev], cudaEventDisableTiming) != cudaSuccess) break;
        if (nev < 5) {
            for (int i = 0; i < nev; ++i) cudaEventDestroy(ev[i]);
            nev = 0;
            side = nullptr;
        }
    }
    if (!side) {   // one stream: blocks in order, no overlap
        for (int b = 0; b < nblocks && err == cudaSuccess; ++b) {
            err = launch_prep(b, stream, nsm);
            if (err == cudaSuccess) err = launch_scan(b);
        }
        return err;
    }
    // two streams: prep(b + 1) overlaps scan(b); prep(b + 2) reuses the ring
    // slot of block b only after scan(b) has finished with it
    cudaEvent_t ev_prep[2] = {ev[1], ev[2]}, ev_scan[2] = {ev[3], ev[4]};
    err = cudaEventRecord(ev[0], stream);
    if (err == cudaSuccess) err = cudaStreamWaitEvent(side, ev[0], 0);
    if (err == cudaSuccess) err = launch_prep(0, side, nsm);
    if (err == cudaSuccess) err = cudaEventRecord(ev_prep[0], side);
    for (int b = 0; b < nblocks && err == cudaSuccess; ++b) {
        err = cudaStreamWaitEvent(stream, ev_prep[b & 1], 0);
        if (err == cudaSuccess) err = launch_scan(b);
        if (err == cudaSuccess) err = cudaEventRecord(ev_scan[b & 1], stream);
        if (err == cudaSuccess && b + 1 < nblocks) {
            if (b + 1 >= 2) err = cudaStreamWaitEvent(side, ev_scan[(b + 1) & 1], 0);
            if (err == cudaSuccess) err = launch_prep(b + 1, side, scan_ctas < nsm ? nsm - scan_ctas : nsm);
            if (err == cudaSuccess) err = cudaEventRecord(ev_prep[(b + 1) & 1], side);
        }
    }
    if (err != cudaSuccess) {   // join the side stream back whatever happened
        cudaEventRecord(ev[0], side);
        cudaStreamWaitEvent(stream, ev[0], 0);
    }
    for (int i = 0; i < nev; ++i) cudaEventDestroy(ev[i]);
    return err;
}

}  // namespace split

bool chunk_fwd_split_supported(int dk, int dv, kda_dtype dtype)
{
    return dtype == KDA_BF16 && (dk == 64 || dk == 128) && (dv == 64 || dv == 128);
}

size_t chunk_fwd_split_workspace(int nseq, int T, long long tokens, int H, int dk, int dv, bool varlen, int mode)
{
    (void)mode;
    return dk == 128 ? split::ws_layout<128>(nseq, T, tokens, H, dv, varlen).bytes
                     : split::ws_layout<64>(nseq, T, tokens, H, dv, varlen).bytes;
}

cudaError_t chunk_fwd_split(const void* q, const void* k, const void* v, const float* beta,
                            const float* log_alpha, const float* s0, void* o, float* sT, const int32_t* cu,
                            int nseq, int T, long long tokens, int H, int dk, int dv, kda_dtype o_dtype,
                            long long timeout_cycles, int mode, void* ws, size_t ws_bytes, cudaStream_t stream)
{
    unsigned char* w = static_cast<unsigned char*>(ws);
    if (o_dtype == KDA_F32) {
        if (dk == 128) return split::run<float, 128>(q, k, v, beta, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dv, timeout_cycles, mode, w, ws_bytes, stream);
        if (dk == 64) return split::run<float, 64>(q, k, v, beta, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dv, timeout_cycles, mode, w, ws_bytes, stream);
    } else {
        if (dk == 128) return split::run<__nv_bfloat16, 128>(q, k, v, beta, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dv, timeout_cycles, mode, w, ws_bytes, stream);
        if (dk == 64) return split::run<__nv_bfloat16, 64>(q, k, v, beta, log_alpha, s0, o, sT, cu, nseq, T, tokens, H, dv, timeout_cycles, mode, w, ws_bytes, stream);
    }
    return cudaErrorInvalidValue;
}

bool chunk_fwd_noalloc_fits(int nseq, int T, int H, int dk, int dv, bool has_final)
{
    const int nch = (T + tcu::C - 1) / tcu::C;
    return dk == 128 ? split::noalloc_block<128>(nseq, H, dv, has_final, nch) > 0
                     : split::noalloc_block<64>(nseq, H, dv, has_final, nch) > 0;
}

cudaError_t chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* beta,
                              const float* log_alpha, const float* s0, void* o, float* sT, int nseq, int T,
                              long long tokens, int H, int dk, int dv, kda_dtype o_dtype, long long timeout_cycles,
                              cudaStream_t stream)
{
    if (o_dtype == KDA_F32) {
        if (dk == 128) return split::run_noalloc<float, 128>(q, k, v, beta, log_alpha, s0, o, sT, nseq, T, tokens, H, dv, timeout_cycles, stream);
        if (dk == 64) return split::run_noalloc<float, 64>(q, k, v, beta, log_alpha, s0, o, sT, nseq, T, tokens, H, dv, timeout_cycles, stream);
    } else {
        if (dk == 128) return split::run_noalloc<__nv_bfloat16, 128>(q, k, v, beta, log_alpha, s0, o, sT, nseq, T, tokens, H, dv, timeout_cycles, stream);
        if (dk == 64) return split::run_noalloc<__nv_bfloat16, 64>(q, k, v, beta, log_alpha, s0, o, sT, nseq, T, tokens, H, dv, timeout_cycles, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace kda
