// Chunk indexing of dense and packed (variable-length) batches for the
// kernels that keep one record per (chunk, head) in a caller workspace.
//
// Dense: nseq sequences of T tokens, nch = ceil(T / 64) chunks each; record
// (n, c) = n * nch + c; state slots (n, c) = n * (nch + 1) + c.
// Packed: the chunks of sequence n are numbered from choff[n] (a prefix sum
// of seq_chunks, computed on the device); state slots choff[n] + n + c.  A
// sequence whose token range leaves [0, tokens), or whose records would not
// fit the workspace, has no chunks in any kernel and is reported.
#pragma once

#include "kda_common.cuh"
#include "kda_sm100.cuh"

namespace kda {

namespace packed {

constexpr int C = 64;

// Chunks of packed sequence i: none for a decreasing pair or a token range
// that leaves [0, tokens).
__device__ __forceinline__ int seq_chunks(const int32_t* cu, int i, long long tokens)
{
    const int a = cu[i], b = cu[i + 1];
    if (b <= a || a < 0 || (long long)b > tokens) return 0;
    return (b - a + C - 1) / C;
}

// choff[i] = sum_{j<i} seq_chunks(j), choff[nseq] = the total.  One CTA; each
// thread sums a contiguous range of sequences, then a block-wide scan.
__global__ void __launch_bounds__(1024) chunk_offsets_kernel(const int32_t* cu, int nseq, long long tokens,
                                                             int32_t* choff)
{
    __shared__ int warp_tot[32];
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int per = (nseq + 1023) / 1024;
    const int a = min(nseq, tid * per), b = min(nseq, a + per);
    int local = 0;
    for (int i = a; i < b; ++i) local += seq_chunks(cu, i, tokens);
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
        base += seq_chunks(cu, i, tokens);
    }
    if (tid == 1023) choff[nseq] = base;
}

struct Layout {
    const int32_t* cu;       // packed boundaries [nseq + 1], or nullptr (dense)
    const int32_t* choff;    // packed: first record of each sequence [nseq + 1]
    long long tokens;        // length of the token axis
    long long nrec;          // records per head the workspace holds
    int nseq, T, nch, H;     // dense: T tokens and nch chunks per sequence
};

// Records per head a call needs (an upper bound for packed batches).
inline long long records(int nseq, int T, long long tokens, bool varlen)
{
    return varlen ? tokens / C + nseq : (long long)nseq * ((T + C - 1) / C);
}

// State slots per head: one entering every chunk plus the final one.
inline long long state_slots(int nseq, int T, long long tokens, bool varlen)
{
    return varlen ? tokens / C + 2LL * nseq : (long long)nseq * ((T + C - 1) / C + 1);
}

// Position of one (record, head) item, item = record * H + head.
struct Pos {
    long long rc;     // record (chunk) index
    long long slot;   // state slot of the state entering the chunk
    int n, tok, L, h;
    bool ok;
};

__device__ __forceinline__ Pos locate(const Layout& g, long long item)
{
    Pos x{};
    x.h = (int)(item % g.H);
    x.rc = item / g.H;
    x.ok = false;
    if (g.cu) {
        if (x.rc >= g.choff[g.nseq]) return x;
        int lo = 0, hi = g.nseq - 1;   // the last sequence whose first record is <= rc
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (g.choff[mid] <= x.rc) lo = mid;
            else hi = mid - 1;
        }
        const int nc = seq_chunks(g.cu, lo, g.tokens);
        if (nc == 0 || g.choff[lo] + nc > g.nrec) return x;   // skipped by every kernel
        const int t0 = g.cu[lo], len = g.cu[lo + 1] - t0;
        const int c = (int)(x.rc - g.choff[lo]);
        x.n = lo;
        x.tok = t0 + c * C;
        x.L = min(C, len - c * C);
        x.slot = (long long)g.choff[lo] + lo + c;
    } else {
        const int c = (int)(x.rc % g.nch);
        x.n = (int)(x.rc / g.nch);
        x.tok = x.n * g.T + c * C;
        x.L = min(C, g.T - c * C);
        x.slot = (long long)x.n * (g.nch + 1) + c;
    }
    x.ok = x.L > 0;
    return x;
}

// Walk range of sequence n: first token, length, first record and state
// slot.  A skipped packed sequence gets length 0, and has_slots tells whether
// its slot index is still inside the workspace.
struct Walk {
    int tok0, len;
    long long rbase, sbase;
    bool has_slots;
};

__device__ __forceinline__ Walk walk_of(const Layout& g, int n, bool report)
{
    Walk w{};
    w.has_slots = true;
    if (g.cu) {
        const int a = g.cu[n], b = g.cu[n + 1];
        w.tok0 = a;
        w.len = max(0, b - a);
        w.rbase = g.choff[n];
        w.sbase = w.rbase + n;
        const bool bad = w.len > 0 && (a < 0 || (long long)b > g.tokens);
        if (bad || w.rbase + (w.len + C - 1) / C > g.nrec) {
            if (report && threadIdx.x == 0) flag_bad_input();
            w.tok0 = 0;
            w.len = 0;
            w.has_slots = !bad && w.rbase <= g.nrec;
        }
    } else {
        w.tok0 = n * g.T;
        w.len = g.T;
        w.rbase = (long long)n * g.nch;
        w.sbase = (long long)n * (g.nch + 1);
    }
    return w;
}

// Loads rows [0, L) of a [64][D] tile of TIn elements (row r at
// src + r * stride elements, rows 16-byte aligned) into shared memory as
// floats with row pitch ld; rows >= L become zero.  Every load of a thread is
// issued before its first store.  NTHR threads take part.
template <typename TIn, int D, int NTHR>
__device__ __forceinline__ void load_rows(float* dst, int ld, const TIn* src, size_t stride, int L)
{
    constexpr int EPV = 16 / (int)sizeof(TIn);   // elements per 16-byte vector
    constexpr int VPR = D / EPV;                 // vectors per row
    constexpr int N = C * VPR / NTHR;            // vectors per thread
    static_assert(C * VPR % NTHR == 0, "tile not a multiple of the CTA");
    uint4 x[N];
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const int e = threadIdx.x + i * NTHR, r = e / VPR;
        x[i] = r < L ? __ldg(reinterpret_cast<const uint4*>(src + (size_t)r * stride + (e % VPR) * EPV))
                     : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const int e = threadIdx.x + i * NTHR;
        float* d = dst + (e / VPR) * ld + (e % VPR) * EPV;
        const TIn* xv = reinterpret_cast<const TIn*>(&x[i]);
#pragma unroll
        for (int u = 0; u < EPV; ++u) d[u] = Elem<TIn>::load(xv + u);
    }
}

// Record streaming: bulk copies of record parts into shared memory that
// complete on an mbarrier (one phase per fetch), waited for with a bound.
constexpr long long kWaitCycles = 1LL << 31;   // about 1 s at the B200 clock

// One thread: copies `bytes` (a multiple of 16; both addresses 16-byte
// aligned) in pieces of at most 32 KB, all completing on `bar`.  The fence
// orders this CTA's earlier generic accesses of dst before the async writes.
__device__ __forceinline__ void fetch(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    sm100::fence_proxy_async();
    sm100::mbar_expect_tx(bar, bytes);
    for (uint32_t off = 0; off < bytes; off += 32768u)
        sm100::bulk_load(static_cast<char*>(dst) + off, static_cast<const char*>(src) + off,
                         min(32768u, bytes - off), bar);
}

// Per-CTA state of up to two streamed parts.  issued[i] / done[i] count the
// fetches of part i that were issued / seen complete by thread 0.
struct Stream {
    uint64_t bar[2];
    int issued[2], done[2];
    int abort;
};

__device__ __forceinline__ void stream_init(Stream& st)
{
    if (threadIdx.x == 0) {
        sm100::mbar_init(&st.bar[0], 1);
        sm100::mbar_init(&st.bar[1], 1);
        st.issued[0] = st.issued[1] = st.done[0] = st.done[1] = 0;
        st.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
}

__device__ __forceinline__ void stream_fetch(Stream& st, int i, void* dst, const void* src, uint32_t bytes)
{
    fetch(dst, src, bytes, &st.bar[i]);
    ++st.issued[i];
}

// Every thread waits for fetch number `k` (0-based) of part i; returns false
// for every thread of the CTA if any thread's wait ran out (status word set).
__device__ __forceinline__ bool stream_wait(Stream& st, int i, int k)
{
    const bool ok = sm100::mbar_wait(&st.bar[i], (uint32_t)(k & 1), &st.abort, kWaitCycles);
    if (threadIdx.x == 0 && ok) st.done[i] = k + 1;
    return !__syncthreads_or(!ok);
}

// After a failed wait: thread 0 waits (bounded again) for the copies still in
// flight, so that none lands in shared memory after the CTA has exited.
__device__ __forceinline__ void stream_drain(Stream& st)
{
    if (threadIdx.x == 0) {
        volatile int never = 0;
        for (int i = 0; i < 2; ++i)
            for (int k = st.done[i]; k < st.issued[i]; ++k)
                if (!sm100::mbar_wait(&st.bar[i], (uint32_t)(k & 1), &never, kWaitCycles)) break;
    }
    __syncthreads();
}

}  // namespace packed

}  // namespace kda
