// dispatch_scan.cuh -- the per-expert scan over 32-token chunks that turns the
// chunk histogram of a2 (capacity dispatch, "Llama 3 Meets MoE: Efficient
// Upcycling", section 3 "容量因子") into rank bases.  Shared by the dispatch
// count kernel and the tensor-core router, whose gate epilogue counts the chunks
// of the tokens it has just routed.
#pragma once

#include "common.cuh"

namespace moe {

// Copies n 32-bit words from global memory (written by other CTAs, read at L2) to
// shared memory, the nthr calling threads striding by nthr: every thread issues
// kStageBatch loads before it stores any, so the copy takes a few L2 round trips
// instead of one per word a thread handles.
constexpr int kStageBatch = 8;
template <typename W>
__device__ __forceinline__ void stage_words(W *dst, const W *src, int64_t n, int tid, int nthr)
{
    for (int64_t i0 = tid; i0 < n; i0 += (int64_t)nthr * kStageBatch) {
        W v[kStageBatch];
#pragma unroll
        for (int u = 0; u < kStageBatch; ++u) {
            const int64_t i = i0 + (int64_t)u * nthr;
            if (i < n)
                v[u] = __ldcg(src + i);
        }
#pragma unroll
        for (int u = 0; u < kStageBatch; ++u) {
            const int64_t i = i0 + (int64_t)u * nthr;
            if (i < n)
                dst[i] = v[u];
        }
    }
}

// hist [E][nch]: on entry the number of tokens of chunk c routed to expert e; on
// exit the exclusive prefix over chunks (the rank inside expert e of the chunk's
// first such token).  dcounts [E] receives each expert's total (its routed count).
// Run by the nthr threads (whole warps) of one CTA, tid = 0..nthr-1; `bar`
// synchronises exactly those threads.  The histogram is staged in shared memory
// (s_hist, room for smem_ints entries) when it fits, with coalesced loads; the
// scan of an expert is one warp, lane l owning a contiguous run of chunks.  Every
// sum is over integers, so the result does not depend on nthr.
template <class Bar>
__device__ __forceinline__ void scan_chunk_counts(int32_t *hist, int E, int nch,
                                                  int32_t *dcounts, int32_t *s_hist,
                                                  int64_t smem_ints, int tid, int nthr, Bar bar)
{
    const int warp = tid >> 5, lane = tid & 31, nwarps = nthr >> 5;
    const int per = (nch + 31) / 32;
    const int64_t nhist = (int64_t)E * nch;
    const bool staged = nhist <= smem_ints;
    if (staged) {
        stage_words(s_hist, hist, nhist, tid, nthr);
        bar();
    }
    for (int e = warp; e < E; e += nwarps) {
        int32_t *h = staged ? s_hist + (int64_t)e * nch : hist + (int64_t)e * nch;
        const int c0 = lane * per, c1 = min(nch, c0 + per);
        int32_t sum = 0;
#pragma unroll 8
        for (int cc = c0; cc < c1; ++cc)
            sum += staged ? h[cc] : __ldcg(h + cc);
        int32_t incl = sum;
#pragma unroll
        for (int sh = 1; sh < 32; sh <<= 1) {
            const int32_t u = __shfl_up_sync(0xffffffffu, incl, sh);
            if (lane >= sh)
                incl += u;
        }
        int32_t run = incl - sum;
        for (int cc = c0; cc < c1; ++cc) {
            const int32_t v = staged ? h[cc] : __ldcg(h + cc);
            h[cc] = run;
            run += v;
        }
        if (lane == 31)
            dcounts[e] = incl;
    }
    bar();
    if (staged)  // the chunk bases go back to global memory for the scatter kernel
        for (int64_t i = tid; i < nhist; i += nthr)
            hist[i] = s_hist[i];
}

}  // namespace moe
