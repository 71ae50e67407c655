// dispatch.cu -- a2: capacity-factor dispatch ("Llama 3 Meets MoE: Efficient
// Upcycling", section 3 "容量因子": expert capacity = tokens per batch / N x CF;
// overflow tokens are left out of the expert computation).
//
// A deterministic stable counting sort of the T*k (token, expert) assignments
// by expert, token-ascending inside an expert.  An assignment is kept iff its
// rank inside its expert is < C, so the lower token index wins.
//
//   count kernel: per 32-token chunk and expert, the number of tokens of the
//     chunk routed to the expert (one warp ballot per expert); the CTA that
//     finishes last then scans over chunks per expert -> the rank base of each
//     chunk and each expert's routed count.  (The tensor-core router does the
//     same in its gate epilogue, so a dispatch right after it skips this kernel.)
//   scatter kernel: kept = min(counts, C) and offsets = exclusive scan of kept;
//     each CTA takes an equal contiguous range of the 16-byte vectors of x, ranks
//     the tokens it touches (rank = chunk base + ballot prefix inside the chunk),
//     writes slot_row / row_token for the tokens whose first vector it holds, and
//     copies every x vector to each of the token's kept rows.
// No atomics decide any output, so every output is bit-reproducible.
#include "common.cuh"
#include "dispatch_scan.cuh"
#include "kernels.h"

#ifndef MOE_SCATTER_U
#define MOE_SCATTER_U 8  // row vectors loaded per thread before they are stored
#endif

namespace moe {

constexpr int kCountWarps = 8;         // chunks per count CTA
constexpr int kCountSmemInts = 8192;   // histogram entries the last CTA scans in shared memory
constexpr int kScatterMaxTok = 256;    // tokens of one scatter CTA (its row table)

struct SyncCta {
    __device__ void operator()() const { __syncthreads(); }
};

// Per-chunk expert counts (one warp ballot per expert and 32-token chunk), then, in
// whichever CTA finishes last, the exclusive scan over chunks per expert (rank base
// of every chunk) and the routed count of every expert (dcounts).  The last CTA is
// found with a ticket counter (threadfence + atomicAdd); it resets the counter, so
// the next launch on the stream starts from zero.  No thread ever waits on another
// CTA, and the outputs do not depend on which CTA happens to be last.
__global__ void __launch_bounds__(256) dispatch_count_kernel(
    const int32_t *__restrict__ idx, int T, int k, int E, int32_t *__restrict__ hist,
    int32_t *counter, int32_t *__restrict__ dcounts, int32_t *status)
{
    pdl_wait();
    pdl_trigger();
    __shared__ int s_last;
    __shared__ int32_t s_hist[kCountSmemInts];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nch = (T + kDispatchChunk - 1) / kDispatchChunk;
    const int c = blockIdx.x * kCountWarps + warp;
    if (c < nch) {
        const int64_t t = (int64_t)c * kDispatchChunk + lane;
        int ej[MOE_MAX_TOPK];
        for (int j = 0; j < k; ++j) {
            int e = -1;
            if (t < T) {
                e = idx[t * k + j];
                if (e < 0 || e >= E) {
                    set_status(status, MOE_ERR_DEVICE_BADINDEX);
                    e = -1;
                }
            }
            ej[j] = e;
        }
        for (int e = 0; e < E; ++e) {
            bool has = false;
            for (int j = 0; j < k; ++j)
                has |= ej[j] == e;
            const unsigned b = __ballot_sync(0xffffffffu, has);
            if (lane == (e & 31))
                hist[(int64_t)e * nch + c] = __popc(b);
        }
    }
    if (gridDim.x > 1) {
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0)
            s_last = atomicAdd(counter, 1) == (int)gridDim.x - 1;
        __syncthreads();
        if (!s_last)
            return;
        __threadfence();
    } else {
        __syncthreads();  // one CTA: its own writes are visible after the barrier
    }
    if (T == 0) {
        for (int e = threadIdx.x; e < E; e += blockDim.x)
            dcounts[e] = 0;
    } else {
        scan_chunk_counts(hist, E, nch, dcounts, s_hist, kCountSmemInts, threadIdx.x,
                          blockDim.x, SyncCta());
    }
    if (threadIdx.x == 0 && gridDim.x > 1)
        *counter = 0;
}

static unsigned count_grid(int T)
{
    const int nch = ceil_div(T, kDispatchChunk);
    const int g = ceil_div(nch, kCountWarps);
    return (unsigned)(g > 0 ? g : 1);
}

// kept / offsets from the routed counts, then, for the tokens [b*tpc, (b+1)*tpc) of
// CTA b (tpc <= kScatterMaxTok): their ranks, slot_row / row_token, and the copy of
// their rows of x into x_perm (x_perm NULL: tables only).
__global__ void __launch_bounds__(256) dispatch_scatter_kernel(
    const char *__restrict__ x, int64_t row_bytes, int T, int k, int E, int C,
    const int32_t *__restrict__ idx, const int32_t *__restrict__ bases,
    const int32_t *__restrict__ dcounts, char *__restrict__ x_perm,
    int32_t *__restrict__ row_token, int32_t *__restrict__ slot_row, int32_t *__restrict__ counts,
    int32_t *__restrict__ kept, int32_t *__restrict__ offsets, int tpc)
{
    pdl_trigger();  // early: the GEMM after it may prefetch its weights meanwhile
    pdl_wait();
    __shared__ int32_t s_cnt[MOE_MAX_EXPERTS];
    __shared__ int32_t s_kept[MOE_MAX_EXPERTS];
    __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1];
    __shared__ int32_t s_rows[kScatterMaxTok * MOE_MAX_TOPK];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        s_cnt[e] = dcounts[e];
    __syncthreads();
    if (warp == 0) {  // kept = min(count, C); offsets = exclusive scan of kept
        int32_t kp[2], incl[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = lane + 32 * h;
            const int32_t cnt = e < E ? s_cnt[e] : 0;
            kp[h] = (C < 0 || cnt < C) ? cnt : C;
            incl[h] = kp[h];
#pragma unroll
            for (int sh = 1; sh < 32; sh <<= 1) {
                const int32_t u = __shfl_up_sync(0xffffffffu, incl[h], sh);
                if (lane >= sh)
                    incl[h] += u;
            }
        }
        const int32_t tot0 = __shfl_sync(0xffffffffu, incl[0], 31);
        incl[1] += tot0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = lane + 32 * h;
            if (e < E) {
                s_kept[e] = kp[h];
                s_off[e + 1] = incl[h];
            }
        }
        if (lane == 0)
            s_off[0] = 0;
    }
    __syncthreads();
    if (blockIdx.x == 0) {
        for (int e = threadIdx.x; e < E; e += blockDim.x) {
            counts[e] = s_cnt[e];
            kept[e] = s_kept[e];
        }
        for (int e = threadIdx.x; e <= E; e += blockDim.x)
            offsets[e] = s_off[e];
    }
    if (T == 0)
        return;
    const int tb = blockIdx.x * tpc;                         // this CTA's tokens [tb, te)
    const int te = tb + tpc < T ? tb + tpc : T;
    if (tb >= te)
        return;
    const int nch = (T + kDispatchChunk - 1) / kDispatchChunk;
    const unsigned lt = (1u << lane) - 1u;
    // ranks of every token of the chunks this CTA touches (one warp per chunk)
    for (int c = tb / kDispatchChunk + warp; c <= (te - 1) / kDispatchChunk;
         c += blockDim.x >> 5) {
        const int t = c * kDispatchChunk + lane;
        // the chunk's rank base of every expert, fetched in one round of loads (lane l
        // holds experts l and l + 32)
        int32_t base_l[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = lane + 32 * h;
            base_l[h] = e < E ? __ldg(bases + (int64_t)e * nch + c) : 0;
        }
        int ej[MOE_MAX_TOPK], rowj[MOE_MAX_TOPK];
        for (int j = 0; j < k; ++j) {
            int e = -1;
            if (t < T) {
                e = idx[(int64_t)t * k + j];
                if (e < 0 || e >= E)
                    e = -1;  // reported by the kernel that counted
            }
            ej[j] = e;
            rowj[j] = -1;
        }
        for (int e = 0; e < E; ++e) {
            bool has = false;
            for (int j = 0; j < k; ++j)
                has |= ej[j] == e;
            const unsigned b = __ballot_sync(0xffffffffu, has);
            const int32_t ebase = __shfl_sync(0xffffffffu, e < 32 ? base_l[0] : base_l[1], e & 31);
            if (has) {
                const int32_t rank = ebase + __popc(b & lt);
                const int32_t row = rank < s_kept[e] ? s_off[e] + rank : -1;
                for (int j = 0; j < k; ++j)
                    if (ej[j] == e)
                        rowj[j] = row;
            }
        }
        if (t >= tb && t < te)
            for (int j = 0; j < k; ++j) {
                s_rows[(t - tb) * k + j] = rowj[j];
                slot_row[(int64_t)t * k + j] = rowj[j];
                if (rowj[j] >= 0)
                    row_token[rowj[j]] = t;
            }
    }
    if (x_perm == nullptr)
        return;
    __syncthreads();
    // the copy: one warp per token, each lane U 16-byte vectors of the row in flight
    // before they are stored to every kept row of the token
    constexpr int U = MOE_SCATTER_U;
    const int nv = (int)(row_bytes / 16);
    for (int t = tb + warp; t < te; t += blockDim.x >> 5) {
        int32_t rows[MOE_MAX_TOPK];
        bool any = false;
        for (int j = 0; j < k; ++j) {
            rows[j] = s_rows[(t - tb) * k + j];
            any |= rows[j] >= 0;
        }
        if (!any)
            continue;
        const char *src = x + (int64_t)t * row_bytes;
        for (int v0 = lane; v0 < nv; v0 += 32 * U) {
            uint4 val[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (v0 + 32 * u < nv)
                    val[u] = ld_nc_na(src + (int64_t)(v0 + 32 * u) * 16);
            for (int j = 0; j < k; ++j) {
                if (rows[j] < 0)
                    continue;
                char *dst = x_perm + (int64_t)rows[j] * row_bytes;
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (v0 + 32 * u < nv)
                        st_v4(dst + (int64_t)(v0 + 32 * u) * 16, val[u]);
            }
        }
    }
}

// CTAs of the scatter kernel that fit on the device at once (cached per device).
static int64_t scatter_wave()
{
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 148;
    if (cached[dev] == 0) {
        int sms = 0, per = 0;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, dispatch_scatter_kernel, 256, 0);
        cached[dev] = (sms > 0 ? sms : 148) * (per > 0 ? per : 1);
    }
    return cached[dev];
}

// The scatter launch shared by every dispatch entry point: `bases` / `dcounts` hold
// the scanned chunk histogram and the routed counts of topk_idx.
cudaError_t launch_scatter(const moe_params_t *p, const void *x, const int32_t *idx,
                           const int32_t *bases, const int32_t *dcounts, void *x_perm,
                           int32_t *row_token, int32_t *slot_row, int32_t *counts,
                           int32_t *kept, int32_t *offsets, cudaStream_t s)
{
    const int64_t row_bytes = (int64_t)p->d * (p->dtype == MOE_BF16 ? 2 : 4);
    // whole tokens per CTA: one wave when the row tables fit, more CTAs otherwise
    int64_t grid = scatter_wave();
    if (grid > p->T)
        grid = p->T;
    if (grid < 1)
        grid = 1;
    int64_t tpc = (p->T + grid - 1) / grid;
    if (tpc > kScatterMaxTok)
        tpc = kScatterMaxTok;
    if (tpc < 1)
        tpc = 1;
    grid = p->T > 0 ? (p->T + tpc - 1) / tpc : 1;
    launch_pdl(dispatch_scatter_kernel, dim3((unsigned)grid), dim3(256), 0, s,
               (const char *)x, row_bytes, p->T, p->k, p->E, p->capacity, idx, bases, dcounts,
               (char *)x_perm, row_token, slot_row, counts, kept, offsets, (int)tpc);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_count(const moe_params_t *p, const int32_t *idx, int32_t *hist,
                         int32_t *counter, int32_t *dcounts, int32_t *status, cudaStream_t s)
{
    launch_pdl(dispatch_count_kernel, dim3(count_grid(p->T)), dim3(256), 0, s, idx, p->T, p->k,
               p->E, hist, counter, dcounts, status);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_dispatch(const moe_params_t *p, const void *x, const int32_t *idx,
                            void *x_perm, int32_t *row_token, int32_t *slot_row,
                            int32_t *counts, int32_t *kept, int32_t *offsets, char *ws,
                            int32_t *status, bool routed, cudaStream_t s)
{
    const WsLayout L = ws_layout(p);
    int32_t *hist = reinterpret_cast<int32_t *>(ws + L.hist);
    int32_t *dcounts = reinterpret_cast<int32_t *>(ws + L.dcounts);
    int32_t *counter = reinterpret_cast<int32_t *>(ws) + kWsCounterWord;
    if (!routed) {
        cudaError_t e = launch_count(p, idx, hist, counter, dcounts, status, s);
        if (e != cudaSuccess)
            return e;
    }
    return launch_scatter(p, x, idx, hist, dcounts, x_perm, row_token, slot_row, counts, kept,
                          offsets, s);
}

}  // namespace moe

// ---------------------------------------------------------------------------
// Allocation-free dispatch.  Some callers cannot allocate device memory or hand
// the library a workspace -- for example a host engine whose plugin interface
// gives a layer only its input and output tensors and forbids allocation while
// it enqueues work, or a latency-critical loop that must never enter an
// allocator.  For them moe_dispatch_noalloc keeps the per-chunk histogram in a
// fixed array in device memory that is part of the library image itself: it is
// reserved on every GPU that loads libmoe.so and stays reserved until the
// process exits.  Every call reuses the same array, so calls whose kernels
// overlap on the GPU (different streams, different host threads) race and
// corrupt each other's results; serialise them.  The count kernel overwrites
// every histogram entry and routed count a call reads, so stale contents from an
// earlier call are never used, and it returns its ticket counter to zero (the
// array starts zeroed when the library loads).
#include <mutex>

namespace moe {

constexpr int kNoallocHistInts = 65536;  // 256 KiB of per-(expert, chunk) counts
constexpr int kNoallocTailInts = 128;    // word 1: ticket counter; words 64..127: routed counts
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoallocHistInts + kNoallocTailInts];

static std::mutex g_noalloc_mu;
static int32_t *g_noalloc_ptr[64] = {};

// Device address of g_noalloc_scratch on the current device (host code must not
// use the symbol itself: on the host it names a stand-in, not device memory).
static cudaError_t noalloc_scratch(int32_t **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess)
            return e;
        g_noalloc_ptr[dev] = static_cast<int32_t *>(ptr);
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}

}  // namespace moe

extern "C" int moe_dispatch_noalloc(const moe_params_t *p, const void *x,
                                    const int32_t *topk_idx, void *x_perm, int32_t *row_token,
                                    int32_t *slot_row, int32_t *counts, int32_t *kept,
                                    int32_t *offsets, int32_t *status, void *stream)
{
    using namespace moe;
    const char *fn = "moe_dispatch_noalloc";
    int rc = validate_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    const void *tok[] = {x, topk_idx, x_perm, row_token, slot_row};
    const void *exp_[] = {counts, kept, offsets};
    for (const void *q : tok)
        if ((q == nullptr && p->T > 0) || (reinterpret_cast<uintptr_t>(q) & 15u))
            return report_error(q == nullptr ? MOE_ERR_INVALID_ARG : MOE_ERR_ALIGN,
                                "moe_dispatch_noalloc: a token buffer is NULL or not 16-byte "
                                "aligned");
    for (const void *q : exp_)
        if (q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15u))
            return report_error(q == nullptr ? MOE_ERR_INVALID_ARG : MOE_ERR_ALIGN,
                                "moe_dispatch_noalloc: counts/kept/offsets is NULL or not "
                                "16-byte aligned");
    const int64_t chunks = ceil_div(p->T > 0 ? p->T : 1, kDispatchChunk);
    if ((int64_t)p->E * chunks > kNoallocHistInts)
        return report_error(MOE_ERR_SHAPE,
                            "moe_dispatch_noalloc: E * ceil(T/32) exceeds the fixed scratch of "
                            "65536 entries (e.g. T <= 32768 at E = 64, T <= 262144 at E = 8)");
    // a device-side index error is reported through `status` only, so it is required
    // whenever there is a token whose index could be bad
    if (status == nullptr && p->T > 0)
        return report_error(MOE_ERR_INVALID_ARG,
                            "moe_dispatch_noalloc: status is NULL (required for T > 0: it is "
                            "the only place a bad expert index is reported)");
    if (reinterpret_cast<uintptr_t>(status) & 3u)
        return report_error(MOE_ERR_ALIGN, "moe_dispatch_noalloc: status is not 4-byte aligned");
    int32_t *scratch = nullptr;
    cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess)
        return report_cuda(e, fn);
    int32_t *hist = scratch;
    int32_t *counter = scratch + kNoallocHistInts + 1;  // zero at load, reset by every call
    int32_t *dcounts = scratch + kNoallocHistInts + 64;  // written by every call before use
    cudaStream_t s = (cudaStream_t)stream;
    e = launch_count(p, topk_idx, hist, counter, dcounts, status, s);
    if (e == cudaSuccess)
        e = launch_scatter(p, x, topk_idx, hist, dcounts, x_perm, row_token, slot_row, counts,
                           kept, offsets, s);
    return e == cudaSuccess ? report_ok() : report_cuda(e, fn);
}
