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
//     chunk; counts, kept = min(counts, C), offsets = exclusive scan of kept.
//   rank kernel (one warp per chunk): each assignment's rank = chunk base + ballot
//     prefix inside the chunk -> slot_row / row_token.
//   copy kernel: every x row is read once (16-byte loads) and written to each of
//     its kept rows; equal contiguous work ranges for a grid that fills the device.
// No atomics decide any output, so every output is bit-reproducible.
#include "common.cuh"
#include "kernels.h"

#ifndef MOE_SCATTER_U
#define MOE_SCATTER_U 8  // row vectors loaded per thread before they are stored
#endif

namespace moe {

constexpr int kCountWarps = 8;         // chunks per count CTA
constexpr int kCountSmemInts = 8192;   // histogram entries the last CTA scans in shared memory

// Per-chunk expert counts (one warp ballot per expert and 32-token chunk), then, in
// whichever CTA finishes last, the exclusive scan over chunks per expert (rank base
// of every chunk), counts, kept = min(counts, C) and offsets.  The last CTA is
// found with a ticket counter (threadfence + atomicAdd); it resets the counter, so
// the next launch on the stream starts from zero.  No thread ever waits on another
// CTA, and the outputs do not depend on which CTA happens to be last.
__global__ void __launch_bounds__(256) dispatch_count_kernel(
    const int32_t *__restrict__ idx, int T, int k, int E, int C, int32_t *__restrict__ hist,
    int32_t *counter, int32_t *__restrict__ counts, int32_t *__restrict__ kept,
    int32_t *__restrict__ offsets, int32_t *status)
{
    pdl_wait();
    pdl_trigger();
    __shared__ int s_last;
    __shared__ int32_t s_count[MOE_MAX_EXPERTS];
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
    // exclusive scan over chunks, one warp per expert; lane l owns a contiguous run.
    // The histogram is staged in shared memory with coalesced loads when it fits.
    const int per = (nch + 31) / 32;
    const int64_t nhist = (int64_t)E * nch;
    const bool staged = nhist <= kCountSmemInts;
    if (staged) {
        for (int64_t i = threadIdx.x; i < nhist; i += blockDim.x)
            s_hist[i] = __ldcg(hist + i);
        __syncthreads();
    }
    for (int e = warp; e < E; e += kCountWarps) {
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
        const int32_t total = __shfl_sync(0xffffffffu, incl, 31);
        if (lane == 0)
            s_count[e] = total;
    }
    __syncthreads();
    if (staged)  // the chunk bases go back to global memory for the rank kernel
        for (int64_t i = threadIdx.x; i < nhist; i += blockDim.x)
            hist[i] = s_hist[i];
    if (threadIdx.x == 0) {
        int32_t off = 0;
        offsets[0] = 0;
        for (int e = 0; e < E; ++e) {
            const int32_t cnt = s_count[e];
            const int32_t kp = (C < 0 || cnt < C) ? cnt : C;
            counts[e] = cnt;
            kept[e] = kp;
            off += kp;
            offsets[e + 1] = off;
        }
        if (gridDim.x > 1)
            *counter = 0;
    }
}

static unsigned count_grid(int T)
{
    const int nch = ceil_div(T, kDispatchChunk);
    const int g = ceil_div(nch, kCountWarps);
    return (unsigned)(g > 0 ? g : 1);
}

// Ranks of one 32-token chunk per warp: rank = chunk base + ballot prefix inside
// the chunk; writes slot_row and row_token.
__global__ void __launch_bounds__(256) dispatch_rank_kernel(
    const int32_t *__restrict__ idx, int T, int k, int E, const int32_t *__restrict__ hist,
    const int32_t *__restrict__ kept, const int32_t *__restrict__ offsets,
    int32_t *__restrict__ row_token, int32_t *__restrict__ slot_row)
{
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nch = (T + kDispatchChunk - 1) / kDispatchChunk;
    const int c = blockIdx.x * (blockDim.x >> 5) + warp;
    if (c >= nch)
        return;
    const int64_t t = (int64_t)c * kDispatchChunk + lane;
    const unsigned lt = (1u << lane) - 1u;
    // the chunk's rank base, kept count and first row of every expert, fetched in one
    // round of loads (lane l holds experts l and l + 32)
    int32_t base_l[2], kept_l[2], off_l[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int e = lane + 32 * h;
        base_l[h] = e < E ? hist[(int64_t)e * nch + c] : 0;
        kept_l[h] = e < E ? kept[e] : 0;
        off_l[h] = e < E ? offsets[e] : 0;
    }
    int ej[MOE_MAX_TOPK], rowj[MOE_MAX_TOPK];
    for (int j = 0; j < k; ++j) {
        int e = -1;
        if (t < T) {
            e = idx[t * k + j];
            if (e < 0 || e >= E)
                e = -1;  // reported by the count kernel
        }
        ej[j] = e;
        rowj[j] = -1;
    }
    for (int e = 0; e < E; ++e) {
        bool has = false;
        for (int j = 0; j < k; ++j)
            has |= ej[j] == e;
        const unsigned b = __ballot_sync(0xffffffffu, has);
        const int h = e >> 5, src = e & 31;
        const int32_t ebase = __shfl_sync(0xffffffffu, h ? base_l[1] : base_l[0], src);
        const int32_t ekept = __shfl_sync(0xffffffffu, h ? kept_l[1] : kept_l[0], src);
        const int32_t eoff = __shfl_sync(0xffffffffu, h ? off_l[1] : off_l[0], src);
        if (has) {
            const int32_t rank = ebase + __popc(b & lt);
            const int32_t row = rank < ekept ? eoff + rank : -1;
            for (int j = 0; j < k; ++j)
                if (ej[j] == e)
                    rowj[j] = row;
        }
    }
    if (t < T)
        for (int j = 0; j < k; ++j) {
            slot_row[t * k + j] = rowj[j];
            if (rowj[j] >= 0)
                row_token[rowj[j]] = (int32_t)t;
        }
}

// x_perm[slot_row[t][j]] = x[t] for every kept slot.  The T * (row bytes / 16)
// vector items are split into equal contiguous ranges, one per CTA of a grid that
// fills the device once; each thread issues U loads before their stores.
__global__ void __launch_bounds__(256) dispatch_copy_kernel(const char *__restrict__ x,
                                                            int64_t row_bytes, int T, int k,
                                                            const int32_t *__restrict__ slot_row,
                                                            char *__restrict__ x_perm)
{
    pdl_wait();
    pdl_trigger();
    const int64_t nv = row_bytes / 16;
    const int64_t items = (int64_t)T * nv;
    const int64_t per = (items + gridDim.x - 1) / gridDim.x;
    const int64_t i0 = (int64_t)blockIdx.x * per;
    const int64_t i1 = i0 + per < items ? i0 + per : items;
    constexpr int U = MOE_SCATTER_U;
    for (int64_t base = i0 + threadIdx.x; base < i1; base += (int64_t)blockDim.x * U) {
        uint4 val[U];
        int tv[U], vv[U];  // token and vector of each item (T < 2^31, nv < 2^17)
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = base + (int64_t)u * blockDim.x;
            tv[u] = -1;
            if (i < i1) {
                tv[u] = (int)(i / nv);
                vv[u] = (int)(i - (int64_t)tv[u] * nv);
                val[u] = ld_nc_na(x + (int64_t)tv[u] * row_bytes + (int64_t)vv[u] * 16);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (tv[u] < 0)
                continue;
            for (int j = 0; j < k; ++j) {
                const int32_t row = slot_row[(int64_t)tv[u] * k + j];
                if (row >= 0)
                    st_v4(x_perm + (int64_t)row * row_bytes + (int64_t)vv[u] * 16, val[u]);
            }
        }
    }
}

// CTAs of the copy kernel that fit on the device at once (cached per device).
static unsigned copy_wave()
{
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 148;
    if (cached[dev] == 0) {
        int sms = 0, per = 0;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, dispatch_copy_kernel, 256, 0);
        cached[dev] = (sms > 0 ? sms : 148) * (per > 0 ? per : 1);
    }
    return (unsigned)cached[dev];
}

// rank + copy launches shared by moe_dispatch and moe_dispatch_noalloc
static cudaError_t launch_rank_copy(const moe_params_t *p, const void *x, const int32_t *idx,
                                    const int32_t *hist, const int32_t *kept,
                                    const int32_t *offsets, void *x_perm, int32_t *row_token,
                                    int32_t *slot_row, cudaStream_t s)
{
    const int nch = ceil_div(p->T, kDispatchChunk);
    launch_pdl(dispatch_rank_kernel, dim3(ceil_div(nch, 8)), dim3(256), 0, s, idx, p->T, p->k, p->E, hist, kept,
                                                          offsets, row_token, slot_row);
    count_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || x_perm == nullptr)
        return e;
    const int64_t row_bytes = (int64_t)p->d * (p->dtype == MOE_BF16 ? 2 : 4);
    const int64_t items = (int64_t)p->T * (row_bytes / 16);
    const int64_t min_per = 256;  // at least one vector per thread per CTA
    int64_t grid = (items + min_per - 1) / min_per;
    if (grid > copy_wave())
        grid = copy_wave();
    launch_pdl(dispatch_copy_kernel, dim3((unsigned)grid), dim3(256), 0, s, (const char *)x, row_bytes, p->T, p->k,
                                                         slot_row, (char *)x_perm);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_dispatch(const moe_params_t *p, const void *x, const int32_t *idx,
                            void *x_perm, int32_t *row_token, int32_t *slot_row,
                            int32_t *counts, int32_t *kept, int32_t *offsets, char *ws,
                            int32_t *status, cudaStream_t s)
{
    const WsLayout L = ws_layout(p);
    int32_t *hist = reinterpret_cast<int32_t *>(ws + L.hist);
    int32_t *counter = reinterpret_cast<int32_t *>(ws) + kWsCounterWord;
    launch_pdl(dispatch_count_kernel, dim3(count_grid(p->T)), dim3(256), 0, s, idx, p->T, p->k, p->E, p->capacity,
                                                           hist, counter, counts, kept, offsets,
                                                           status);
    count_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || p->T == 0)
        return e;
    return launch_rank_copy(p, x, idx, hist, kept, offsets, x_perm, row_token, slot_row, s);
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
// every histogram entry a call reads, so stale contents from an earlier call
// are never used, and it returns its ticket counter to zero (the array starts
// zeroed when the library loads).
#include <mutex>

namespace moe {

constexpr int kNoallocHistInts = 65536;  // 256 KiB of per-(expert, chunk) counts
constexpr int kNoallocStatusInts = 64;   // status word used when the caller passes none
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoallocHistInts + kNoallocStatusInts];

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
    int32_t *scratch = nullptr;
    cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess)
        return report_cuda(e, fn);
    int32_t *hist = scratch;
    int32_t *st = status != nullptr ? status : scratch + kNoallocHistInts;
    int32_t *counter = scratch + kNoallocHistInts + 1;  // zero at load, reset by every call
    cudaStream_t s = (cudaStream_t)stream;
    launch_pdl(dispatch_count_kernel, dim3(count_grid(p->T)), dim3(256), 0, s, topk_idx, p->T, p->k, p->E,
                                                           p->capacity, hist, counter, counts,
                                                           kept, offsets, st);
    count_launch();
    e = cudaGetLastError();
    if (e == cudaSuccess && p->T > 0)
        e = launch_rank_copy(p, x, topk_idx, hist, kept, offsets, x_perm, row_token, slot_row, s);
    return e == cudaSuccess ? report_ok() : report_cuda(e, fn);
}
