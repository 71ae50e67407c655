// pipeline.cu -- host-buffer pipeline around moe_forward (no kernels here).
//
// Three streams per pipeline: h2d (copy engine in), compute (the layer), d2h
// (copy engine out).  Batch i uses slot s = i % depth; the per-slot events
// chain the streams so that
//   h2d(i)     waits until compute(i - depth) has consumed x/noise of slot s,
//   compute(i) waits until h2d(i) landed and d2h(i - depth) emptied y of slot s,
//   d2h(i)     waits until compute(i) finished.
// The intermediates are shared by all slots because compute runs one batch at a
// time on its own stream.  So is the workspace's status word: after each batch
// the compute stream moves it into the slot's own device word and clears it, so
// every batch reports only what its own kernels recorded.
#include <cstring>
#include <new>

#include "common.cuh"
#include "kernels.h"
#include "moe_pipeline.h"

struct moe_pipeline {
    moe_params_t p;
    int depth = 0;
    int device = -1;
    const void *Wg = nullptr, *Wnoise = nullptr, *W13_e = nullptr, *W2_e = nullptr;
    const float *bias = nullptr;
    cudaStream_t h2d = nullptr, compute = nullptr, d2h = nullptr;
    cudaEvent_t in_ready[MOE_PIPELINE_MAX_DEPTH] = {};
    cudaEvent_t consumed[MOE_PIPELINE_MAX_DEPTH] = {};
    cudaEvent_t out_done[MOE_PIPELINE_MAX_DEPTH] = {};
    int64_t slot_ticket[MOE_PIPELINE_MAX_DEPTH] = {};
    void *arena = nullptr;
    int32_t *host_status = nullptr;  // pinned, one word per ticket modulo MOE_PIPELINE_STATUS_RING
    int32_t *dev_status[MOE_PIPELINE_MAX_DEPTH] = {};  // the slot's batch's status word
    void *x[MOE_PIPELINE_MAX_DEPTH] = {};
    float *noise[MOE_PIPELINE_MAX_DEPTH] = {};
    void *y[MOE_PIPELINE_MAX_DEPTH] = {};
    float *loss[MOE_PIPELINE_MAX_DEPTH] = {};
    moe_buffers_t shared{};  // intermediates and statistics
    void *ws = nullptr;
    size_t ws_bytes = 0;
    size_t x_bytes = 0, noise_bytes = 0;
    int64_t next_ticket = 0;
    bool broken = false;
};

namespace moe {

static size_t up256(size_t n) { return (n + 255) / 256 * 256; }

static int pl_cuda(moe_pipeline_t *pl, cudaError_t e, const char *where)
{
    if (pl != nullptr)
        pl->broken = true;
    return report_cuda(e, where);
}

static void release(moe_pipeline_t *pl)
{
    for (int s = 0; s < MOE_PIPELINE_MAX_DEPTH; ++s) {
        if (pl->in_ready[s])
            cudaEventDestroy(pl->in_ready[s]);
        if (pl->consumed[s])
            cudaEventDestroy(pl->consumed[s]);
        if (pl->out_done[s])
            cudaEventDestroy(pl->out_done[s]);
    }
    if (pl->h2d)
        cudaStreamDestroy(pl->h2d);
    if (pl->compute)
        cudaStreamDestroy(pl->compute);
    if (pl->d2h)
        cudaStreamDestroy(pl->d2h);
    if (pl->arena)
        cudaFree(pl->arena);
    if (pl->host_status)
        cudaFreeHost(pl->host_status);
    delete pl;
}

}  // namespace moe

using namespace moe;

extern "C" {

int moe_pipeline_create(const moe_params_t *p, const void *Wg, const void *Wnoise,
                        const float *bias, const void *W13_e, const void *W2_e, int32_t depth,
                        moe_pipeline_t **out)
{
    const char *fn = "moe_pipeline_create";
    if (out == nullptr)
        return report_error(MOE_ERR_INVALID_ARG, "moe_pipeline_create: out is NULL");
    *out = nullptr;
    int rc = validate_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    if (p->T < 1)
        return report_error(MOE_ERR_INVALID_ARG, "moe_pipeline_create: T must be >= 1");
    if (depth < 2 || depth > MOE_PIPELINE_MAX_DEPTH)
        return report_error(MOE_ERR_INVALID_ARG,
                            "moe_pipeline_create: depth must be in [2, MOE_PIPELINE_MAX_DEPTH]");
    if (Wg == nullptr || W13_e == nullptr || W2_e == nullptr)
        return report_error(MOE_ERR_INVALID_ARG,
                            "moe_pipeline_create: Wg, W13_e and W2_e are required");

    moe_pipeline_t *pl = new (std::nothrow) moe_pipeline_t();
    if (pl == nullptr)
        return report_error(MOE_ERR_INVALID_ARG, "moe_pipeline_create: out of host memory");
    pl->p = *p;
    pl->depth = depth;
    pl->Wg = Wg;
    pl->Wnoise = Wnoise;
    pl->bias = bias;
    pl->W13_e = W13_e;
    pl->W2_e = W2_e;

    cudaError_t e = cudaGetDevice(&pl->device);
#define PL_TRY(call)                                                                           \
    do {                                                                                       \
        if (e == cudaSuccess)                                                                  \
            e = (call);                                                                        \
    } while (0)
    for (int s = 0; s < depth; ++s) {
        PL_TRY(cudaEventCreateWithFlags(&pl->in_ready[s], cudaEventDisableTiming));
        PL_TRY(cudaEventCreateWithFlags(&pl->consumed[s], cudaEventDisableTiming));
        PL_TRY(cudaEventCreateWithFlags(&pl->out_done[s], cudaEventDisableTiming));
    }
    PL_TRY(cudaStreamCreateWithFlags(&pl->h2d, cudaStreamNonBlocking));
    PL_TRY(cudaStreamCreateWithFlags(&pl->compute, cudaStreamNonBlocking));
    PL_TRY(cudaStreamCreateWithFlags(&pl->d2h, cudaStreamNonBlocking));
    PL_TRY(cudaHostAlloc((void **)&pl->host_status,
                         sizeof(int32_t) * MOE_PIPELINE_STATUS_RING, cudaHostAllocDefault));
    if (e != cudaSuccess) {
        release(pl);
        return report_cuda(e, fn);
    }

    // one arena: per-slot inputs/outputs, then the shared intermediates, then the workspace
    const size_t T = (size_t)p->T, d = (size_t)p->d, E = (size_t)p->E, k = (size_t)p->k;
    const size_t es = p->dtype == MOE_BF16 ? 2 : 4;
    const size_t rows = T * k, m8 = (size_t)round_up(p->m, 8);
    pl->x_bytes = T * d * es;
    pl->noise_bytes = Wnoise != nullptr ? T * E * sizeof(float) : 0;
    pl->ws_bytes = moe_workspace_size(p);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += up256(bytes > 0 ? bytes : 1);
        return o;
    };
    size_t o_x[MOE_PIPELINE_MAX_DEPTH], o_n[MOE_PIPELINE_MAX_DEPTH], o_y[MOE_PIPELINE_MAX_DEPTH],
        o_l[MOE_PIPELINE_MAX_DEPTH], o_st[MOE_PIPELINE_MAX_DEPTH];
    for (int s = 0; s < depth; ++s) {
        o_x[s] = take(pl->x_bytes);
        o_n[s] = take(pl->noise_bytes);
        o_y[s] = take(pl->x_bytes);
        o_l[s] = take(sizeof(float));
        o_st[s] = take(sizeof(int32_t));
    }
    const size_t o_counts = take(E * 4), o_imp = take(E * 4), o_f = take(E * 4),
                 o_P = take(E * 4), o_idx = take(T * k * 4), o_w = take(T * k * 4),
                 o_ps = take(E * 4), o_xp = take(rows * d * es), o_rt = take(rows * 4),
                 o_sr = take(T * k * 4), o_kept = take(E * 4), o_off = take((E + 1) * 4),
                 o_h = take(rows * m8 * es), o_out = take(rows * d * es),
                 o_ws = take(pl->ws_bytes);
    // the router weights packed once (they stay unchanged until destroy)
    const bool pack = p->dtype == MOE_BF16;
    const size_t o_wt =
        take(pack ? (size_t)router_packed_rows(p->E, Wnoise != nullptr) * d * es : 0);
    PL_TRY(cudaMalloc(&pl->arena, off));
    if (e != cudaSuccess) {
        release(pl);
        return report_cuda(e, fn);
    }
    char *a = (char *)pl->arena;
    for (int s = 0; s < depth; ++s) {
        pl->x[s] = a + o_x[s];
        pl->noise[s] = pl->noise_bytes ? (float *)(a + o_n[s]) : nullptr;
        pl->y[s] = a + o_y[s];
        pl->loss[s] = (float *)(a + o_l[s]);
        pl->dev_status[s] = (int32_t *)(a + o_st[s]);
        pl->slot_ticket[s] = -1;
    }
    moe_buffers_t &b = pl->shared;
    b.Wg = Wg;
    b.Wnoise = Wnoise;
    b.bias = bias;
    b.W13_e = W13_e;
    b.W2_e = W2_e;
    b.counts = (int32_t *)(a + o_counts);
    b.importance = (float *)(a + o_imp);
    b.f = (float *)(a + o_f);
    b.P = (float *)(a + o_P);
    b.topk_idx = (int32_t *)(a + o_idx);
    b.topk_w = (float *)(a + o_w);
    b.probs_sum = (float *)(a + o_ps);
    b.x_perm = a + o_xp;
    b.row_token = (int32_t *)(a + o_rt);
    b.slot_row = (int32_t *)(a + o_sr);
    b.kept = (int32_t *)(a + o_kept);
    b.offsets = (int32_t *)(a + o_off);
    b.h = a + o_h;
    b.out = a + o_out;
    b.router_packed = nullptr;
    pl->ws = a + o_ws;
    rc = moe_workspace_init(pl->ws, pl->ws_bytes, pl->compute);
    if (rc == MOE_OK && pack) {
        e = launch_router_pack(p, Wg, Wnoise, a + o_wt, pl->compute);
        if (e != cudaSuccess) {
            release(pl);
            return report_cuda(e, fn);
        }
        b.router_packed = a + o_wt;
    }
    if (rc != MOE_OK) {
        release(pl);
        return rc;
    }
    PL_TRY(cudaStreamSynchronize(pl->compute));
#undef PL_TRY
    if (e != cudaSuccess) {
        release(pl);
        return report_cuda(e, fn);
    }
    *out = pl;
    return report_ok();
}

int moe_pipeline_submit(moe_pipeline_t *pl, const void *x_host, const float *noise_host,
                        void *y_host, float *loss_host, int64_t *ticket)
{
    const char *fn = "moe_pipeline_submit";
    if (pl == nullptr || x_host == nullptr || y_host == nullptr || loss_host == nullptr ||
        ticket == nullptr)
        return report_error(MOE_ERR_INVALID_ARG,
                            "moe_pipeline_submit: pipeline, x_host, y_host, loss_host and "
                            "ticket are required");
    if ((noise_host != nullptr) != (pl->Wnoise != nullptr))
        return report_error(MOE_ERR_INVALID_ARG,
                            "moe_pipeline_submit: noise_host must be given iff the pipeline "
                            "has Wnoise");
    if (pl->broken)
        return report_error(MOE_ERR_CUDA, "moe_pipeline_submit: an earlier CUDA call of this "
                                          "pipeline failed");
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess && dev != pl->device)
        e = cudaSetDevice(pl->device);
    if (e != cudaSuccess)
        return pl_cuda(pl, e, fn);

    const int64_t i = pl->next_ticket;
    const int s = (int)(i % pl->depth);
    const bool reuse = pl->slot_ticket[s] >= 0;
    // in: wait until the previous user of slot s has consumed its inputs
    if (reuse)
        e = cudaStreamWaitEvent(pl->h2d, pl->consumed[s], 0);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(pl->x[s], x_host, pl->x_bytes, cudaMemcpyHostToDevice, pl->h2d);
    if (e == cudaSuccess && pl->noise_bytes)
        e = cudaMemcpyAsync(pl->noise[s], noise_host, pl->noise_bytes, cudaMemcpyHostToDevice,
                            pl->h2d);
    if (e == cudaSuccess)
        e = cudaEventRecord(pl->in_ready[s], pl->h2d);
    // layer: inputs landed and the previous user's y of slot s copied out
    if (e == cudaSuccess)
        e = cudaStreamWaitEvent(pl->compute, pl->in_ready[s], 0);
    if (e == cudaSuccess && reuse)
        e = cudaStreamWaitEvent(pl->compute, pl->out_done[s], 0);
    if (e != cudaSuccess)
        return pl_cuda(pl, e, fn);
    moe_buffers_t b = pl->shared;
    b.x = pl->x[s];
    b.noise = pl->noise[s];
    b.y = pl->y[s];
    b.loss = pl->loss[s];
    int rc = moe_forward(&pl->p, &b, pl->ws, pl->ws_bytes, pl->compute);
    if (rc != MOE_OK) {
        pl->broken = true;
        return rc;
    }
    // this batch's status word into the slot, then cleared for the next batch; both on
    // the compute stream, so no later batch's kernels can touch it first
    e = cudaMemcpyAsync(pl->dev_status[s], pl->ws, sizeof(int32_t), cudaMemcpyDeviceToDevice,
                        pl->compute);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(pl->ws, 0, sizeof(int32_t), pl->compute);
    if (e == cudaSuccess)
        e = cudaEventRecord(pl->consumed[s], pl->compute);
    // out: y, L_balance and the status word of this batch
    if (e == cudaSuccess)
        e = cudaStreamWaitEvent(pl->d2h, pl->consumed[s], 0);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(y_host, pl->y[s], pl->x_bytes, cudaMemcpyDeviceToHost, pl->d2h);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(loss_host, pl->loss[s], sizeof(float), cudaMemcpyDeviceToHost,
                            pl->d2h);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(&pl->host_status[i % MOE_PIPELINE_STATUS_RING], pl->dev_status[s],
                            sizeof(int32_t), cudaMemcpyDeviceToHost, pl->d2h);
    if (e == cudaSuccess)
        e = cudaEventRecord(pl->out_done[s], pl->d2h);
    if (e != cudaSuccess)
        return pl_cuda(pl, e, fn);
    pl->slot_ticket[s] = i;
    pl->next_ticket = i + 1;
    *ticket = i;
    return report_ok();
}

int moe_pipeline_wait(moe_pipeline_t *pl, int64_t ticket)
{
    const char *fn = "moe_pipeline_wait";
    if (pl == nullptr)
        return report_error(MOE_ERR_INVALID_ARG, "moe_pipeline_wait: pipeline is NULL");
    if (ticket < 0 || ticket >= pl->next_ticket)
        return report_error(MOE_ERR_INVALID_ARG, "moe_pipeline_wait: ticket was never issued");
    if (pl->next_ticket - ticket > MOE_PIPELINE_STATUS_RING)
        return report_error(MOE_ERR_INVALID_ARG,
                            "moe_pipeline_wait: ticket older than the last "
                            "MOE_PIPELINE_STATUS_RING batches (its status is no longer held)");
    const int s = (int)(ticket % pl->depth);
    // the slot's event marks its latest batch; d2h is in order, so that batch
    // finishing implies this one has
    cudaError_t e = cudaEventSynchronize(pl->out_done[s]);
    if (e != cudaSuccess)
        return pl_cuda(pl, e, fn);
    const int32_t st = pl->host_status[ticket % MOE_PIPELINE_STATUS_RING];
    if (st != 0)
        return report_error(st, "moe_pipeline_wait: a kernel recorded an error for this batch "
                                "(status word of the pipeline's workspace)");
    return report_ok();
}

int moe_pipeline_destroy(moe_pipeline_t *pl)
{
    if (pl == nullptr)
        return report_ok();
    // drain all three streams (device status words were reported by wait)
    cudaError_t e = cudaStreamSynchronize(pl->d2h);
    const cudaError_t e2 = cudaStreamSynchronize(pl->compute);
    const cudaError_t e3 = cudaStreamSynchronize(pl->h2d);
    if (e == cudaSuccess)
        e = e2 != cudaSuccess ? e2 : e3;
    release(pl);
    if (e != cudaSuccess)
        return report_cuda(e, "moe_pipeline_destroy");
    return report_ok();
}

}  // extern "C"
