// ep.cu -- the pieces of the expert-parallel layer that are not collectives
// ("Llama 3 Meets MoE", section "训练框架": 5-D hybrid parallelism, whose Expert
// Parallelism places the experts of a MoE layer on different devices; the
// training configuration runs 8-way expert parallelism).
//
// N ranks each hold T_r tokens and the experts [r E/N, (r+1) E/N).  A rank
// routes and dispatches its own tokens without a capacity (a1, a2), the ranks
// exchange their per-expert counts, and every rank then derives the same plan
// from those counts (moe_ep_plan, host): how many rows of each (rank, expert)
// pair the capacity keeps and where each contiguous run of rows goes.  Capacity
// scope GLOBAL ranks the assignments of one expert over the concatenation of the
// ranks' batches in rank order, which makes the layer equal to the one-device
// layer run on that concatenated batch; scope LOCAL applies the capacity to each
// rank's own batch.  The rows themselves move as contiguous runs: the run of
// expert e on rank p is the first keep[p][e] rows of e's block of p's dispatch
// output (token-ascending, so the kept rows are a prefix), and it lands at its
// place in the owner's expert-major receive buffer, after the runs of the lower
// ranks: no pack or regroup kernel is needed on either side.
#include <cstdio>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

struct KeepVec {
    int32_t v[MOE_MAX_EXPERTS];
};

// slot_row[t][j] = -1 where the capacity drops assignment (t, j): its position
// inside its expert's block, slot_row - offsets[e], is at or past keep[e].
__global__ void ep_mask_slots_kernel(const int32_t *__restrict__ idx,
                                     const int32_t *__restrict__ offsets, KeepVec keep, int64_t n,
                                     int E, int32_t *__restrict__ slot_row)
{
    pdl_wait();
    pdl_trigger();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t r = slot_row[i];
        const int32_t e = idx[i];
        if (r < 0 || e < 0 || e >= E)
            continue;
        if (r - offsets[e] >= keep.v[e])
            slot_row[i] = -1;
    }
}

// counts[e] = sum over ranks of counts_all[p][e] (saturating at INT32_MAX).
__global__ void ep_sum_counts_kernel(const int32_t *__restrict__ counts_all, int N, int E,
                                     int32_t *__restrict__ counts)
{
    pdl_wait();
    pdl_trigger();
    const int e = threadIdx.x;
    if (e >= E)
        return;
    int64_t s = 0;
    for (int p = 0; p < N; ++p)
        s += counts_all[(int64_t)p * E + e];
    counts[e] = s > INT32_MAX ? INT32_MAX : (int32_t)s;
}

int ep_fail(int code, const char *fn, const char *what)
{
    char msg[256];
    snprintf(msg, sizeof msg, "%s: %s", fn, what);
    return report_error(code, msg);
}

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" int moe_ep_plan(const int32_t *counts_all, int32_t N, int32_t E, int32_t rank,
                           int32_t capacity, int32_t scope, int32_t *keep_all,
                           int32_t *send_row, int32_t *send_cnt, int32_t *recv_row,
                           int32_t *recv_cnt, int32_t *in_offsets)
{
    const char *fn = "moe_ep_plan";
    if (!counts_all || !keep_all || !send_row || !send_cnt || !recv_row || !recv_cnt ||
        !in_offsets)
        return ep_fail(MOE_ERR_INVALID_ARG, fn, "a pointer argument is NULL");
    if (E < 1 || E > MOE_MAX_EXPERTS || N < 1 || N > E || E % N != 0)
        return ep_fail(MOE_ERR_SHAPE, fn, "need 1 <= E <= 64 and N dividing E");
    if (rank < 0 || rank >= N)
        return ep_fail(MOE_ERR_INVALID_ARG, fn, "rank outside [0, N)");
    if (scope != MOE_EP_CAPACITY_GLOBAL && scope != MOE_EP_CAPACITY_LOCAL)
        return ep_fail(MOE_ERR_INVALID_ARG, fn, "scope is neither GLOBAL nor LOCAL");
    const int64_t lim = INT32_MAX / 2;
    for (int p = 0; p < N; ++p) {
        int64_t rows = 0;
        for (int e = 0; e < E; ++e) {
            const int32_t c = counts_all[(int64_t)p * E + e];
            if (c < 0)
                return ep_fail(MOE_ERR_INVALID_ARG, fn, "a count is negative");
            rows += c;
        }
        if (rows > lim)
            return ep_fail(MOE_ERR_SHAPE, fn, "a rank has too many rows");
    }
    // keep[p][e]: the capacity keeps the assignments of rank ("Llama 3 Meets MoE",
    // section 3 "容量因子": an expert takes at most C tokens, the rest overflow)
    // whose rank inside expert e is below C; under GLOBAL the ranks before p come
    // first, so p keeps C minus what they hold, clamped to [0, counts[p][e]].
    for (int e = 0; e < E; ++e) {
        int64_t before = 0;
        for (int p = 0; p < N; ++p) {
            const int64_t c = counts_all[(int64_t)p * E + e];
            int64_t kp = c;
            if (capacity >= 0) {
                const int64_t room = scope == MOE_EP_CAPACITY_GLOBAL ? capacity - before : capacity;
                kp = room < 0 ? 0 : (room < c ? room : c);
            }
            keep_all[(int64_t)p * E + e] = (int32_t)kp;
            before += c;
        }
    }
    const int El = E / N;
    // sends: expert e's run starts at e's block of this rank's dispatch output
    // (the blocks are the dropless counts, in expert order)
    int64_t off = 0;
    for (int e = 0; e < E; ++e) {
        send_row[e] = (int32_t)off;
        send_cnt[e] = keep_all[(int64_t)rank * E + e];
        off += counts_all[(int64_t)rank * E + e];
    }
    // receive buffer: expert-major over the local experts, ranks ascending inside
    int64_t pos = 0;
    for (int l = 0; l < El; ++l) {
        const int e = rank * El + l;
        in_offsets[l] = (int32_t)pos;
        for (int p = 0; p < N; ++p) {
            const int32_t kp = keep_all[(int64_t)p * E + e];
            recv_row[p * El + l] = (int32_t)pos;
            recv_cnt[p * El + l] = kp;
            pos += kp;
        }
        if (pos > lim)
            return ep_fail(MOE_ERR_SHAPE, fn, "the receive buffer has too many rows");
    }
    in_offsets[El] = (int32_t)pos;
    return report_ok();
}

extern "C" int moe_ep_mask_slots(const moe_params_t *p, const int32_t *topk_idx,
                                 const int32_t *offsets, const int32_t *keep, int32_t *slot_row,
                                 void *stream)
{
    const char *fn = "moe_ep_mask_slots";
    int rc = validate_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    if (!topk_idx || !offsets || !keep || !slot_row)
        return ep_fail(MOE_ERR_INVALID_ARG, fn, "a pointer argument is NULL");
    KeepVec kv{};
    for (int e = 0; e < p->E; ++e) {
        if (keep[e] < 0)
            return ep_fail(MOE_ERR_INVALID_ARG, fn, "a keep entry is negative");
        kv.v[e] = keep[e];
    }
    const int64_t n = (int64_t)p->T * p->k;
    if (n == 0)
        return report_ok();
    int64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 16)
        blocks = 148 * 16;
    cudaError_t e = launch_pdl(ep_mask_slots_kernel, dim3((unsigned)blocks), dim3(256), 0,
                               (cudaStream_t)stream, topk_idx, offsets, kv, n, p->E, slot_row);
    count_launch();
    if (e == cudaSuccess)
        e = cudaGetLastError();
    if (e != cudaSuccess)
        return report_cuda(e, fn);
    return report_ok();
}

extern "C" int moe_ep_gate_stats(const moe_params_t *p, const int32_t *counts_all, int32_t N,
                                 const float *probs_sum, int32_t *counts, float *f, float *P,
                                 float *loss, void *stream)
{
    const char *fn = "moe_ep_gate_stats";
    int rc = validate_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    if (!counts_all || !probs_sum || !counts || !f || !P || !loss)
        return ep_fail(MOE_ERR_INVALID_ARG, fn, "a pointer argument is NULL");
    if (N < 1 || N > p->E || p->E % N != 0)
        return ep_fail(MOE_ERR_SHAPE, fn, "N must divide E");
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = launch_pdl(ep_sum_counts_kernel, dim3(1), dim3(MOE_MAX_EXPERTS), 0, s,
                               counts_all, (int)N, p->E, counts);
    count_launch();
    if (e == cudaSuccess)
        e = launch_gate_stats(p, counts, probs_sum, f, P, loss, s);
    if (e == cudaSuccess)
        e = cudaGetLastError();
    if (e != cudaSuccess)
        return report_cuda(e, fn);
    return report_ok();
}
