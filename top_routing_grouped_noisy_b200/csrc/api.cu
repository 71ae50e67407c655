// api.cu -- the extern "C" entry points of libmoe.so: argument validation,
// workspace layout and the launch sequence of each step.  No kernel here does
// arithmetic of the layer; that lives in the kernel translation units.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "common.cuh"
#include "kernels.h"

namespace moe {

static thread_local char g_err[512] = "";
static std::atomic<uint64_t> g_launches{0};
static std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};
// 8 pair m-tiles: with the 74 clusters of a B200 at work, about an 8 x 9 block of
// output tiles at a time, each A band and B tile read about once per block
static std::atomic<int32_t> g_band_rows{2048};

void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
uint64_t wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }
int gemm_band_rows() { return g_band_rows.load(std::memory_order_relaxed); }

static int fail(int code, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

static int ok()
{
    g_err[0] = 0;
    return MOE_OK;
}

static int cuda_fail(cudaError_t e, const char *where)
{
    return fail(MOE_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorString(e), cudaGetErrorName(e));
}

static bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define REQUIRE_PTR(ptr)                                                               \
    do {                                                                               \
        if ((ptr) == nullptr)                                                          \
            return fail(MOE_ERR_INVALID_ARG, "%s: argument '%s' is NULL", fn, #ptr);   \
        if (!al16(ptr))                                                                \
            return fail(MOE_ERR_ALIGN, "%s: argument '%s' is not 16-byte aligned", fn, \
                        #ptr);                                                         \
    } while (0)

// Token-sized buffers may be NULL when the batch is empty (T == 0).
#define REQUIRE_TOK(ptr)                                                               \
    do {                                                                               \
        if (p->T > 0 || (ptr) != nullptr)                                              \
            REQUIRE_PTR(ptr);                                                          \
    } while (0)

#define OPTIONAL_PTR(ptr)                                                              \
    do {                                                                               \
        if ((ptr) != nullptr && !al16(ptr))                                            \
            return fail(MOE_ERR_ALIGN, "%s: argument '%s' is not 16-byte aligned", fn, \
                        #ptr);                                                         \
    } while (0)

static int check_params(const char *fn, const moe_params_t *p)
{
    if (p == nullptr)
        return fail(MOE_ERR_INVALID_ARG, "%s: params is NULL", fn);
    if (p->T < 0)
        return fail(MOE_ERR_INVALID_ARG, "%s: T=%d < 0", fn, p->T);
    if (p->E < 1 || p->E > MOE_MAX_EXPERTS)
        return fail(MOE_ERR_INVALID_ARG, "%s: E=%d outside [1,%d]", fn, p->E, MOE_MAX_EXPERTS);
    if (p->k < 1 || p->k > p->E || p->k > MOE_MAX_TOPK)
        return fail(MOE_ERR_INVALID_ARG, "%s: k=%d outside [1,min(E,%d)]", fn, p->k,
                    MOE_MAX_TOPK);
    if (p->d < 8 || p->d % 8 != 0)
        return fail(MOE_ERR_SHAPE, "%s: d=%d is not a positive multiple of 8", fn, p->d);
    if (p->m < 1)
        return fail(MOE_ERR_SHAPE, "%s: m=%d < 1", fn, p->m);
    if (p->dtype != MOE_BF16 && p->dtype != MOE_F32)
        return fail(MOE_ERR_DTYPE, "%s: dtype=%d is neither MOE_BF16 nor MOE_F32", fn, p->dtype);
    if (p->router_type != MOE_ROUTER_MIXTRAL && p->router_type != MOE_ROUTER_ST)
        return fail(MOE_ERR_INVALID_ARG, "%s: router_type=%d", fn, p->router_type);
    const int64_t rows = (int64_t)p->T * p->k;
    if (rows > (int64_t)INT32_MAX / 2)
        return fail(MOE_ERR_SHAPE, "%s: T*k=%lld rows is too large", fn, (long long)rows);
    if (p->m > 1 << 20 || p->d > 1 << 20)
        return fail(MOE_ERR_SHAPE, "%s: d=%d or m=%d is too large", fn, p->d, p->m);
    return MOE_OK;
}

WsLayout ws_layout(const moe_params_t *p)
{
    WsLayout L{};
    const size_t es = p->dtype == MOE_BF16 ? 2 : 4;
    size_t off = kWsHeader;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += (bytes + 255) / 256 * 256;
        return o;
    };
    L.wt = take((size_t)kWtRows * p->d * es);
    const size_t blocks = (size_t)ceil_div(p->T > 0 ? p->T : 1, kRouterMinTokens);
    L.rpart = take(blocks * 2 * p->E * sizeof(float));
    const size_t chunks = (size_t)ceil_div(p->T > 0 ? p->T : 1, kDispatchChunk);
    L.hist = take(chunks * p->E * sizeof(int32_t));
    L.dcounts = take(MOE_MAX_EXPERTS * sizeof(int32_t));
    // Sections for small batches are sized for min(T, 64) tokens even when T is
    // larger, so that a workspace sized for T also serves every smaller batch.
    const int t_small = p->T < kRouterSmallTokens ? (p->T > 0 ? p->T : 1) : kRouterSmallTokens;
    L.rsmall = take((size_t)kRouterSmallSplit * t_small * 2 * p->E * sizeof(float));
    L.gsmall = take((size_t)2 * t_small * p->E * sizeof(float));
    L.total = off;
    return L;
}

static int check_ws(const char *fn, const moe_params_t *p, void *ws, size_t ws_bytes)
{
    if (ws == nullptr)
        return fail(MOE_ERR_INVALID_ARG, "%s: workspace is NULL", fn);
    if (!al16(ws))
        return fail(MOE_ERR_ALIGN, "%s: workspace is not 16-byte aligned", fn);
    const size_t need = ws_layout(p).total;
    if (ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "%s: workspace has %zu bytes, needs %zu", fn, ws_bytes,
                    need);
    return MOE_OK;
}

static int after_launch(const char *fn, cudaError_t e)
{
    if (e == cudaSuccess)
        e = cudaGetLastError();
    if (e != cudaSuccess)
        return cuda_fail(e, fn);
    return ok();
}

// Accessors for entry points defined in other translation units.
int validate_params(const char *fn, const moe_params_t *p) { return check_params(fn, p); }
int report_error(int code, const char *msg) { return fail(code, "%s", msg); }
int report_cuda(cudaError_t e, const char *where) { return cuda_fail(e, where); }
int report_ok() { return ok(); }

}  // namespace moe

using namespace moe;

extern "C" {

const char *moe_version(void) { return "libmoe 0.1 (sm_100a)"; }

const char *moe_last_error_string(void) { return g_err; }

uint64_t moe_launch_count(void) { return g_launches.load(); }

void moe_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns); }

void moe_set_gemm_band_rows(int32_t rows) { g_band_rows.store(rows < 0 ? 0 : rows); }

int32_t moe_capacity(int32_t T, int32_t E, double cf)
{
    if (cf < 0 || E <= 0 || T < 0)
        return -1;
    // ceil(T * cf / E) without the rounding trap of T*cf/E landing just above an integer
    const double v = (double)T * cf / (double)E;
    double c = (double)(int64_t)v;
    if (c < v)
        c += 1.0;
    if (c > (double)INT32_MAX)
        return INT32_MAX;
    return (int32_t)c;
}

int64_t moe_packed_w13_elems(int32_t E, int32_t m, int32_t d)
{
    if (E <= 0 || m <= 0 || d <= 0)
        return 0;
    return (int64_t)E * 2 * round_up(m, 16) * d;
}

int64_t moe_packed_w2_elems(int32_t E, int32_t m, int32_t d)
{
    if (E <= 0 || m <= 0 || d <= 0)
        return 0;
    return (int64_t)E * d * round_up(m, 8);
}

int32_t moe_h_ld(int32_t m) { return m > 0 ? round_up(m, 8) : 0; }

size_t moe_workspace_size(const moe_params_t *p)
{
    if (check_params("moe_workspace_size", p) != MOE_OK)
        return 0;
    return ws_layout(p).total;
}

int moe_workspace_init(void *ws, size_t ws_bytes, void *stream)
{
    const char *fn = "moe_workspace_init";
    REQUIRE_PTR(ws);
    if (ws_bytes < kWsHeader)
        return fail(MOE_ERR_WORKSPACE, "%s: %zu bytes is below the %zu-byte header", fn,
                    ws_bytes, kWsHeader);
    cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, fn);
}

int moe_get_device_status(void *ws, int32_t *status, int32_t clear, void *stream)
{
    const char *fn = "moe_get_device_status";
    REQUIRE_PTR(ws);
    if (status == nullptr)
        return fail(MOE_ERR_INVALID_ARG, "%s: status is NULL", fn);
    cudaStream_t s = (cudaStream_t)stream;
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(s);
    if (e == cudaSuccess && clear)  // status word and the launch counters
        e = cudaMemsetAsync(ws, 0, kWsResetBytes, s);
    if (e != cudaSuccess)
        return cuda_fail(e, fn);
    *status = v;
    return ok();
}

int moe_partition_experts(const void *W1, const void *W3, const void *W2, int32_t d,
                          int32_t d_ff, int32_t E, int32_t mode, const int32_t *perm,
                          int32_t dtype, void *W13_e, void *W2_e, void *ws, void *stream)
{
    const char *fn = "moe_partition_experts";
    REQUIRE_PTR(W1);
    REQUIRE_PTR(W3);
    REQUIRE_PTR(W2);
    REQUIRE_PTR(W13_e);
    REQUIRE_PTR(W2_e);
    OPTIONAL_PTR(ws);
    if (dtype != MOE_BF16 && dtype != MOE_F32)
        return fail(MOE_ERR_DTYPE, "%s: dtype=%d", fn, dtype);
    if (E < 1 || E > MOE_MAX_EXPERTS)
        return fail(MOE_ERR_INVALID_ARG, "%s: E=%d outside [1,%d]", fn, E, MOE_MAX_EXPERTS);
    if (d < 8 || d % 8 != 0)
        return fail(MOE_ERR_SHAPE, "%s: d=%d is not a positive multiple of 8", fn, d);
    if (d_ff < 1 || d_ff > (1 << 22))
        return fail(MOE_ERR_SHAPE, "%s: d_ff=%d", fn, d_ff);
    int m;
    if (mode == MOE_PARTITION_DISJOINT) {
        if (d_ff % E != 0)
            return fail(MOE_ERR_SHAPE, "%s: d_ff=%d is not divisible by E=%d", fn, d_ff, E);
        if (perm == nullptr)
            return fail(MOE_ERR_INVALID_ARG, "%s: DISJOINT mode needs perm", fn);
        m = d_ff / E;
    } else if (mode == MOE_PARTITION_COPY || mode == MOE_PARTITION_STACKED) {
        m = d_ff;
    } else {
        return fail(MOE_ERR_INVALID_ARG, "%s: mode=%d", fn, mode);
    }
    int32_t *status = reinterpret_cast<int32_t *>(ws);
    cudaError_t e = launch_partition(W1, W3, W2, d, d_ff, E, m, mode, perm, dtype, W13_e, W2_e,
                                     status, (cudaStream_t)stream);
    return after_launch(fn, e);
}

static int route_impl(const char *fn, const moe_params_t *p, const void *x, const void *Wg,
                      const void *Wnoise, const void *Wt, const float *noise, const float *bias,
                      int32_t *topk_idx, float *topk_w, float *probs_sum, float *importance,
                      void *ws, size_t ws_bytes, void *stream)
{
    int rc = check_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    REQUIRE_TOK(x);
    REQUIRE_PTR(Wg);
    OPTIONAL_PTR(Wnoise);
    OPTIONAL_PTR(noise);
    OPTIONAL_PTR(bias);
    REQUIRE_TOK(topk_idx);
    REQUIRE_TOK(topk_w);
    REQUIRE_PTR(probs_sum);
    REQUIRE_PTR(importance);
    if (Wnoise != nullptr && noise == nullptr && p->T > 0)
        return fail(MOE_ERR_INVALID_ARG, "%s: Wnoise given without the noise draws", fn);
    if ((rc = check_ws(fn, p, ws, ws_bytes)) != MOE_OK)
        return rc;
    char *w = static_cast<char *>(ws);
    cudaError_t e = launch_route(p, x, Wg, Wnoise, Wt, noise, bias, topk_idx, topk_w,
                                 probs_sum, importance, w, reinterpret_cast<int32_t *>(w),
                                 (cudaStream_t)stream);
    return after_launch(fn, e);
}

int moe_route(const moe_params_t *p, const void *x, const void *Wg, const void *Wnoise,
              const float *noise, const float *bias, int32_t *topk_idx, float *topk_w,
              float *probs_sum, float *importance, void *ws, size_t ws_bytes, void *stream)
{
    return route_impl("moe_route", p, x, Wg, Wnoise, nullptr, noise, bias, topk_idx, topk_w,
                      probs_sum, importance, ws, ws_bytes, stream);
}

size_t moe_router_packed_bytes(const moe_params_t *p, int32_t noisy)
{
    if (check_params("moe_router_packed_bytes", p) != MOE_OK)
        return 0;
    const size_t es = p->dtype == MOE_BF16 ? 2 : 4;
    return (size_t)router_packed_rows(p->E, noisy != 0) * p->d * es;
}

int moe_router_pack(const moe_params_t *p, const void *Wg, const void *Wnoise, void *Wt,
                    void *stream)
{
    const char *fn = "moe_router_pack";
    int rc = check_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    REQUIRE_PTR(Wg);
    OPTIONAL_PTR(Wnoise);
    REQUIRE_PTR(Wt);
    if (p->dtype != MOE_BF16)
        return fail(MOE_ERR_DTYPE, "%s: only bf16 router weights are packed", fn);
    return after_launch(fn, launch_router_pack(p, Wg, Wnoise, Wt, (cudaStream_t)stream));
}

int moe_route_packed(const moe_params_t *p, const void *x, const void *Wg, const void *Wnoise,
                     const void *Wt, const float *noise, const float *bias, int32_t *topk_idx,
                     float *topk_w, float *probs_sum, float *importance, void *ws,
                     size_t ws_bytes, void *stream)
{
    const char *fn = "moe_route_packed";
    REQUIRE_PTR(Wt);
    return route_impl(fn, p, x, Wg, Wnoise, Wt, noise, bias, topk_idx, topk_w, probs_sum,
                      importance, ws, ws_bytes, stream);
}

int moe_dispatch(const moe_params_t *p, const void *x, const int32_t *topk_idx, void *x_perm,
                 int32_t *row_token, int32_t *slot_row, int32_t *counts, int32_t *kept,
                 int32_t *offsets, void *ws, size_t ws_bytes, void *stream)
{
    const char *fn = "moe_dispatch";
    int rc = check_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    REQUIRE_TOK(x);
    REQUIRE_TOK(topk_idx);
    REQUIRE_TOK(x_perm);
    REQUIRE_TOK(row_token);
    REQUIRE_TOK(slot_row);
    REQUIRE_PTR(counts);
    REQUIRE_PTR(kept);
    REQUIRE_PTR(offsets);
    if ((rc = check_ws(fn, p, ws, ws_bytes)) != MOE_OK)
        return rc;
    char *w = static_cast<char *>(ws);
    cudaError_t e = launch_dispatch(p, x, topk_idx, x_perm, row_token, slot_row, counts, kept,
                                    offsets, w, reinterpret_cast<int32_t *>(w), false,
                                    (cudaStream_t)stream);
    return after_launch(fn, e);
}

int moe_dispatch_routed(const moe_params_t *p, const void *x, const int32_t *topk_idx,
                        void *x_perm, int32_t *row_token, int32_t *slot_row, int32_t *counts,
                        int32_t *kept, int32_t *offsets, void *ws, size_t ws_bytes, void *stream)
{
    const char *fn = "moe_dispatch_routed";
    int rc = check_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    REQUIRE_TOK(x);
    REQUIRE_TOK(topk_idx);
    REQUIRE_TOK(x_perm);
    REQUIRE_TOK(row_token);
    REQUIRE_TOK(slot_row);
    REQUIRE_PTR(counts);
    REQUIRE_PTR(kept);
    REQUIRE_PTR(offsets);
    if ((rc = check_ws(fn, p, ws, ws_bytes)) != MOE_OK)
        return rc;
    char *w = static_cast<char *>(ws);
    cudaError_t e = launch_dispatch(p, x, topk_idx, x_perm, row_token, slot_row, counts, kept,
                                    offsets, w, reinterpret_cast<int32_t *>(w), true,
                                    (cudaStream_t)stream);
    return after_launch(fn, e);
}

int moe_dispatch_rows(const moe_params_t *p, const int32_t *topk_idx, int32_t *row_token,
                      int32_t *slot_row, int32_t *counts, int32_t *kept, int32_t *offsets,
                      void *ws, size_t ws_bytes, void *stream)
{
    const char *fn = "moe_dispatch_rows";
    int rc = check_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    REQUIRE_TOK(topk_idx);
    REQUIRE_TOK(row_token);
    REQUIRE_TOK(slot_row);
    REQUIRE_PTR(counts);
    REQUIRE_PTR(kept);
    REQUIRE_PTR(offsets);
    if ((rc = check_ws(fn, p, ws, ws_bytes)) != MOE_OK)
        return rc;
    char *w = static_cast<char *>(ws);
    cudaError_t e = launch_dispatch(p, nullptr, topk_idx, nullptr, row_token, slot_row, counts,
                                    kept, offsets, w, reinterpret_cast<int32_t *>(w), false,
                                    (cudaStream_t)stream);
    return after_launch(fn, e);
}

int moe_expert_up_gather(const moe_params_t *p, const void *x, const int32_t *row_token,
                         const int32_t *offsets, const void *W13_e, void *h, void *ws,
                         size_t ws_bytes, void *stream)
{
    const char *fn = "moe_expert_up_gather";
    int rc = check_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    if (p->dtype != MOE_BF16)
        return fail(MOE_ERR_DTYPE, "%s: the gathering expert GEMM is bf16 only", fn);
    REQUIRE_TOK(x);
    REQUIRE_TOK(row_token);
    REQUIRE_PTR(offsets);
    REQUIRE_PTR(W13_e);
    REQUIRE_TOK(h);
    if ((rc = check_ws(fn, p, ws, ws_bytes)) != MOE_OK)
        return rc;
    if (p->T == 0)
        return ok();
    cudaError_t e = launch_up_tc_gather(p, x, row_token, offsets, W13_e, h,
                                        reinterpret_cast<int32_t *>(ws), (cudaStream_t)stream);
    return after_launch(fn, e);
}

int moe_expert_up(const moe_params_t *p, const void *x_perm, const int32_t *offsets,
                  const void *W13_e, void *h, void *ws, size_t ws_bytes, void *stream)
{
    const char *fn = "moe_expert_up";
    int rc = check_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    REQUIRE_TOK(x_perm);
    REQUIRE_PTR(offsets);
    REQUIRE_PTR(W13_e);
    REQUIRE_TOK(h);
    if ((rc = check_ws(fn, p, ws, ws_bytes)) != MOE_OK)
        return rc;
    if (p->T == 0)
        return ok();
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (p->dtype == MOE_F32)
        e = launch_up_simt(p, (const float *)x_perm, offsets, (const float *)W13_e, (float *)h, s);
    else if (decode_fits(p))
        e = launch_up_decode(p, x_perm, offsets, W13_e, h, static_cast<char *>(ws), s);
    else
        e = launch_up_tc(p, x_perm, offsets, W13_e, h, reinterpret_cast<int32_t *>(ws), s);
    return after_launch(fn, e);
}

int moe_expert_down(const moe_params_t *p, const void *h, const int32_t *offsets,
                    const void *W2_e, void *out, void *ws, size_t ws_bytes, void *stream)
{
    const char *fn = "moe_expert_down";
    int rc = check_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    REQUIRE_TOK(h);
    REQUIRE_PTR(offsets);
    REQUIRE_PTR(W2_e);
    REQUIRE_TOK(out);
    if ((rc = check_ws(fn, p, ws, ws_bytes)) != MOE_OK)
        return rc;
    if (p->T == 0)
        return ok();
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (p->dtype == MOE_F32)
        e = launch_down_simt(p, (const float *)h, offsets, (const float *)W2_e, (float *)out, s);
    else if (decode_fits(p))
        e = launch_down_decode(p, h, offsets, W2_e, out, static_cast<char *>(ws), s);
    else
        e = launch_down_tc(p, h, offsets, W2_e, out, reinterpret_cast<int32_t *>(ws), s);
    return after_launch(fn, e);
}

int moe_expert_ffn(const moe_params_t *p, const void *x_perm, const int32_t *offsets,
                   const void *W13_e, const void *W2_e, void *h, void *out, void *ws,
                   size_t ws_bytes, void *stream)
{
    int rc = moe_expert_up(p, x_perm, offsets, W13_e, h, ws, ws_bytes, stream);
    if (rc != MOE_OK)
        return rc;
    return moe_expert_down(p, h, offsets, W2_e, out, ws, ws_bytes, stream);
}

int moe_combine(const moe_params_t *p, const void *out, const int32_t *slot_row,
                const float *topk_w, void *y, void *stream)
{
    const char *fn = "moe_combine";
    int rc = check_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    REQUIRE_TOK(out);
    REQUIRE_TOK(slot_row);
    REQUIRE_TOK(topk_w);
    REQUIRE_TOK(y);
    if (p->T == 0)
        return ok();
    cudaError_t e = launch_combine(p, out, slot_row, topk_w, y, (cudaStream_t)stream);
    return after_launch(fn, e);
}

int moe_gate_stats(const moe_params_t *p, const int32_t *counts, const float *probs_sum,
                   float *f, float *P, float *loss, void *stream)
{
    const char *fn = "moe_gate_stats";
    int rc = check_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    REQUIRE_PTR(counts);
    REQUIRE_PTR(probs_sum);
    REQUIRE_PTR(f);
    REQUIRE_PTR(P);
    REQUIRE_PTR(loss);
    cudaError_t e = launch_gate_stats(p, counts, probs_sum, f, P, loss, (cudaStream_t)stream);
    return after_launch(fn, e);
}

int moe_forward(const moe_params_t *p, const moe_buffers_t *b, void *ws, size_t ws_bytes,
                void *stream)
{
    const char *fn = "moe_forward";
    int rc = check_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    if (b == nullptr)
        return fail(MOE_ERR_INVALID_ARG, "%s: buffers is NULL", fn);
    REQUIRE_TOK(b->y);
    REQUIRE_PTR(b->loss);
    REQUIRE_PTR(b->f);
    REQUIRE_PTR(b->P);
    if (decode_forward_fits(p, b->Wnoise != nullptr)) {
        // decode-shaped batch: the whole layer in one cooperative launch
        REQUIRE_PTR(b->x);
        REQUIRE_PTR(b->Wg);
        OPTIONAL_PTR(b->Wnoise);
        OPTIONAL_PTR(b->noise);
        OPTIONAL_PTR(b->bias);
        REQUIRE_PTR(b->W13_e);
        REQUIRE_PTR(b->W2_e);
        REQUIRE_PTR(b->counts);
        REQUIRE_PTR(b->importance);
        REQUIRE_PTR(b->topk_idx);
        REQUIRE_PTR(b->topk_w);
        REQUIRE_PTR(b->probs_sum);
        REQUIRE_PTR(b->x_perm);
        REQUIRE_PTR(b->row_token);
        REQUIRE_PTR(b->slot_row);
        REQUIRE_PTR(b->kept);
        REQUIRE_PTR(b->offsets);
        REQUIRE_PTR(b->h);
        REQUIRE_PTR(b->out);
        if (b->Wnoise != nullptr && b->noise == nullptr)
            return fail(MOE_ERR_INVALID_ARG, "%s: Wnoise given without the noise draws", fn);
        if ((rc = check_ws(fn, p, ws, ws_bytes)) != MOE_OK)
            return rc;
        char *w = static_cast<char *>(ws);
        cudaStream_t s = (cudaStream_t)stream;
        return after_launch(fn, launch_forward_decode(p, b, w, s));
    }
    if (front_small_fits(p, b->Wnoise != nullptr)) {
        // at most 64 tokens: routing, dispatch and the gate statistics in one launch
        REQUIRE_PTR(b->x);
        REQUIRE_PTR(b->Wg);
        OPTIONAL_PTR(b->Wnoise);
        OPTIONAL_PTR(b->noise);
        OPTIONAL_PTR(b->bias);
        REQUIRE_PTR(b->topk_idx);
        REQUIRE_PTR(b->topk_w);
        REQUIRE_PTR(b->probs_sum);
        REQUIRE_PTR(b->importance);
        REQUIRE_PTR(b->x_perm);
        REQUIRE_PTR(b->row_token);
        REQUIRE_PTR(b->slot_row);
        REQUIRE_PTR(b->counts);
        REQUIRE_PTR(b->kept);
        REQUIRE_PTR(b->offsets);
        if (b->Wnoise != nullptr && b->noise == nullptr)
            return fail(MOE_ERR_INVALID_ARG, "%s: Wnoise given without the noise draws", fn);
        if ((rc = check_ws(fn, p, ws, ws_bytes)) != MOE_OK)
            return rc;
        if ((rc = after_launch(fn, launch_front_small(p, b, static_cast<char *>(ws),
                                                      (cudaStream_t)stream))) != MOE_OK)
            return rc;
        if ((rc = moe_expert_ffn(p, b->x_perm, b->offsets, b->W13_e, b->W2_e, b->h, b->out, ws,
                                 ws_bytes, stream)) != MOE_OK)
            return rc;
        return moe_combine(p, b->out, b->slot_row, b->topk_w, b->y, stream);
    }
    if ((rc = route_impl("moe_forward", p, b->x, b->Wg, b->Wnoise, b->router_packed, b->noise,
                         b->bias, b->topk_idx, b->topk_w, b->probs_sum, b->importance, ws,
                         ws_bytes, stream)) != MOE_OK)
        return rc;
    if ((rc = moe_dispatch_routed(p, b->x, b->topk_idx, b->x_perm, b->row_token, b->slot_row,
                                  b->counts, b->kept, b->offsets, ws, ws_bytes, stream)) !=
        MOE_OK)
        return rc;
    if ((rc = moe_expert_ffn(p, b->x_perm, b->offsets, b->W13_e, b->W2_e, b->h, b->out, ws,
                             ws_bytes, stream)) != MOE_OK)
        return rc;
    if ((rc = moe_combine(p, b->out, b->slot_row, b->topk_w, b->y, stream)) != MOE_OK)
        return rc;
    return moe_gate_stats(p, b->counts, b->probs_sum, b->f, b->P, b->loss, stream);
}

// ---------------------------------------------------------------- residual MoE

int moe_partition_residual(const void *W1, const void *W3, const void *W2, int32_t d,
                           int32_t d_ff, int32_t E, const int32_t *shared_idx, int32_t m_s,
                           const int32_t *perm_rest, int32_t dtype, void *W13_e, void *W2_e,
                           void *W13_s, void *W2_s, void *ws, void *stream)
{
    const char *fn = "moe_partition_residual";
    REQUIRE_PTR(W1);
    REQUIRE_PTR(W3);
    REQUIRE_PTR(W2);
    REQUIRE_PTR(shared_idx);
    REQUIRE_PTR(perm_rest);
    REQUIRE_PTR(W13_e);
    REQUIRE_PTR(W2_e);
    REQUIRE_PTR(W13_s);
    REQUIRE_PTR(W2_s);
    OPTIONAL_PTR(ws);
    if (dtype != MOE_BF16 && dtype != MOE_F32)
        return fail(MOE_ERR_DTYPE, "%s: dtype=%d", fn, dtype);
    if (E < 1 || E > MOE_MAX_EXPERTS)
        return fail(MOE_ERR_INVALID_ARG, "%s: E=%d outside [1,%d]", fn, E, MOE_MAX_EXPERTS);
    if (d < 8 || d % 8 != 0)
        return fail(MOE_ERR_SHAPE, "%s: d=%d is not a positive multiple of 8", fn, d);
    if (d_ff < 2 || d_ff > (1 << 22))
        return fail(MOE_ERR_SHAPE, "%s: d_ff=%d", fn, d_ff);
    if (m_s < 1 || m_s >= d_ff || (d_ff - m_s) % E != 0)
        return fail(MOE_ERR_SHAPE,
                    "%s: need 1 <= m_s < d_ff and (d_ff - m_s) divisible by E (m_s=%d, d_ff=%d, "
                    "E=%d)",
                    fn, m_s, d_ff, E);
    const int m = (d_ff - m_s) / E;
    int32_t *status = reinterpret_cast<int32_t *>(ws);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = launch_partition(W1, W3, W2, d, d_ff, E, m, MOE_PARTITION_DISJOINT, perm_rest,
                                     dtype, W13_e, W2_e, status, s);
    if (e == cudaSuccess)
        e = launch_partition(W1, W3, W2, d, d_ff, 1, m_s, MOE_PARTITION_DISJOINT, shared_idx,
                             dtype, W13_s, W2_s, status, s);
    return after_launch(fn, e);
}

int moe_combine_residual(const moe_params_t *p, const void *out, const int32_t *slot_row,
                         const float *topk_w, const void *resid, void *y, void *stream)
{
    const char *fn = "moe_combine_residual";
    int rc = check_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    REQUIRE_TOK(out);
    REQUIRE_TOK(slot_row);
    REQUIRE_TOK(topk_w);
    REQUIRE_TOK(resid);
    REQUIRE_TOK(y);
    if (p->T == 0)
        return ok();
    cudaError_t e = launch_combine(p, out, slot_row, topk_w, y, (cudaStream_t)stream, resid);
    return after_launch(fn, e);
}

int moe_forward_residual(const moe_params_t *p, const moe_buffers_t *b, const void *W13_s,
                         const void *W2_s, int32_t m_s, void *h_s, void *out_s, void *ws,
                         size_t ws_bytes, void *stream)
{
    const char *fn = "moe_forward_residual";
    int rc = check_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    if (b == nullptr)
        return fail(MOE_ERR_INVALID_ARG, "%s: buffers is NULL", fn);
    if (m_s < 1 || m_s > 1 << 20)
        return fail(MOE_ERR_SHAPE, "%s: m_s=%d", fn, m_s);
    REQUIRE_PTR(W13_s);
    REQUIRE_PTR(W2_s);
    REQUIRE_TOK(h_s);
    REQUIRE_TOK(out_s);
    REQUIRE_TOK(b->y);
    REQUIRE_PTR(b->loss);
    REQUIRE_PTR(b->f);
    REQUIRE_PTR(b->P);
    if ((rc = check_ws(fn, p, ws, ws_bytes)) != MOE_OK)
        return rc;
    // the shared block: one expert of width m_s that every token goes to
    moe_params_t ps = *p;
    ps.E = 1;
    ps.k = 1;
    ps.m = m_s;
    ps.capacity = -1;
    if ((rc = check_params(fn, &ps)) != MOE_OK || (rc = check_ws(fn, &ps, ws, ws_bytes)) != MOE_OK)
        return rc;
    if ((rc = moe_route(p, b->x, b->Wg, b->Wnoise, b->noise, b->bias, b->topk_idx, b->topk_w,
                        b->probs_sum, b->importance, ws, ws_bytes, stream)) != MOE_OK)
        return rc;
    if ((rc = moe_dispatch_routed(p, b->x, b->topk_idx, b->x_perm, b->row_token, b->slot_row,
                                  b->counts, b->kept, b->offsets, ws, ws_bytes, stream)) !=
        MOE_OK)
        return rc;
    if ((rc = moe_expert_ffn(p, b->x_perm, b->offsets, b->W13_e, b->W2_e, b->h, b->out, ws,
                             ws_bytes, stream)) != MOE_OK)
        return rc;
    if (p->T > 0) {
        int32_t *range = reinterpret_cast<int32_t *>(ws) + kWsTokenRangeWord;
        cudaError_t e = launch_token_range(range, p->T, (cudaStream_t)stream);
        if (e != cudaSuccess)
            return cuda_fail(e, fn);
        if ((rc = moe_expert_ffn(&ps, b->x, range, W13_s, W2_s, h_s, out_s, ws, ws_bytes,
                                 stream)) != MOE_OK)
            return rc;
    }
    if ((rc = moe_combine_residual(p, b->out, b->slot_row, b->topk_w, out_s, b->y, stream)) !=
        MOE_OK)
        return rc;
    return moe_gate_stats(p, b->counts, b->probs_sum, b->f, b->P, b->loss, stream);
}

}  // extern "C"
