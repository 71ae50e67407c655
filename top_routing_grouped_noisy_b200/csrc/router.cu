// router.cu -- a1: noisy Top-K gate ("Llama 3 Meets MoE: Efficient Upcycling",
// section 3 "核心公式", Noisy Top-k routing; section 5, Mixtral vs ST router).
//
//   L_t = x_t W_g (+ b),  H_t = L_t + eps_t * Softplus(x_t W_noise)
//   idx_t = KeepTopK(H_t, k)   (ties -> lower expert index; slot j = j-th largest)
//   Mixtral: G_tj = softmax over the k kept H;  ST: G_tj = softmax(H_t)[idx_tj]
// plus per-CTA partial sums of softmax(H_t) (for P) and of G (importance).
//
// Kernels here: the f32 router (one warp per token on the CUDA cores), the
// split-K router for batches of at most 64 tokens, and the fixed-order sum of
// per-CTA partials.  bf16 batches above that size run on the tensor cores
// (router_tc.cu).
#include <math.h>

#include "common.cuh"
#include "dispatch_scan.cuh"
#include "gate.cuh"
#include "kernels.h"

namespace moe {


// Per-CTA partial sums over its tokens, in token order.
__device__ void write_partials(int ntok, int E, const float *prob_s, const float *gw_s,
                               float *__restrict__ part)
{
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float sp = 0.f, sg = 0.f;
        for (int i = 0; i < ntok; ++i) {
            sp += prob_s[i * E + e];
            sg += gw_s[i * E + e];
        }
        part[((int64_t)blockIdx.x * 2 + 0) * E + e] = sp;
        part[((int64_t)blockIdx.x * 2 + 1) * E + e] = sg;
    }
}

// f32 router on the CUDA cores: one warp per token, 8 tokens per CTA.
__global__ void __launch_bounds__(256) router_f32_kernel(
    const float *__restrict__ x, const float *__restrict__ Wg, const float *__restrict__ Wn,
    int T, int d, int E, int k, const float *__restrict__ noise, const float *__restrict__ bias,
    int router_type, int32_t *__restrict__ idx_out, float *__restrict__ w_out,
    float *__restrict__ part, int32_t *status)
{
    pdl_wait();
    pdl_trigger();
    constexpr int TOK = kRouterWarps;
    extern __shared__ float smem[];
    const int nout = Wn ? 2 * E : E;
    float *lg = smem;                          // [TOK][2E]
    float *prob_s = lg + TOK * 2 * E;          // [TOK][E]
    float *gw_s = prob_s + TOK * E;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * TOK + warp;
    if (t < T) {
        for (int o0 = 0; o0 < nout; o0 += 16) {
            float acc[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                acc[i] = 0.f;
            for (int c = lane; c < d; c += 32) {
                const float xv = x[t * d + c];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int o = o0 + i;
                    if (o < nout) {
                        const float w = o < E ? Wg[(int64_t)c * E + o] : Wn[(int64_t)c * E + o - E];
                        acc[i] = fmaf(xv, w, acc[i]);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float v = acc[i];
#pragma unroll
                for (int s = 16; s > 0; s >>= 1)
                    v += __shfl_xor_sync(0xffffffffu, v, s);
                if (lane == 0 && o0 + i < nout)
                    lg[warp * 2 * E + o0 + i] = v;
            }
        }
        __syncwarp();
        if (lane == 0)
            finish_token(t, lg + warp * 2 * E, E, k, Wn != nullptr, noise, bias, router_type,
                         idx_out, w_out, prob_s + warp * E, gw_s + warp * E, status);
    }
    __syncthreads();
    const int ntok = (int)((int64_t)T - (int64_t)blockIdx.x * TOK < TOK ? (int64_t)T - (int64_t)blockIdx.x * TOK : TOK);
    write_partials(ntok, E, prob_s, gw_s, part);
}

// probs_sum[e], importance[e] = fixed-order sums of the per-CTA partials (f64 accumulate).
__global__ void __launch_bounds__(1024) router_finalize_kernel(const float *__restrict__ part,
                                                               int nblk, int E,
                                                               float *__restrict__ probs_sum,
                                                               float *__restrict__ importance)
{
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int o = warp; o < 2 * E; o += blockDim.x / 32) {
        const int which = o / E, e = o % E;
        double s = 0.0;
        for (int b = lane; b < nblk; b += 32)
            s += (double)part[((int64_t)b * 2 + which) * E + e];
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1)
            s += __shfl_xor_sync(0xffffffffu, s, sh);
        if (lane == 0)
            (which == 0 ? probs_sum : importance)[e] = (float)s;
    }
}


// ---------------------------------------------------------------- T <= 64 tokens
// Decode-sized batches: a few tokens cannot keep the split-over-warps kernel
// busy, so K is split over kRouterSmallSplit CTAs instead.  Each CTA stages its K slice
// of x and of [W_g | W_noise] (read in place, no transpose) in shared memory and
// writes partial logits part[ks][t][o]; one finishing CTA adds the slices in a
// fixed order, runs the per-token gate and the token sums.

template <typename E_T>
__global__ void __launch_bounds__(256) router_small_partial_kernel(
    const E_T *__restrict__ x, const E_T *__restrict__ Wg, const E_T *__restrict__ Wn, int T,
    int d, int E, float *__restrict__ part)
{
    pdl_trigger();  // early, so that the kernels after it are resident sooner
    pdl_wait();
    extern __shared__ float sm[];
    router_small_slice(blockIdx.x, x, Wg, Wn, T, d, E, part, sm);
}

struct SmallFinishBar {
    __device__ void operator()() const { __syncthreads(); }
};

// ... then, for a2, the count step of the counting sort on the indices just written
// (dispatch_count_kernel's arithmetic: one ballot per expert and 32-token chunk, then
// the exclusive scan over chunks per expert into rank bases and routed counts), so no
// count launch follows the small router.
__global__ void __launch_bounds__(256) router_small_finish_kernel(
    const float *__restrict__ part, int T, int E, int k, int noisy,
    const float *__restrict__ noise, const float *__restrict__ bias, int router_type,
    int32_t *__restrict__ idx_out, float *__restrict__ w_out, float *__restrict__ probs_sum,
    float *__restrict__ importance, int32_t *status, int32_t *__restrict__ hist,
    int32_t *__restrict__ dcounts)
{
    pdl_trigger();  // early, as in the partial kernel
    pdl_wait();
    extern __shared__ float sm[];
    router_small_finish(part, T, E, k, noisy, noise, bias, router_type, idx_out, w_out,
                        probs_sum, importance, status, sm);
    __syncthreads();  // this CTA's indices are visible to all its threads
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nch = (T + kDispatchChunk - 1) / kDispatchChunk;
    for (int c = warp; c < nch; c += (int)(blockDim.x >> 5)) {
        const int t = c * kDispatchChunk + lane;
        int ej[MOE_MAX_TOPK];
        for (int j = 0; j < k; ++j) {
            int e = -1;
            if (t < T) {
                e = idx_out[t * k + j];
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
                hist[e * nch + c] = __popc(b);
        }
    }
    __syncthreads();
    scan_chunk_counts(hist, E, nch, dcounts, nullptr, 0, (int)threadIdx.x, (int)blockDim.x,
                      SmallFinishBar());
}

// ---------------------------------------------------------------- front of the layer
// moe_forward on a batch of at most 64 tokens that the decode kernel does not take:
// a1 (split-K logits, then the gate), a2 (tables and the copy of x into expert
// order) and a6 (the gate statistics) in one cooperative launch of
// kRouterSmallSplit CTAs, joined by two grid barriers instead of four launches
// that each wait for the one before.  Arithmetic and orders are those of the
// separate kernels: slices added in slice order, finish_token per token, token sums
// in token order, ranks stable by token, the gate statistics in f64.
struct FrontArgs {
    const void *x, *Wg, *Wn;
    const float *noise, *bias;
    int T, d, E, k, C, router_type;
    float lambda;
    float *part;            // [32][T][nout] slice logits
    float *prob, *gw;       // [T][E] softmax rows and gate weight rows
    int32_t *idx;
    float *w, *probs_sum, *importance;
    char *x_perm;
    int32_t *row_token, *slot_row, *counts, *kept, *offsets;
    float *f, *P, *loss;
    int32_t *status;
    int32_t *gbar;          // arrivals, CTAs done (both zero between launches)
    uint64_t wait_ns;
};

// Grid barrier `n` (1 or 2) of the front kernel: every CTA adds one arrival and waits
// for n * gridDim.x of them.  The count only grows within a launch; the last CTA to
// finish the launch sets both words back to zero (front_small_done), so they are
// zero again after a wait that ran out too.  A wait past the limit records
// MOE_ERR_DEVICE_TIMEOUT and stops waiting.
__device__ __forceinline__ void front_grid_sync(const FrontArgs &a, int n,
                                                volatile int32_t *abort_flag)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(a.gbar, 1);
        const int target = n * (int)gridDim.x;
        const uint64_t t0 = globaltimer_ns();
        while (!*abort_flag && ld_acquire_gpu(a.gbar) < target) {
            if (globaltimer_ns() - t0 > a.wait_ns) {
                set_status(a.status, MOE_ERR_DEVICE_TIMEOUT);
                *abort_flag = 1;
                break;
            }
            __nanosleep(32);
        }
        __threadfence();
    }
    __syncthreads();
}

// Called by thread 0 of every CTA once it is past both barriers.
__device__ __forceinline__ void front_small_done(const FrontArgs &a)
{
    if (atomicAdd(a.gbar + 1, 1) == (int)gridDim.x - 1) {  // no CTA reads the count any more
        atomicExch(a.gbar, 0);
        atomicExch(a.gbar + 1, 0);
    }
}

template <typename E_T>
__global__ void __launch_bounds__(256) front_small_kernel(const __grid_constant__ FrontArgs a)
{
    pdl_trigger();  // the expert GEMM may become resident and prefetch its weights
    pdl_wait();
    extern __shared__ float sm[];
    __shared__ int32_t s_idx[kRouterSmallTokens * MOE_MAX_TOPK];
    __shared__ int32_t s_row[kRouterSmallTokens * MOE_MAX_TOPK];
    __shared__ int32_t s_cnt[MOE_MAX_EXPERTS], s_kept[MOE_MAX_EXPERTS];
    __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1];
    __shared__ float s_lg[8][2 * MOE_MAX_EXPERTS];
    constexpr int kChunks = kRouterSmallTokens * MOE_MAX_TOPK / 32;
    __shared__ int32_t s_ccnt[kChunks][MOE_MAX_EXPERTS], s_cbase[kChunks][MOE_MAX_EXPERTS];
    __shared__ double s_fp[MOE_MAX_EXPERTS];
    constexpr int kTokPerCta = kRouterSmallTokens / kRouterSmallSplit;
    static_assert(kRouterSmallTokens % kRouterSmallSplit == 0, "tokens per CTA");
    __shared__ float s_noise[kTokPerCta][MOE_MAX_EXPERTS], s_bias[MOE_MAX_EXPERTS];
    __shared__ int32_t s_abort;
    const int T = a.T, E = a.E, k = a.k, G = (int)gridDim.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nout = a.Wn != nullptr ? 2 * E : E;
    if (threadIdx.x == 0)
        s_abort = 0;
    // the noise draws and bias of this CTA's tokens, fetched while the logits are made
    for (int i = threadIdx.x; i < kTokPerCta * E; i += blockDim.x) {
        const int q = i / E, e = i % E, t = (int)blockIdx.x + G * q;
        if (a.noise != nullptr && t < T)
            s_noise[q][e] = __ldg(a.noise + (int64_t)t * E + e);
        if (a.bias != nullptr && q == 0)
            s_bias[e] = __ldg(a.bias + e);
    }
    // a1, step 1: this CTA's K slice of every token's logits
    router_small_slice(blockIdx.x, static_cast<const E_T *>(a.x), static_cast<const E_T *>(a.Wg),
                       static_cast<const E_T *>(a.Wn), T, a.d, E, a.part, sm);
    front_grid_sync(a, 1, &s_abort);
    // a1, step 2: the gate of tokens blockIdx.x and blockIdx.x + G (warps 0 and 1)
    if (warp < kTokPerCta && (int)blockIdx.x + G * warp < T) {
        const int t = (int)blockIdx.x + G * warp;
        float *lg = s_lg[warp];
        for (int o = lane; o < nout; o += 32) {
            float v[kRouterSmallSplit];
#pragma unroll
            for (int ks = 0; ks < kRouterSmallSplit; ++ks)
                v[ks] = __ldcg(a.part + ((int64_t)ks * T + t) * nout + o);
            float acc = 0.f;
#pragma unroll
            for (int ks = 0; ks < kRouterSmallSplit; ++ks)
                acc += v[ks];
            lg[o] = acc;
        }
        __syncwarp();
        // token t's outputs as row 0 of shifted arrays; noise and bias from smem
        const float *bias_s = a.bias != nullptr ? s_bias : nullptr;
        if (E <= 32)
            gate_token_warp(lg, E, k, a.Wn != nullptr, s_noise[warp], bias_s, a.router_type,
                            a.idx + (int64_t)t * k, a.w + (int64_t)t * k,
                            a.prob + (int64_t)t * E, a.gw + (int64_t)t * E, a.status);
        else if (lane == 0)
            finish_token(0, lg, E, k, a.Wn != nullptr, s_noise[warp], bias_s, a.router_type,
                         a.idx + (int64_t)t * k, a.w + (int64_t)t * k, a.prob + (int64_t)t * E,
                         a.gw + (int64_t)t * E, a.status);
        __syncwarp();
    }
    front_grid_sync(a, 2, &s_abort);
    if (threadIdx.x == 0)
        front_small_done(a);
    // a2: every CTA counts all T*k assignments; CTAs 1..G-1 write the tables and x_perm
    // rows of tokens 1 + t mod (G - 1), so that CTA 0 goes straight on to the token sums
    // and a6.  The entries are token-major and a token's k experts differ, so an entry's rank
    // (its expert's entries of earlier tokens) is the count of equal entries before it:
    // per 32-entry chunk one ballot per expert, a scan over chunks, then match_any.
    const int n = T * k, nch = (n + 31) / 32, nwarps = (int)(blockDim.x >> 5);
    for (int i = threadIdx.x; i < n; i += blockDim.x)
        s_idx[i] = __ldcg(a.idx + i);
    __syncthreads();
    for (int c = warp; c < nch; c += nwarps) {
        const int i = c * 32 + lane;
        const int e = i < n ? s_idx[i] : -1;
        for (int x = 0; x < E; ++x) {
            const unsigned b = __ballot_sync(0xffffffffu, e == x);
            if (lane == 0)
                s_ccnt[c][x] = __popc(b);
        }
    }
    __syncthreads();
    for (int x = threadIdx.x; x < E; x += blockDim.x) {
        int run = 0;
        for (int c = 0; c < nch; ++c) {
            s_cbase[c][x] = run;
            run += s_ccnt[c][x];
        }
        s_cnt[x] = run;
        s_kept[x] = a.C < 0 ? run : min(run, a.C);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int e = 0; e < E; ++e) {
            s_off[e] = acc;
            acc += s_kept[e];
        }
        s_off[E] = acc;
    }
    __syncthreads();
    for (int c = warp; c < nch; c += nwarps) {
        const int i = c * 32 + lane;
        const int e = i < n ? s_idx[i] : -1;
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int t = i / k;
        if (i < n && 1 + t % (G - 1) == (int)blockIdx.x) {
            int row = -1;
            if (e < 0 || e >= E) {
                set_status(a.status, MOE_ERR_DEVICE_BADINDEX);
            } else {
                const int rank = s_cbase[c][e] + __popc(same & ((1u << lane) - 1u));
                if (rank < s_kept[e]) {
                    row = s_off[e] + rank;
                    a.row_token[row] = t;
                }
            }
            s_row[i] = row;
            a.slot_row[i] = row;
        }
    }
    __syncthreads();
    const int nv = a.d * (int)sizeof(E_T) / 16;
    const char *xb = static_cast<const char *>(a.x);
    for (int t = (int)blockIdx.x - 1; blockIdx.x > 0 && t < T; t += G - 1) {
        const char *src = xb + (int64_t)t * nv * 16;
        for (int v = threadIdx.x; v < nv; v += blockDim.x) {
            const uint4 val = ld_nc(src + (int64_t)v * 16);
            for (int j = 0; j < k; ++j) {
                const int row = s_row[t * k + j];
                if (row >= 0)
                    st_v4(a.x_perm + ((int64_t)row * nv + v) * 16, val);
            }
        }
    }
    if (blockIdx.x != 0)
        return;
    // CTA 0: counts, kept, offsets, the token sums and a6
    for (int e = threadIdx.x; e <= E; e += blockDim.x) {
        a.offsets[e] = s_off[e];
        if (e < E) {
            a.counts[e] = s_cnt[e];
            a.kept[e] = s_kept[e];
        }
    }
    float *pg = sm;  // [2][T][E]: every token's softmax row, then its gate weight row
    for (int i = threadIdx.x; i < 2 * T * E; i += blockDim.x)
        pg[i] = __ldcg(a.prob + i);  // gw follows prob in the workspace
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float sp = 0.f, sg = 0.f;
#pragma unroll 16
        for (int t = 0; t < T; ++t) {
            sp += pg[t * E + e];
            sg += pg[(T + t) * E + e];
        }
        a.probs_sum[e] = sp;
        a.importance[e] = sg;
        const double fe = (double)s_cnt[e] / ((double)T * k);
        const double pe = (double)sp / (double)T;
        a.f[e] = (float)fe;
        a.P[e] = (float)pe;
        s_fp[e] = fe * pe;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double sum = 0.0;
        for (int e = 0; e < E; ++e)
            sum += s_fp[e];
        a.loss[0] = (float)(a.lambda * sum);
    }
}

// The split-K slice (x and weight columns), reused for the token sums' [2][T][E] rows.
static size_t front_small_smem(const moe_params_t *p, bool noisy)
{
    const int nout = noisy ? 2 * p->E : p->E;
    const size_t slice = router_small_slice_smem(p->T, p->d, nout, p->dtype);
    const size_t sums = sizeof(float) * 2 * (size_t)p->T * p->E;
    return slice > sums ? slice : sums;
}

// Exactly the batches whose moe_route takes the split-K router (so moe_forward and
// the step calls give the same bytes): not the decode router's, at most 64 tokens,
// and both of the split-K kernels' shared memory within 48 KB.
bool front_small_fits(const moe_params_t *p, bool noisy)
{
    const int nout = noisy ? 2 * p->E : p->E;
    const size_t finish_smem =
        sizeof(float) * ((size_t)p->T * nout + 2 * (size_t)p->T * p->E);
    return p->T > 0 && p->T <= kRouterSmallTokens && !decode_route_fits(p, noisy) &&
           front_small_smem(p, noisy) <= 48 * 1024 && finish_smem <= 48 * 1024 &&
           (p->dtype == MOE_BF16 || p->dtype == MOE_F32);
}

cudaError_t launch_front_small(const moe_params_t *p, const moe_buffers_t *b, char *ws,
                               cudaStream_t s)
{
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    if (!attr_done[dev]) {  // up to 48 KB of slices on top of the static tables
        if ((e = cudaFuncSetAttribute(front_small_kernel<bf16>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      48 * 1024)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(front_small_kernel<float>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      48 * 1024)) != cudaSuccess)
            return e;
        attr_done[dev] = true;
    }
    const WsLayout L = ws_layout(p);
    FrontArgs a{};
    a.x = b->x;
    a.Wg = b->Wg;
    a.Wn = b->Wnoise;
    a.noise = b->noise;
    a.bias = b->bias;
    a.T = p->T;
    a.d = p->d;
    a.E = p->E;
    a.k = p->k;
    a.C = p->capacity;
    a.router_type = p->router_type;
    a.lambda = p->balance_lambda;
    a.part = reinterpret_cast<float *>(ws + L.rsmall);
    a.prob = reinterpret_cast<float *>(ws + L.gsmall);
    a.gw = a.prob + (size_t)p->T * p->E;
    a.idx = b->topk_idx;
    a.w = b->topk_w;
    a.probs_sum = b->probs_sum;
    a.importance = b->importance;
    a.x_perm = static_cast<char *>(b->x_perm);
    a.row_token = b->row_token;
    a.slot_row = b->slot_row;
    a.counts = b->counts;
    a.kept = b->kept;
    a.offsets = b->offsets;
    a.f = b->f;
    a.P = b->P;
    a.loss = b->loss;
    a.status = reinterpret_cast<int32_t *>(ws);
    a.gbar = reinterpret_cast<int32_t *>(ws) + kWsFrontBarrierWord;
    a.wait_ns = wait_limit_ns();
    // every CTA must be resident for the grid barriers: a cooperative launch
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.gridDim = dim3(kRouterSmallSplit);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = front_small_smem(p, b->Wnoise != nullptr);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = p->dtype == MOE_BF16 ? cudaLaunchKernelEx(&cfg, front_small_kernel<bf16>, a)
                             : cudaLaunchKernelEx(&cfg, front_small_kernel<float>, a);
    count_launch();
    return e == cudaSuccess ? cudaGetLastError() : e;
}

cudaError_t launch_route(const moe_params_t *p, const void *x, const void *Wg,
                         const void *Wnoise, const void *Wt, const float *noise,
                         const float *bias, int32_t *idx, float *w, float *probs_sum,
                         float *importance, char *ws, int32_t *status, cudaStream_t s)
{
    const WsLayout L = ws_layout(p);
    float *part = reinterpret_cast<float *>(ws + L.rpart);
    // every path leaves the chunk bases and routed counts of its indices in the
    // workspace (for moe_dispatch_routed): the tensor-core router counts them in its
    // gate epilogue, the other paths end with the count kernel of a2
    int32_t *hist = reinterpret_cast<int32_t *>(ws + L.hist);
    int32_t *dcounts = reinterpret_cast<int32_t *>(ws + L.dcounts);
    int32_t *dcounter = reinterpret_cast<int32_t *>(ws) + kWsCounterWord;
    int nblk = 0;
    cudaError_t e = cudaSuccess;
    const int small_noisy = Wnoise != nullptr;
    const int small_nout = small_noisy ? 2 * p->E : p->E;
    const size_t sm1 = router_small_slice_smem(p->T, p->d, small_nout, p->dtype);
    const size_t sm2 =
        sizeof(float) * ((size_t)p->T * small_nout + 2 * (size_t)p->T * p->E);
    if (decode_route_fits(p, Wnoise != nullptr)) {  // the decode forward's router, one CTA
        if ((e = launch_route_decode(p, x, Wg, Wnoise, noise, bias, idx, w, probs_sum,
                                     importance, status, s)) != cudaSuccess)
            return e;
        return launch_count(p, idx, hist, dcounter, dcounts, status, s);
    }
    if (p->T > 0 && p->T <= kRouterSmallTokens && sm1 <= 48 * 1024 && sm2 <= 48 * 1024) {
        const int noisy = small_noisy;
        float *sp = reinterpret_cast<float *>(ws + L.rsmall);
        if (p->dtype == MOE_BF16)
            launch_pdl(router_small_partial_kernel<bf16>, dim3(kRouterSmallSplit), dim3(256), sm1, s, 
                (const bf16 *)x, (const bf16 *)Wg, (const bf16 *)Wnoise, p->T, p->d, p->E, sp);
        else
            launch_pdl(router_small_partial_kernel<float>, dim3(kRouterSmallSplit), dim3(256), sm1, s, 
                (const float *)x, (const float *)Wg, (const float *)Wnoise, p->T, p->d, p->E, sp);
        count_launch();
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
        launch_pdl(router_small_finish_kernel, dim3(1), dim3(256), sm2, s, sp, p->T, p->E, p->k, noisy, noise, bias,
                                                       p->router_type, idx, w, probs_sum,
                                                       importance, status, hist, dcounts);
        count_launch();
        return cudaGetLastError();  // the finishing CTA also did a2's count step
    }
    if (p->T > 0 && p->dtype == MOE_BF16) {
        int32_t *counter = reinterpret_cast<int32_t *>(ws) + kWsRouterCounterWord;
        if (Wt == nullptr) {  // pack the router weights into the workspace first
            Wt = ws + L.wt;
            if ((e = launch_router_pack(p, Wg, Wnoise, ws + L.wt, s)) != cudaSuccess)
                return e;
        }
        return launch_route_tc(p, x, Wt, Wnoise != nullptr, noise, bias, idx, w, probs_sum,
                               importance, part, counter, hist, dcounts, status, s);
    }
    if (p->T > 0) {
        nblk = ceil_div(p->T, kRouterWarps);
        const size_t smem = sizeof(float) * ((size_t)kRouterWarps * 4 * p->E);
        launch_pdl(router_f32_kernel, dim3(nblk), dim3(256), smem, s, 
            (const float *)x, (const float *)Wg, (const float *)Wnoise, p->T, p->d, p->E, p->k,
            noise, bias, p->router_type, idx, w, part, status);
        count_launch();
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
    }
    launch_pdl(router_finalize_kernel, dim3(1), dim3(1024), 0, s, part, nblk, p->E, probs_sum, importance);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess)
        return e;
    return launch_count(p, idx, hist, dcounter, dcounts, status, s);
}

}  // namespace moe
