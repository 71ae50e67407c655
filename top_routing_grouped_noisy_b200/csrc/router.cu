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
    pdl_wait();
    pdl_trigger();
    extern __shared__ float sm[];
    router_small_slice(blockIdx.x, x, Wg, Wn, T, d, E, part, sm);
}

__global__ void __launch_bounds__(256) router_small_finish_kernel(
    const float *__restrict__ part, int T, int E, int k, int noisy,
    const float *__restrict__ noise, const float *__restrict__ bias, int router_type,
    int32_t *__restrict__ idx_out, float *__restrict__ w_out, float *__restrict__ probs_sum,
    float *__restrict__ importance, int32_t *status)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ float sm[];
    router_small_finish(part, T, E, k, noisy, noise, bias, router_type, idx_out, w_out,
                        probs_sum, importance, status, sm);
}

// ---------------------------------------------------------------- small-batch forward
// For at most kDecodeMaxTokens tokens moe_forward runs the split-K router slices
// and then, in the CTA that finishes its slice last, adds the slices, builds the
// dispatch tables and computes the gate statistics: one launch on a path that is
// bound by latency.  The arithmetic is that of router_small_finish_kernel,
// dispatch_count_kernel + dispatch_scatter_kernel ("Llama 3 Meets MoE", section 3
// "容量因子": stable by token, assignments past the capacity dropped) and
// gate_stats_kernel ("LLaMA-MoE v2", section "门控机制设计"), so moe_forward gives the
// same bits as the step calls.  x_perm is written by the GEMM 1 kernel, which reads
// the rows of x through row_token.
__device__ void route_dispatch_small_body(
    float *lg, int T, int E, int k, int C, int noisy,
    const float *__restrict__ noise, const float *__restrict__ bias, int router_type,
    float lambda, int32_t *__restrict__ idx, float *__restrict__ w_out,
    float *__restrict__ probs_sum, float *__restrict__ importance, int32_t *__restrict__ counts,
    int32_t *__restrict__ kept, int32_t *__restrict__ offsets, int32_t *__restrict__ row_token,
    int32_t *__restrict__ slot_row, float *__restrict__ f, float *__restrict__ P,
    float *__restrict__ loss, int32_t *status)
{
    __shared__ int32_t s_idx[kDecodeMaxTokens * MOE_MAX_TOPK];
    __shared__ int32_t s_cnt[MOE_MAX_EXPERTS], s_kept[MOE_MAX_EXPERTS];
    __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1];
    __shared__ double s_fp[MOE_MAX_EXPERTS];
    const int nout = noisy ? 2 * E : E;
    router_gate_tokens(lg, T, E, k, noisy, noise, bias, router_type, idx, w_out, probs_sum,
                       importance, status, lg + (size_t)T * nout);
    __syncthreads();
    for (int i = threadIdx.x; i < T * k; i += blockDim.x)
        s_idx[i] = idx[i];
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int c = 0;
        for (int i = 0; i < T * k; ++i)
            c += s_idx[i] == e;
        s_cnt[e] = c;
        s_kept[e] = C < 0 ? c : min(c, C);
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
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        counts[e] = s_cnt[e];
        kept[e] = s_kept[e];
    }
    for (int e = threadIdx.x; e <= E; e += blockDim.x)
        offsets[e] = s_off[e];
    for (int i = threadIdx.x; i < T * k; i += blockDim.x) {
        const int t = i / k, e = s_idx[i];
        int row = -1;
        if (e < 0 || e >= E) {
            set_status(status, MOE_ERR_DEVICE_BADINDEX);
        } else {
            int rank = 0;  // the expert's assignments of earlier tokens
            for (int i2 = 0; i2 < t * k; ++i2)
                rank += s_idx[i2] == e;
            if (rank < s_kept[e]) {
                row = s_off[e] + rank;
                row_token[row] = t;
            }
        }
        slot_row[i] = row;
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const double fe = (double)s_cnt[e] / ((double)T * k);
        const double pe = (double)probs_sum[e] / (double)T;
        f[e] = (float)fe;
        P[e] = (float)pe;
        s_fp[e] = fe * pe;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double sfp = 0.0;
        for (int i = 0; i < E; ++i)
            sfp += s_fp[i];
        loss[0] = (float)(lambda * sfp);
    }
}

// The slices of the split-K router in kRouterSmallSplit CTAs; the CTA that finishes
// last (ticket counter, zero between calls, reset by that CTA) runs the body above.
// No CTA waits for another.
__global__ void __launch_bounds__(256) route_dispatch_small_kernel(
    const bf16 *__restrict__ x, const bf16 *__restrict__ Wg, const bf16 *__restrict__ Wn,
    int d, float *__restrict__ part, int32_t *counter, int T, int E, int k, int C,
    const float *__restrict__ noise, const float *__restrict__ bias, int router_type,
    float lambda, int32_t *__restrict__ idx, float *__restrict__ w_out,
    float *__restrict__ probs_sum, float *__restrict__ importance, int32_t *__restrict__ counts,
    int32_t *__restrict__ kept, int32_t *__restrict__ offsets, int32_t *__restrict__ row_token,
    int32_t *__restrict__ slot_row, float *__restrict__ f, float *__restrict__ P,
    float *__restrict__ loss, int32_t *status)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ float sm[];
    __shared__ int s_last;
    router_small_slice(blockIdx.x, x, Wg, Wn, T, d, E, part, sm);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
        s_last = atomicAdd(counter, 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (!s_last)
        return;
    __threadfence();
    const int nout = Wn != nullptr ? 2 * E : E;
    float *lg = sm;  // the slices added in order
    for (int i = threadIdx.x; i < T * nout; i += blockDim.x) {
        float v[kRouterSmallSplit];
#pragma unroll
        for (int ks = 0; ks < kRouterSmallSplit; ++ks)
            v[ks] = __ldcg(part + (int64_t)ks * T * nout + i);
        float acc = 0.f;
#pragma unroll
        for (int ks = 0; ks < kRouterSmallSplit; ++ks)
            acc += v[ks];
        lg[i] = acc;
    }
    __syncthreads();
    route_dispatch_small_body(lg, T, E, k, C, Wn != nullptr ? 1 : 0, noise, bias, router_type,
                              lambda, idx, w_out, probs_sum, importance, counts, kept, offsets,
                              row_token, slot_row, f, P, loss, status);
    if (threadIdx.x == 0)
        *counter = 0;
}

// ---------------------------------------------------------------- one-CTA router
// bf16 batches of at most 16 tokens with at most 32 logits: the logits on the tensor
// cores in one CTA (router_logits_one_cta), then the gate; with `dispatch`, also the
// dispatch tables and the gate statistics (moe_forward's decode path).  moe_route and
// moe_forward run the same logit and gate code, so the step calls reproduce the
// forward bit for bit.
template <int NT>
__global__ void __launch_bounds__(kOneWarps * 32) router_one_cta_kernel(
    const bf16 *__restrict__ x, const bf16 *__restrict__ Wg, const bf16 *__restrict__ Wn, int d,
    int T, int E, int k, int C, const float *__restrict__ noise, const float *__restrict__ bias,
    int router_type, float lambda, int dispatch, int32_t *__restrict__ idx,
    float *__restrict__ w_out, float *__restrict__ probs_sum, float *__restrict__ importance,
    int32_t *__restrict__ counts, int32_t *__restrict__ kept, int32_t *__restrict__ offsets,
    int32_t *__restrict__ row_token, int32_t *__restrict__ slot_row, float *__restrict__ f,
    float *__restrict__ P, float *__restrict__ loss, int32_t *status)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(16) char smo[];
    const int nout = Wn != nullptr ? 2 * E : E;
    float *lg = reinterpret_cast<float *>(smo + one_cta_logits_smem(NT));
    router_logits_one_cta<NT>(x, Wg, Wn, T, d, E, lg, smo);
    if (dispatch)
        route_dispatch_small_body(lg, T, E, k, C, Wn != nullptr ? 1 : 0, noise, bias,
                                  router_type, lambda, idx, w_out, probs_sum, importance, counts,
                                  kept, offsets, row_token, slot_row, f, P, loss, status);
    else
        router_gate_tokens(lg, T, E, k, Wn != nullptr ? 1 : 0, noise, bias, router_type, idx,
                           w_out, probs_sum, importance, status, lg + (size_t)T * nout);
}

static int one_cta_nt(const moe_params_t *p, bool noisy)
{
    const int nout = noisy ? 2 * p->E : p->E;
    if (p->dtype != MOE_BF16 || p->T < 1 || p->T > 16 || nout > 32)
        return 0;
    return (nout + 7) / 8;
}

static cudaError_t launch_one_cta(const moe_params_t *p, const void *x, const void *Wg,
                                  const void *Wn, const float *noise, const float *bias,
                                  int dispatch, int32_t *idx, float *w, float *probs_sum,
                                  float *importance, const moe_buffers_t *b, int32_t *status,
                                  cudaStream_t s)
{
    const int nt = one_cta_nt(p, Wn != nullptr);
    const size_t smem = one_cta_logits_smem(nt) + sizeof(float) * 16 * (32 + 2 * 32);
    static bool attr_done[64][5] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
#define MOE_ONE(NT)                                                                                do {                                                                                               if (!attr_done[dev][NT]) {                                                                         e = cudaFuncSetAttribute(router_one_cta_kernel<NT>,                                                                     cudaFuncAttributeMaxDynamicSharedMemorySize,                                                  (int)(one_cta_logits_smem(NT) + sizeof(float) * 16 * 96));             if (e != cudaSuccess)                                                                              return e;                                                                                  attr_done[dev][NT] = true;                                                                 }                                                                                              e = launch_pdl(router_one_cta_kernel<NT>, dim3(1), dim3(kOneWarps * 32), smem, s,                             (const bf16 *)x, (const bf16 *)Wg, (const bf16 *)Wn, p->d, p->T, p->E,                         p->k, p->capacity, noise, bias, p->router_type, p->balance_lambda,                            dispatch, idx, w, probs_sum, importance, b ? b->counts : nullptr,                             b ? b->kept : nullptr, b ? b->offsets : nullptr,                                             b ? b->row_token : nullptr, b ? b->slot_row : nullptr,                                       b ? b->f : nullptr, b ? b->P : nullptr, b ? b->loss : nullptr, status);     } while (0)
    if (nt == 1)
        MOE_ONE(1);
    else if (nt == 2)
        MOE_ONE(2);
    else if (nt == 3)
        MOE_ONE(3);
    else
        MOE_ONE(4);
#undef MOE_ONE
    count_launch();
    return e == cudaSuccess ? cudaGetLastError() : e;
}

static void small_router_smem(const moe_params_t *p, bool noisy, size_t *sm1, size_t *sm2)
{
    const int nout = noisy ? 2 * p->E : p->E;
    const int kc = router_small_kc(p->d);
    *sm1 = sizeof(float) * ((size_t)p->T * kc + (size_t)kc * nout);
    *sm2 = sizeof(float) * ((size_t)p->T * nout + 2 * (size_t)p->T * p->E);
}

bool small_forward_fits(const moe_params_t *p, bool noisy)
{
    if (p->dtype != MOE_BF16 || p->T < 1 || p->T > kDecodeMaxTokens)
        return false;
    size_t sm1, sm2;
    small_router_smem(p, noisy, &sm1, &sm2);
    return sm1 <= 48 * 1024 && sm2 <= 48 * 1024;
}

cudaError_t launch_route_dispatch_small(const moe_params_t *p, const moe_buffers_t *b, char *ws,
                                        int32_t *status, cudaStream_t s)
{
    const WsLayout L = ws_layout(p);
    float *sp = reinterpret_cast<float *>(ws + L.rsmall);
    const bool noisy = b->Wnoise != nullptr;
    if (one_cta_nt(p, noisy) > 0)
        return launch_one_cta(p, b->x, b->Wg, b->Wnoise, b->noise, b->bias, 1, b->topk_idx,
                              b->topk_w, b->probs_sum, b->importance, b, status, s);
    size_t sm1, sm2;
    small_router_smem(p, noisy, &sm1, &sm2);
    int32_t *counter = reinterpret_cast<int32_t *>(ws) + kWsSmallCounterWord;
    cudaError_t e = launch_pdl(route_dispatch_small_kernel, dim3(kRouterSmallSplit), dim3(256),
                               sm1 > sm2 ? sm1 : sm2, s, (const bf16 *)b->x, (const bf16 *)b->Wg,
                               (const bf16 *)b->Wnoise, p->d, sp, counter, p->T, p->E, p->k,
                               p->capacity, b->noise, b->bias, p->router_type,
                               p->balance_lambda, b->topk_idx, b->topk_w, b->probs_sum,
                               b->importance, b->counts, b->kept, b->offsets, b->row_token,
                               b->slot_row, b->f, b->P, b->loss, status);
    count_launch();
    return e;
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
    const int small_kc = router_small_kc(p->d);
    const size_t sm1 = sizeof(float) * ((size_t)p->T * small_kc + (size_t)small_kc * small_nout);
    const size_t sm2 =
        sizeof(float) * ((size_t)p->T * small_nout + 2 * (size_t)p->T * p->E);
    if (one_cta_nt(p, Wnoise != nullptr) > 0) {
        if ((e = launch_one_cta(p, x, Wg, Wnoise, noise, bias, 0, idx, w, probs_sum, importance,
                                nullptr, status, s)) != cudaSuccess)
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
                                                       importance, status);
        count_launch();
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
        return launch_count(p, idx, hist, dcounter, dcounts, status, s);
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
