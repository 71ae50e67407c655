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
// For at most kDecodeMaxTokens tokens moe_forward finishes the split-K router,
// builds the dispatch tables and computes the gate statistics in ONE CTA (three
// launches fewer on a path that is bound by launch latency).  The arithmetic is
// that of router_small_finish_kernel, dispatch_count/rank_kernel ("Llama 3 Meets
// MoE", section 3 "容量因子": stable by token, assignments past the capacity
// dropped) and gate_stats_kernel ("LLaMA-MoE v2", section "门控机制设计"), so
// moe_forward gives the same bits as the step calls.  x_perm is written by the
// GEMM 1 kernel, which reads the rows of x through row_token.
__global__ void __launch_bounds__(256) route_dispatch_small_kernel(
    const float *__restrict__ part, int T, int E, int k, int C, int noisy,
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
    __shared__ int32_t s_idx[kDecodeMaxTokens * MOE_MAX_TOPK];
    __shared__ int32_t s_cnt[MOE_MAX_EXPERTS], s_kept[MOE_MAX_EXPERTS];
    __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1];
    __shared__ double s_fp[MOE_MAX_EXPERTS];
    router_small_finish(part, T, E, k, noisy, noise, bias, router_type, idx, w_out, probs_sum,
                        importance, status, sm);
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
    size_t sm1, sm2;
    small_router_smem(p, noisy, &sm1, &sm2);
    cudaError_t e = launch_pdl(router_small_partial_kernel<bf16>, dim3(kRouterSmallSplit),
                               dim3(256), sm1, s, (const bf16 *)b->x, (const bf16 *)b->Wg,
                               (const bf16 *)b->Wnoise, p->T, p->d, p->E, sp);
    count_launch();
    if (e != cudaSuccess)
        return e;
    e = launch_pdl(route_dispatch_small_kernel, dim3(1), dim3(256), sm2, s, (const float *)sp,
                   p->T, p->E, p->k, p->capacity, noisy ? 1 : 0, b->noise, b->bias,
                   p->router_type, p->balance_lambda, b->topk_idx, b->topk_w, b->probs_sum,
                   b->importance, b->counts, b->kept, b->offsets, b->row_token, b->slot_row,
                   b->f, b->P, b->loss, status);
    count_launch();
    return e;
}

cudaError_t launch_route(const moe_params_t *p, const void *x, const void *Wg,
                         const void *Wnoise, const float *noise, const float *bias,
                         int32_t *idx, float *w, float *probs_sum, float *importance,
                         char *ws, int32_t *status, cudaStream_t s)
{
    const WsLayout L = ws_layout(p);
    float *part = reinterpret_cast<float *>(ws + L.rpart);
    int nblk = 0;
    cudaError_t e = cudaSuccess;
    const int small_noisy = Wnoise != nullptr;
    const int small_nout = small_noisy ? 2 * p->E : p->E;
    const int small_kc = router_small_kc(p->d);
    const size_t sm1 = sizeof(float) * ((size_t)p->T * small_kc + (size_t)small_kc * small_nout);
    const size_t sm2 =
        sizeof(float) * ((size_t)p->T * small_nout + 2 * (size_t)p->T * p->E);
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
        return cudaGetLastError();
    }
    if (p->T > 0 && p->dtype == MOE_BF16) {
        bf16 *Wt = reinterpret_cast<bf16 *>(ws + L.wt);
        int32_t *counter = reinterpret_cast<int32_t *>(ws) + kWsRouterCounterWord;
        return launch_route_tc(p, x, Wg, Wnoise, noise, bias, idx, w, probs_sum, importance,
                               part, counter, Wt, status, s);
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
    return cudaGetLastError();
}

}  // namespace moe
