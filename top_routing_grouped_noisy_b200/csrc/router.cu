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
    pdl_wait();
    pdl_trigger();
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
    pdl_wait();
    pdl_trigger();
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
