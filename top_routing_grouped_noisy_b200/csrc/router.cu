// router.cu -- a1: noisy Top-K gate ("Llama 3 Meets MoE: Efficient Upcycling",
// section 3 "核心公式", Noisy Top-k routing; section 5, Mixtral vs ST router).
//
//   L_t = x_t W_g (+ b),  H_t = L_t + eps_t * Softplus(x_t W_noise)
//   idx_t = KeepTopK(H_t, k)   (ties -> lower expert index; slot j = j-th largest)
//   Mixtral: G_tj = softmax over the k kept H;  ST: G_tj = softmax(H_t)[idx_tj]
// plus per-CTA partial sums of softmax(H_t) (for P) and of G (importance).
//
// bf16 path: the logits x.[W_g | W_noise] are a skinny GEMM (T x d x 2E) read
// at HBM speed; it runs on the tensor cores with mma.sync m16n8k16 (bf16 in,
// f32 accumulate), the router weights as the M=16 operand and 8 tokens as N.
// The K dimension is split over the 8 warps of a CTA and reduced through shared
// memory in a fixed order (bit-deterministic).  x is streamed once with 16-byte
// non-allocating loads.  f32 path: one warp per token on the CUDA cores.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

// Tile constants (compile-time; tuned on B200).
#ifndef MOE_ROUTER_NNT1
#define MOE_ROUTER_NNT1 8  // token n-tiles per CTA when the router has <= 16 outputs
#endif
#ifndef MOE_ROUTER_U
#define MOE_ROUTER_U 4  // k32 blocks of loads issued per round
#endif
#ifndef MOE_ROUTER_U_WIDE
#define MOE_ROUTER_U_WIDE 1  // the same for 8 token n-tiles per CTA
#endif

namespace moe {


__device__ __forceinline__ float softplus_f(float z) { return fmaxf(z, 0.f) + log1pf(expf(-fabsf(z))); }

// Gate of one token from its clean logits lg[0..E) and noise logits lg[E..2E).
// Writes the token's k (index, weight) pairs, its full softmax prob[0..E) and its
// per-expert gate weight gw[0..E) (zero where not selected).  The routing logits
// H overwrite lg[0..E) (each lg[e], lg[E+e] is read before H[e] is written).
__device__ void finish_token(int64_t t, float *lg, int E, int k, int noisy,
                             const float *__restrict__ noise, const float *__restrict__ bias,
                             int router_type, int32_t *__restrict__ idx_out,
                             float *__restrict__ w_out, float *prob, float *gw, int32_t *status)
{
    float *H = lg;
    bool bad = false;
    for (int e = 0; e < E; ++e) {
        float h = lg[e];
        if (bias)
            h += bias[e];
        if (noisy)
            h += noise[t * E + e] * softplus_f(lg[E + e]);
        bad |= !isfinite(h);
        H[e] = h;
        gw[e] = 0.f;
    }
    if (bad) {
        set_status(status, MOE_ERR_DEVICE_BADINDEX);
        for (int j = 0; j < k; ++j) {
            idx_out[t * k + j] = -1;
            w_out[t * k + j] = 0.f;
        }
        for (int e = 0; e < E; ++e)
            prob[e] = 0.f;
        return;
    }
    int sel[MOE_MAX_TOPK];
    uint64_t taken = 0;
    for (int j = 0; j < k; ++j) {
        int bi = -1;
        float best = 0.f;
        for (int e = 0; e < E; ++e) {
            if ((taken >> e) & 1ull)
                continue;
            if (bi < 0 || H[e] > best) {
                best = H[e];
                bi = e;
            }
        }
        taken |= 1ull << bi;
        sel[j] = bi;
    }
    const float hmax = H[sel[0]];
    float z = 0.f;
    for (int e = 0; e < E; ++e)
        z += expf(H[e] - hmax);
    const float inv = 1.f / z;
    for (int e = 0; e < E; ++e)
        prob[e] = expf(H[e] - hmax) * inv;
    if (router_type == MOE_ROUTER_MIXTRAL) {
        float zs = 0.f;
        for (int j = 0; j < k; ++j)
            zs += expf(H[sel[j]] - hmax);
        const float is = 1.f / zs;
        for (int j = 0; j < k; ++j) {
            const float w = expf(H[sel[j]] - hmax) * is;
            idx_out[t * k + j] = sel[j];
            w_out[t * k + j] = w;
            gw[sel[j]] = w;
        }
    } else {
        for (int j = 0; j < k; ++j) {
            const float w = prob[sel[j]];
            idx_out[t * k + j] = sel[j];
            w_out[t * k + j] = w;
            gw[sel[j]] = w;
        }
    }
}

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

// Wt[o][c]: o < E -> W_g[c][o]; E <= o < 2E -> W_noise[c][o-E] (if given); else 0.
__global__ void router_transpose_kernel(const bf16 *__restrict__ Wg, const bf16 *__restrict__ Wn,
                                        int d, int E, int rows, bf16 *__restrict__ Wt)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)rows * d)
        return;
    const int o = (int)(i / d), c = (int)(i % d);
    bf16 v = __float2bfloat16_rn(0.f);
    if (o < E)
        v = Wg[(int64_t)c * E + o];
    else if (Wn != nullptr && o < 2 * E)
        v = Wn[(int64_t)c * E + (o - E)];
    Wt[i] = v;
}

// NMT m-tiles of 16 router outputs x NNT n-tiles of 8 tokens per CTA.
// Each thread (g = lane/4, q = lane%4) owns K columns [32kb + 8q, 32kb + 8q + 8) of
// every k32 block kb it visits; the 8 columns feed two m16n8k16 steps, physical
// columns 8q+{0,1},{2,3} as logical k {2q,2q+1},{2q+8,2q+9} of the first step and
// 8q+{4,5},{6,7} of the second.  A and B use the same map, so the dot product is
// unchanged.
template <int NMT, int NNT>
__global__ void __launch_bounds__(256) router_bf16_kernel(
    const bf16 *__restrict__ x, const bf16 *__restrict__ Wt, int T, int d, int E, int k,
    int noisy, const float *__restrict__ noise, const float *__restrict__ bias, int router_type,
    int32_t *__restrict__ idx_out, float *__restrict__ w_out, float *__restrict__ part,
    int32_t *status)
{
    constexpr int TOK = NNT * 8, NOUT = NMT * 16, NW = kRouterWarps;
    extern __shared__ float smem[];
    float *red = smem;                          // [NW][NOUT][TOK]
    float *lg = red + NW * NOUT * TOK;          // [TOK][NOUT + 1]
    float *prob_s = lg + TOK * (NOUT + 1);      // [TOK][E]
    float *gw_s = prob_s + TOK * E;             // [TOK][E]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const int64_t tok0 = (int64_t)blockIdx.x * TOK;

    float acc[NMT][NNT][4];
#pragma unroll
    for (int a = 0; a < NMT; ++a)
#pragma unroll
        for (int b = 0; b < NNT; ++b)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                acc[a][b][c] = 0.f;

    const int nkb = (d + 31) / 32;
    // U k32 blocks per round: all loads of a round are issued before its MMAs
    constexpr int U = NNT >= 8 ? MOE_ROUTER_U_WIDE : MOE_ROUTER_U;
    for (int kb0 = warp; kb0 < nkb; kb0 += NW * U) {
        uint4 xb[U][NNT];
        uint4 wa[U][NMT][2];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = (kb0 + u * NW) * 32 + 8 * q;
            const bool kv = c < d;
#pragma unroll
            for (int nt = 0; nt < NNT; ++nt) {
                const int64_t t = tok0 + nt * 8 + g;
                xb[u][nt] = (kv && t < T) ? ld_nc_na(x + t * d + c) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int mt = 0; mt < NMT; ++mt) {
                wa[u][mt][0] = kv ? ld_nc(Wt + (int64_t)(mt * 16 + g) * d + c)
                                  : make_uint4(0, 0, 0, 0);
                wa[u][mt][1] = kv ? ld_nc(Wt + (int64_t)(mt * 16 + g + 8) * d + c)
                                  : make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NNT; ++nt) {
                    mma_bf16_16816(acc[mt][nt], wa[u][mt][0].x, wa[u][mt][1].x, wa[u][mt][0].y,
                                   wa[u][mt][1].y, xb[u][nt].x, xb[u][nt].y);
                    mma_bf16_16816(acc[mt][nt], wa[u][mt][0].z, wa[u][mt][1].z, wa[u][mt][0].w,
                                   wa[u][mt][1].w, xb[u][nt].z, xb[u][nt].w);
                }
    }
    // D fragment: c0,c1 -> (row g, cols 2q,2q+1); c2,c3 -> (row g+8, cols 2q,2q+1)
#pragma unroll
    for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NNT; ++nt) {
            const int o0 = mt * 16 + g, t0 = nt * 8 + 2 * q;
            red[(warp * NOUT + o0) * TOK + t0] = acc[mt][nt][0];
            red[(warp * NOUT + o0) * TOK + t0 + 1] = acc[mt][nt][1];
            red[(warp * NOUT + o0 + 8) * TOK + t0] = acc[mt][nt][2];
            red[(warp * NOUT + o0 + 8) * TOK + t0 + 1] = acc[mt][nt][3];
        }
    __syncthreads();
    for (int i = threadIdx.x; i < NOUT * TOK; i += blockDim.x) {
        const int o = i / TOK, tk = i % TOK;
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w)
            s += red[(w * NOUT + o) * TOK + tk];
        lg[tk * (NOUT + 1) + o] = s;
    }
    __syncthreads();
    const int ntok = (int)((int64_t)T - tok0 < TOK ? (int64_t)T - tok0 : TOK);
    if (threadIdx.x < ntok) {
        const int tk = threadIdx.x;
        finish_token(tok0 + tk, lg + tk * (NOUT + 1), E, k, noisy, noise, bias, router_type,
                     idx_out, w_out, prob_s + tk * E, gw_s + tk * E, status);
    }
    __syncthreads();
    write_partials(ntok, E, prob_s, gw_s, part);
}

// f32 router on the CUDA cores: one warp per token, 8 tokens per CTA.
__global__ void __launch_bounds__(256) router_f32_kernel(
    const float *__restrict__ x, const float *__restrict__ Wg, const float *__restrict__ Wn,
    int T, int d, int E, int k, const float *__restrict__ noise, const float *__restrict__ bias,
    int router_type, int32_t *__restrict__ idx_out, float *__restrict__ w_out,
    float *__restrict__ part, int32_t *status)
{
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
// busy, so K is split over kSmallKSplit CTAs instead.  Each CTA stages its K slice
// of x and of [W_g | W_noise] (read in place, no transpose) in shared memory and
// writes partial logits part[ks][t][o]; one finishing CTA adds the slices in a
// fixed order, runs the per-token gate and the token sums.
constexpr int kSmallKSplit = kRouterSmallSplit;

template <typename E_T>
__global__ void __launch_bounds__(256) router_small_partial_kernel(
    const E_T *__restrict__ x, const E_T *__restrict__ Wg, const E_T *__restrict__ Wn, int T,
    int d, int E, float *__restrict__ part)
{
    extern __shared__ float sm[];
    const int nout = Wn ? 2 * E : E;
    const int kc = (d + kSmallKSplit - 1) / kSmallKSplit;
    const int k0 = blockIdx.x * kc, k1 = min(d, k0 + kc);
    const int kn = k1 > k0 ? k1 - k0 : 0;
    float *xs = sm;                    // [T][kc]
    float *ws_ = sm + (size_t)T * kc;  // [kc][nout]
    for (int i = threadIdx.x; i < T * kn; i += blockDim.x) {
        const int t = i / kn, c = i % kn;
        xs[t * kc + c] = to_f32(x[(int64_t)t * d + k0 + c]);
    }
    for (int i = threadIdx.x; i < kn * nout; i += blockDim.x) {
        const int c = i / nout, o = i % nout;
        ws_[c * nout + o] = o < E ? to_f32(Wg[(int64_t)(k0 + c) * E + o])
                                  : to_f32(Wn[(int64_t)(k0 + c) * E + o - E]);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < T * nout; i += blockDim.x) {
        const int t = i / nout, o = i % nout;
        float acc = 0.f;
        for (int c = 0; c < kn; ++c)
            acc = fmaf(xs[t * kc + c], ws_[c * nout + o], acc);
        part[((int64_t)blockIdx.x * T + t) * nout + o] = acc;
    }
}

__global__ void __launch_bounds__(256) router_small_finish_kernel(
    const float *__restrict__ part, int T, int E, int k, int noisy,
    const float *__restrict__ noise, const float *__restrict__ bias, int router_type,
    int32_t *__restrict__ idx_out, float *__restrict__ w_out, float *__restrict__ probs_sum,
    float *__restrict__ importance, int32_t *status)
{
    extern __shared__ float sm[];
    const int nout = noisy ? 2 * E : E;
    float *lg = sm;                          // [T][nout]
    float *prob_s = lg + (size_t)T * nout;   // [T][E]
    float *gw_s = prob_s + (size_t)T * E;    // [T][E]
    for (int i = threadIdx.x; i < T * nout; i += blockDim.x) {
        float acc = 0.f;
        for (int ks = 0; ks < kSmallKSplit; ++ks)
            acc += part[(int64_t)ks * T * nout + i];
        lg[i] = acc;
    }
    __syncthreads();
    for (int t = threadIdx.x; t < T; t += blockDim.x)
        finish_token(t, lg + (size_t)t * nout, E, k, noisy, noise, bias, router_type, idx_out,
                     w_out, prob_s + (size_t)t * E, gw_s + (size_t)t * E, status);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float sp = 0.f, sg = 0.f;
        for (int t = 0; t < T; ++t) {
            sp += prob_s[t * E + e];
            sg += gw_s[t * E + e];
        }
        probs_sum[e] = sp;
        importance[e] = sg;
    }
}

template <int NMT, int NNT>
static cudaError_t run_bf16(const moe_params_t *p, const bf16 *x, const bf16 *Wt, int noisy,
                            const float *noise, const float *bias, int32_t *idx, float *w,
                            float *part, int32_t *status, cudaStream_t s, int *nblk)
{
    constexpr int TOK = NNT * 8, NOUT = NMT * 16;
    const size_t smem =
        sizeof(float) * ((size_t)kRouterWarps * NOUT * TOK + TOK * (NOUT + 1) + 2 * TOK * p->E);
    // E <= min(64, 16 * NMT) for this instantiation
    static_assert(sizeof(float) * (kRouterWarps * NOUT * TOK + TOK * (NOUT + 1) +
                                   2 * TOK * (16 * NMT < MOE_MAX_EXPERTS ? 16 * NMT
                                                                         : MOE_MAX_EXPERTS)) <=
                      48 * 1024,
                  "router shared memory must fit the default 48 KB");
    *nblk = ceil_div(p->T, TOK);
    router_bf16_kernel<NMT, NNT><<<*nblk, 256, smem, s>>>(
        x, Wt, p->T, p->d, p->E, p->k, noisy, noise, bias, p->router_type, idx, w, part, status);
    return cudaGetLastError();
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
    const int small_kc = ceil_div(p->d, kSmallKSplit);
    const size_t sm1 = sizeof(float) * ((size_t)p->T * small_kc + (size_t)small_kc * small_nout);
    const size_t sm2 =
        sizeof(float) * ((size_t)p->T * small_nout + 2 * (size_t)p->T * p->E);
    if (p->T > 0 && p->T <= kRouterSmallTokens && sm1 <= 48 * 1024 && sm2 <= 48 * 1024) {
        const int noisy = small_noisy;
        float *sp = reinterpret_cast<float *>(ws + L.rsmall);
        if (p->dtype == MOE_BF16)
            router_small_partial_kernel<bf16><<<kSmallKSplit, 256, sm1, s>>>(
                (const bf16 *)x, (const bf16 *)Wg, (const bf16 *)Wnoise, p->T, p->d, p->E, sp);
        else
            router_small_partial_kernel<float><<<kSmallKSplit, 256, sm1, s>>>(
                (const float *)x, (const float *)Wg, (const float *)Wnoise, p->T, p->d, p->E, sp);
        count_launch();
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
        router_small_finish_kernel<<<1, 256, sm2, s>>>(sp, p->T, p->E, p->k, noisy, noise, bias,
                                                       p->router_type, idx, w, probs_sum,
                                                       importance, status);
        count_launch();
        return cudaGetLastError();
    }
    if (p->T > 0) {
        if (p->dtype == MOE_BF16) {
            const int noisy = Wnoise != nullptr;
            const int nout = noisy ? 2 * p->E : p->E;
            bf16 *Wt = reinterpret_cast<bf16 *>(ws + L.wt);
            const int64_t n = (int64_t)kWtRows * p->d;
            router_transpose_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
                (const bf16 *)Wg, (const bf16 *)Wnoise, p->d, p->E, kWtRows, Wt);
            count_launch();
            if ((e = cudaGetLastError()) != cudaSuccess)
                return e;
            if (nout <= 16)
                e = run_bf16<1, MOE_ROUTER_NNT1>(p, (const bf16 *)x, Wt, noisy, noise, bias, idx, w, part,
                                   status, s, &nblk);
            else if (nout <= 32)
                e = run_bf16<2, 4>(p, (const bf16 *)x, Wt, noisy, noise, bias, idx, w, part,
                                   status, s, &nblk);
            else if (nout <= 64)
                e = run_bf16<4, 2>(p, (const bf16 *)x, Wt, noisy, noise, bias, idx, w, part,
                                   status, s, &nblk);
            else
                e = run_bf16<8, 1>(p, (const bf16 *)x, Wt, noisy, noise, bias, idx, w, part,
                                   status, s, &nblk);
        } else {
            nblk = ceil_div(p->T, kRouterWarps);
            const size_t smem = sizeof(float) * ((size_t)kRouterWarps * 4 * p->E);
            router_f32_kernel<<<nblk, 256, smem, s>>>(
                (const float *)x, (const float *)Wg, (const float *)Wnoise, p->T, p->d, p->E,
                p->k, noise, bias, p->router_type, idx, w, part, status);
            e = cudaGetLastError();
        }
        count_launch();
        if (e != cudaSuccess)
            return e;
    }
    router_finalize_kernel<<<1, 1024, 0, s>>>(part, nblk, p->E, probs_sum, importance);
    count_launch();
    return cudaGetLastError();
}

}  // namespace moe
