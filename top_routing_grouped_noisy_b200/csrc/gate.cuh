// gate.cuh -- the per-token gate of a1 and the split-K router body for batches
// of at most 64 tokens (device functions used by router.cu).
// "Llama 3 Meets MoE: Efficient Upcycling", section 3 "核心公式" (noisy Top-k
// routing, KeepTopK), section 5 (Mixtral vs ST router).
#pragma once

#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

__device__ __forceinline__ float softplus_f(float z) { return fmaxf(z, 0.f) + log1pf(expf(-fabsf(z))); }

// Gate of one token from its clean logits lg[0..E) and noise logits lg[E..2E).
// Writes the token's k (index, weight) pairs, its full softmax prob[0..E) and its
// per-expert gate weight gw[0..E) (zero where not selected).  The routing logits
// H overwrite lg[0..E) (each lg[e], lg[E+e] is read before H[e] is written).
__device__ inline void finish_token(int64_t t, float *lg, int E, int k, int noisy,
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

// Split-K router for batches of at most 64 tokens, slice ks of kRouterSmallSplit:
// the slice's columns of x and of [W_g | W_noise] (read in place) are staged in
// shared memory `sm` ([T][kc] then [kc][nout] f32), and part[ks][t][o] receives
// the f32 dot product over the slice, columns in ascending order.
template <typename E_T>
__device__ inline void router_small_slice(int ks, const E_T *__restrict__ x,
                                          const E_T *__restrict__ Wg,
                                          const E_T *__restrict__ Wn, int T, int d, int E,
                                          float *__restrict__ part, float *sm)
{
    constexpr int VN = 16 / sizeof(E_T);  // elements per 16-byte load
    const int nout = Wn ? 2 * E : E;
    const int kc = router_small_kc(d);
    const int k0 = ks * kc, k1 = min(d, k0 + kc);
    const int kn = k1 > k0 ? k1 - k0 : 0;  // a multiple of 8 (d % 8 == 0)
    float *xs = sm;                    // [T][kc]
    float *ws_ = sm + (size_t)T * kc;  // [kc][nout]
    // x slice: 16-byte loads, four in flight per thread before any is stored
    const int nvx = kn / VN;
    for (int i0 = threadIdx.x; i0 < T * nvx; i0 += 4 * blockDim.x) {
        uint4 u[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = i0 + j * blockDim.x;
            u[j] = make_uint4(0, 0, 0, 0);
            if (i < T * nvx)
                u[j] = ld_nc(x + (int64_t)(i / nvx) * d + k0 + (i % nvx) * VN);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = i0 + j * blockDim.x;
            if (i < T * nvx) {
                const E_T *v = reinterpret_cast<const E_T *>(&u[j]);
                float *dst = xs + (size_t)(i / nvx) * kc + (i % nvx) * VN;
#pragma unroll
                for (int q = 0; q < VN; ++q)
                    dst[q] = to_f32(v[q]);
            }
        }
    }
    // rows k0..k1 of W_g (and W_noise) are contiguous: kn * E elements from k0 * E
    const int nvw = kn * E / VN;  // kn % 8 == 0, so kn * E % VN == 0
    for (int h = 0; h < (Wn ? 2 : 1); ++h) {
        const E_T *W = h == 0 ? Wg : Wn;
        for (int i0 = threadIdx.x; i0 < nvw; i0 += 4 * blockDim.x) {
            uint4 u[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = i0 + j * blockDim.x;
                u[j] = i < nvw ? ld_nc(W + (int64_t)k0 * E + (int64_t)i * VN)
                               : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = i0 + j * blockDim.x;
                if (i < nvw) {
                    const E_T *v = reinterpret_cast<const E_T *>(&u[j]);
#pragma unroll
                    for (int q = 0; q < VN; ++q) {
                        const int f = i * VN + q;  // flat index in the slice: (c, o)
                        ws_[(f / E) * nout + h * E + f % E] = to_f32(v[q]);
                    }
                }
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < T * nout; i += blockDim.x) {
        const int t = i / nout, o = i % nout;
        float acc = 0.f;
        for (int c = 0; c < kn; ++c)
            acc = fmaf(xs[t * kc + c], ws_[c * nout + o], acc);
        part[((int64_t)ks * T + t) * nout + o] = acc;
    }
}

// The gate of every token from its logits lg [T][nout] (shared memory, f32) and the
// token sums (probs_sum, importance) in token order.  Shared memory `sm`: [T][E]
// probabilities, then [T][E] gate weights.
__device__ inline void router_gate_tokens(float *lg, int T, int E, int k, int noisy,
                                          const float *__restrict__ noise,
                                          const float *__restrict__ bias, int router_type,
                                          int32_t *__restrict__ idx_out, float *__restrict__ w_out,
                                          float *__restrict__ probs_sum,
                                          float *__restrict__ importance, int32_t *status,
                                          float *sm)
{
    const int nout = noisy ? 2 * E : E;
    float *prob_s = sm;                      // [T][E]
    float *gw_s = prob_s + (size_t)T * E;    // [T][E]
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

// One CTA finishes the split-K router: adds the slices in order, runs the gate of
// every token and the token sums (probs_sum, importance) in token order.  Shared
// memory `sm`: [T][nout] logits, then the gate's [T][E] probabilities and weights.
__device__ inline void router_small_finish(const float *__restrict__ part, int T, int E, int k,
                                           int noisy, const float *__restrict__ noise,
                                           const float *__restrict__ bias, int router_type,
                                           int32_t *__restrict__ idx_out,
                                           float *__restrict__ w_out,
                                           float *__restrict__ probs_sum,
                                           float *__restrict__ importance, int32_t *status,
                                           float *sm)
{
    const int nout = noisy ? 2 * E : E;
    float *lg = sm;  // [T][nout]
    for (int i = threadIdx.x; i < T * nout; i += blockDim.x) {
        float v[kRouterSmallSplit];  // all slices requested before they are added in order
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
    router_gate_tokens(lg, T, E, k, noisy, noise, bias, router_type, idx_out, w_out, probs_sum,
                       importance, status, lg + (size_t)T * nout);
}

}  // namespace moe
