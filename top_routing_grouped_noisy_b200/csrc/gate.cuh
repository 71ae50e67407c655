// gate.cuh -- the per-token gate of a1 and the split-K router body for batches
// of at most 64 tokens (device functions used by router.cu).
// "Llama 3 Meets MoE: Efficient Upcycling", section 3 "核心公式" (noisy Top-k
// routing, KeepTopK), section 5 (Mixtral vs ST router).
#pragma once

#include <math.h>

#include <type_traits>

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

// The gate of one token by one warp (lane e holds expert e; E <= 32), with
// finish_token's arithmetic: the same routing logits, the first maximum on ties, the
// softmax and the Mixtral renormalisation summed in expert / slot order.  l: the
// token's clean then noise logits; noise_row: its E noise draws.  Writes idx_out[0..k),
// w_out[0..k), prob[0..E) and gw[0..E) (zero where not selected).  Called by all 32
// lanes.  (The decode kernel's ds_gate has the same steps written out in its token
// loop: calling this function from there made its router phase ~6 us slower at 8
// tokens.)
__device__ __forceinline__ void gate_token_warp(const float *l, int E, int k, int noisy,
                                       const float *noise_row, const float *__restrict__ bias,
                                       int router_type, int32_t *__restrict__ idx_out,
                                       float *__restrict__ w_out, float *prob, float *gw,
                                       int32_t *status)
{
    const int lane = threadIdx.x & 31;
    const bool on = lane < E;
    float h = 0.f;
    if (on) {
        h = l[lane];
        if (bias)
            h += bias[lane];
        if (noisy)
            h += noise_row[lane] * softplus_f(l[E + lane]);
    }
    if (__any_sync(0xffffffffu, on && !isfinite(h))) {
        if (lane == 0)
            set_status(status, MOE_ERR_DEVICE_BADINDEX);
        if (lane < k) {
            idx_out[lane] = -1;
            w_out[lane] = 0.f;
        }
        if (on) {
            prob[lane] = 0.f;
            gw[lane] = 0.f;
        }
        return;
    }
    // (the loops over the k picks leave at k: a round of shuffles per pick is the
    // gate's longest chain)
    int sel[MOE_MAX_TOPK];
#pragma unroll
    for (int j = 0; j < MOE_MAX_TOPK; ++j)
        sel[j] = 0;
    bool taken = false;
#pragma unroll
    for (int j = 0; j < MOE_MAX_TOPK; ++j) {
        if (j >= k)
            break;
        float v = (on && !taken) ? h : -INFINITY;
        int vi = (on && !taken) ? lane : 0x7fffffff;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, v, off);
            const int oi = __shfl_xor_sync(0xffffffffu, vi, off);
            if (ov > v || (ov == v && oi < vi)) {
                v = ov;
                vi = oi;
            }
        }
        sel[j] = vi;
        taken |= lane == vi;
    }
    const float hmax = __shfl_sync(0xffffffffu, h, sel[0]);
    const float ex = on ? expf(h - hmax) : 0.f;
    float z = 0.f;
    for (int e = 0; e < E; ++e)
        z += __shfl_sync(0xffffffffu, ex, e);
    const float inv = 1.f / z;
    const float p = ex * inv;
    float wsel = 0.f;  // this lane's gate weight when it is a selected expert
    if (router_type == MOE_ROUTER_MIXTRAL) {
        float zs = 0.f;
#pragma unroll
        for (int j = 0; j < MOE_MAX_TOPK; ++j) {
            if (j >= k)
                break;
            zs += __shfl_sync(0xffffffffu, ex, sel[j]);
        }
        const float is = 1.f / zs;
        wsel = ex * is;
    } else {
        wsel = p;
    }
    if (on) {
        prob[lane] = p;
        gw[lane] = taken ? wsel : 0.f;
    }
#pragma unroll
    for (int j = 0; j < MOE_MAX_TOPK; ++j) {
        if (j >= k)
            break;
        const float wj = __shfl_sync(0xffffffffu, wsel, sel[j]);
        if (lane == j) {
            idx_out[j] = sel[j];
            w_out[j] = wj;
        }
    }
}

// bf16 slice ks on the tensor cores (mma.sync m16n8k16, f32 accumulation): the x
// columns [k0, k0 + kn) of every token and the same rows of [W_g | W_noise] (read in
// place) are staged as bf16 tiles, zero outside the slice and the T tokens (the 8
// extra elements per row spread the rows over the banks); warp w computes the 16 x 8
// output tiles w, w + 8, ..., each over the slice in ascending K, into
// part[ks][t][o].
__device__ inline void router_small_slice_mma(int ks, const bf16 *__restrict__ x,
                                              const bf16 *__restrict__ Wg,
                                              const bf16 *__restrict__ Wn, int T, int d, int E,
                                              float *__restrict__ part, void *sm)
{
    const int nout = Wn ? 2 * E : E;
    const int kc = router_small_kc(d);
    const int k0 = ks * kc, k1 = min(d, k0 + kc);
    const int kn = k1 > k0 ? k1 - k0 : 0;  // a multiple of 8 (d % 8 == 0)
    const int kp = round_up(kc, 16), xp = kp + 8, np = round_up(nout, 8), wp = np + 8;
    const int T16 = round_up(T, 16);
    bf16 *xs = static_cast<bf16 *>(sm);  // [T16][xp]
    bf16 *wsm = xs + (size_t)T16 * xp;  // [kp][wp]
    // x (16-byte vectors) and the weight rows k0 + r (W_g's E columns, then W_noise's;
    // zero padding written with them): each round has four x vectors and four weight
    // elements per thread in flight before any is stored
    const int vx = kp / 8, nvx = T16 * vx, nw = kp * np;
    for (int i0 = threadIdx.x; i0 < nvx || i0 < nw; i0 += 4 * blockDim.x) {
        uint4 u[4];
        bf16 wv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = i0 + j * blockDim.x, t = i / vx, v = i % vx;
            u[j] = make_uint4(0, 0, 0, 0);
            if (i < nvx && t < T && v * 8 < kn)
                u[j] = ld_nc(x + (int64_t)t * d + k0 + v * 8);
            const int r = i / np, o = i % np;
            wv[j] = __float2bfloat16_rn(0.f);
            if (i < nw && r < kn && o < nout)
                wv[j] = o < E ? Wg[(int64_t)(k0 + r) * E + o] : Wn[(int64_t)(k0 + r) * E + o - E];
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = i0 + j * blockDim.x;
            if (i < nvx)
                *reinterpret_cast<uint4 *>(xs + (size_t)(i / vx) * xp + (i % vx) * 8) = u[j];
            if (i < nw)
                wsm[(size_t)(i / np) * wp + i % np] = wv[j];
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const int ntn = np / 8, tiles = (T16 / 16) * ntn;
    const uint32_t xs_a = (uint32_t)__cvta_generic_to_shared(xs);
    const uint32_t ws_a = (uint32_t)__cvta_generic_to_shared(wsm);
    for (int tile = warp; tile < tiles; tile += (int)(blockDim.x >> 5)) {
        const int mt = tile / ntn, nt = tile % ntn;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int kk = 0; kk < kp; kk += 16) {
            uint32_t a0, a1, a2, a3, b0, b1;
            ldsm_x4(xs_a + (uint32_t)(((mt * 16 + (lane & 15)) * xp + kk + (lane >> 4) * 8) * 2),
                    a0, a1, a2, a3);
            ldsm_x2_trans(ws_a + (uint32_t)(((kk + (lane & 15)) * wp + nt * 8) * 2), b0, b1);
            mma_bf16_16816(acc, a0, a1, a2, a3, b0, b1);
        }
        const int t0 = mt * 16 + g, o0 = nt * 8 + 2 * c;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int t = t0 + (q >> 1) * 8, o = o0 + (q & 1);
            if (t < T && o < nout)
                part[((int64_t)ks * T + t) * nout + o] = acc[q];
        }
    }
}

// Split-K router for batches of at most 64 tokens, slice ks of kRouterSmallSplit:
// part[ks][t][o] receives the f32 dot product of token t's x and output o's weight
// column over the slice's columns of x.  bf16 runs on the tensor cores
// (router_small_slice_mma); f32 stages the columns of x and of [W_g | W_noise] (read in
// place) in shared memory `sm` ([T][kc] then [kc][nout] f32) and adds the products in
// ascending column order.
template <typename E_T>
__device__ inline void router_small_slice(int ks, const E_T *__restrict__ x,
                                          const E_T *__restrict__ Wg,
                                          const E_T *__restrict__ Wn, int T, int d, int E,
                                          float *__restrict__ part, float *sm)
{
    if constexpr (std::is_same<E_T, bf16>::value) {
        router_small_slice_mma(ks, x, Wg, Wn, T, d, E, part, sm);
        return;
    }
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
