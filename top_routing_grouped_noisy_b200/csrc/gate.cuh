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

// ------------------------------------------------------------------ one-CTA router
// Logits of at most 16 tokens and NT * 8 >= nout outputs on the tensor cores, in one
// CTA of kOneWarps warps: warp w takes K columns [w kw, (w+1) kw) (kw = d / kOneWarps
// rounded up to 16), staged 64 at a time in its own shared memory (x rows padded by 16
// bytes, so the 32-bit fragment reads are free of bank conflicts; the router rows
// copied as they lie in W_g / W_noise, which are contiguous for a run of K), and
// accumulates mma.sync m16n8k16 fragments (bf16 in, f32); the warps' partial logits are
// then added in warp order.  Output lg [T][nout] f32 in shared memory.  The result is
// one fixed function of the inputs, whichever kernel calls it.
constexpr int kOneWarps = 16;
constexpr int kOneKC = 64;
constexpr int kOneXPitch = kOneKC + 8;  // bf16 per staged x row
__host__ __device__ constexpr size_t one_cta_warp_smem(int nt)
{
    // x [16][kOneXPitch] bf16, then the W_g rows [kOneKC][E] and the W_noise rows
    // [kOneKC][E] (2E <= 8 nt with noise, E <= 8 nt without)
    return (size_t)16 * kOneXPitch * 2 + (size_t)kOneKC * 8 * nt * 2;
}
__host__ __device__ constexpr size_t one_cta_logits_smem(int nt)
{
    return kOneWarps * one_cta_warp_smem(nt) + (size_t)kOneWarps * 16 * nt * 8 * 4;
}

__device__ __forceinline__ uint32_t bf16_pair(const uint16_t *p0, const uint16_t *p1)
{
    return (uint32_t)*p0 | ((uint32_t)*p1 << 16);
}

template <int NT>
__device__ inline void router_logits_one_cta(const bf16 *__restrict__ x, const bf16 *__restrict__ Wg,
                                             const bf16 *__restrict__ Wn, int T, int d, int E,
                                             float *lg, char *smem)
{
    const int nout = Wn ? 2 * E : E;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int kw = (d + kOneWarps * 16 - 1) / (kOneWarps * 16) * 16;
    const int kbeg = warp * kw, kend = min(d, kbeg + kw);
    char *wb = smem + (size_t)warp * one_cta_warp_smem(NT);
    uint16_t *xs = reinterpret_cast<uint16_t *>(wb);
    uint16_t *gs = xs + 16 * kOneXPitch;  // [kOneKC][E]
    uint16_t *ns = gs + kOneKC * E;        // [kOneKC][E] (noise rows)
    float *red = reinterpret_cast<float *>(smem + (size_t)kOneWarps * one_cta_warp_smem(NT));
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c)
            acc[nt][c] = 0.f;
    for (int k0 = kbeg; k0 < kend; k0 += kOneKC) {
        const int kc = min(kOneKC, kend - k0);  // a multiple of 8
        __syncwarp();
        for (int i = lane; i < 16 * (kOneKC / 8); i += 32) {
            const int t = i / (kOneKC / 8), v = i % (kOneKC / 8);
            uint4 val = make_uint4(0, 0, 0, 0);
            if (t < T && v * 8 < kc)
                val = ld_nc(x + (int64_t)t * d + k0 + v * 8);
            *reinterpret_cast<uint4 *>(xs + t * kOneXPitch + v * 8) = val;
        }
        const int wv = kc * E / 8;  // 16-byte vectors of a run of router rows
        for (int i = lane; i < wv; i += 32) {
            reinterpret_cast<uint4 *>(gs)[i] = ld_nc(Wg + (int64_t)k0 * E + (int64_t)i * 8);
            if (Wn != nullptr)
                reinterpret_cast<uint4 *>(ns)[i] = ld_nc(Wn + (int64_t)k0 * E + (int64_t)i * 8);
        }
        __syncwarp();
        for (int kk = 0; kk < kc; kk += 16) {
            // rows past kc read as zero (kc is a multiple of 8: the upper half may be out)
            const bool hi = kk + 8 < kc;
            const uint16_t *xr0 = xs + g * kOneXPitch + kk + 2 * q;
            const uint16_t *xr1 = xs + (g + 8) * kOneXPitch + kk + 2 * q;
            const uint32_t a0 = *reinterpret_cast<const uint32_t *>(xr0);
            const uint32_t a1 = *reinterpret_cast<const uint32_t *>(xr1);
            const uint32_t a2 = hi ? *reinterpret_cast<const uint32_t *>(xr0 + 8) : 0u;
            const uint32_t a3 = hi ? *reinterpret_cast<const uint32_t *>(xr1 + 8) : 0u;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int n = nt * 8 + g;
                const uint16_t *src = n < E ? gs + n : (n < nout ? ns + (n - E) : nullptr);
                const int r = kk + 2 * q;
                uint32_t b0 = 0u, b1 = 0u;
                if (src != nullptr) {
                    b0 = bf16_pair(src + r * E, src + (r + 1) * E);
                    if (hi)
                        b1 = bf16_pair(src + (r + 8) * E, src + (r + 9) * E);
                }
                mma_bf16_16816(acc[nt], a0, a1, a2, a3, b0, b1);
            }
        }
    }
    // this warp's partial logits, then the sum over warps in warp order
    constexpr int NP = NT * 8;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        float *rw = red + (size_t)warp * 16 * NP;
        const int n = nt * 8 + 2 * q;
        rw[g * NP + n] = acc[nt][0];
        rw[g * NP + n + 1] = acc[nt][1];
        rw[(g + 8) * NP + n] = acc[nt][2];
        rw[(g + 8) * NP + n + 1] = acc[nt][3];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < T * nout; i += blockDim.x) {
        const int t = i / nout, o = i % nout;
        float sum = 0.f;
        for (int w = 0; w < kOneWarps; ++w)
            sum += red[((size_t)w * 16 + t) * NP + o];
        lg[i] = sum;
    }
    __syncthreads();
}

}  // namespace moe
