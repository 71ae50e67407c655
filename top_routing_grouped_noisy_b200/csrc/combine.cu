// combine.cu -- a5: gate-weighted combine and a6: gate statistics.
//
// a5 ("Llama 3 Meets MoE: Efficient Upcycling", section 3: y = sum_i G(x)_i E_i(x);
// "LLaMA-MoE v2", section "重新缩放机制与负载均衡": y = N/k sum_i G(x)_i E_i(x)):
//   y[t] = s * sum_{j<k, kept} G[t][j] * out[slot_row[t][j]]
// in the gather form (one writer per output element, slot order, f32 accumulate),
// so it needs no atomics and is bit-reproducible.  16-byte loads and stores.
//
// a6 ("LLaMA-MoE v2", section "门控机制设计": L_balance = lambda sum_i f_i P_i):
//   f[e] = counts[e] / (T k), P[e] = probs_sum[e] / T.
#include "common.cuh"
#include "kernels.h"

namespace moe {

// Each thread produces VPT adjacent 16-byte vectors of one token's output; all k
// slot rows of all of them are requested before any is used.
constexpr int kCombineVPT = 2;

// resid (may be NULL): a dense [T][d] term added after the scaled sum (the shared
// block of a residual MoE: y = s sum_j G_j out_j + resid).
template <typename E_T, int KMAX>
__global__ void __launch_bounds__(256) combine_kernel(const E_T *__restrict__ out,
                                                      const int32_t *__restrict__ slot_row,
                                                      const float *__restrict__ w, int T, int d,
                                                      int k, float scale, E_T *__restrict__ y,
                                                      const E_T *__restrict__ resid)
{
    pdl_wait();
    pdl_trigger();
    constexpr int VN = Vec<E_T>::N;
    constexpr int VPT = kCombineVPT;
    const int nv = d / VN;
    const int ng = (nv + VPT - 1) / VPT;  // vector groups per token
    const int64_t items = (int64_t)T * ng;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < items;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / ng;
        const int v0 = (int)(i - t * ng) * VPT;
        uint4 raw[KMAX][VPT];
        float g[KMAX];
        bool kept[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            const int32_t row = j < k ? slot_row[t * k + j] : -1;
            kept[j] = row >= 0;
            g[j] = kept[j] ? w[t * k + j] : 0.f;
#pragma unroll
            for (int u = 0; u < VPT; ++u)
                raw[j][u] = (kept[j] && v0 + u < nv)
                                ? ld_nc_na(out + (int64_t)row * d + (int64_t)(v0 + u) * VN)
                                : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < VPT; ++u) {
            if (v0 + u >= nv)
                break;
            float acc[VN];
#pragma unroll
            for (int q = 0; q < VN; ++q)
                acc[q] = 0.f;
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (!kept[j])
                    continue;
                float f[VN];
                if constexpr (sizeof(E_T) == 2) {
                    bf16x8_to_f32(raw[j][u], f);
                } else {
                    f[0] = __uint_as_float(raw[j][u].x);
                    f[1] = __uint_as_float(raw[j][u].y);
                    f[2] = __uint_as_float(raw[j][u].z);
                    f[3] = __uint_as_float(raw[j][u].w);
                }
#pragma unroll
                for (int q = 0; q < VN; ++q)
                    acc[q] = fmaf(g[j], f[q], acc[q]);
            }
#pragma unroll
            for (int q = 0; q < VN; ++q)
                acc[q] *= scale;
            if (resid != nullptr) {
                const uint4 rv = ld_nc_na(resid + t * d + (int64_t)(v0 + u) * VN);
                float rf[VN];
                if constexpr (sizeof(E_T) == 2) {
                    bf16x8_to_f32(rv, rf);
                } else {
                    rf[0] = __uint_as_float(rv.x);
                    rf[1] = __uint_as_float(rv.y);
                    rf[2] = __uint_as_float(rv.z);
                    rf[3] = __uint_as_float(rv.w);
                }
#pragma unroll
                for (int q = 0; q < VN; ++q)
                    acc[q] += rf[q];
            }
            uint4 o;
            if constexpr (sizeof(E_T) == 2) {
                o = f32x8_to_bf16(acc);
            } else {
                o = make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]),
                               __float_as_uint(acc[2]), __float_as_uint(acc[3]));
            }
            st_v4(y + t * d + (int64_t)(v0 + u) * VN, o);
        }
    }
}

__global__ void gate_stats_kernel(const int32_t *__restrict__ counts,
                                  const float *__restrict__ probs_sum, int T, int E, int k,
                                  float lambda, float *__restrict__ f, float *__restrict__ P,
                                  float *__restrict__ loss)
{
    pdl_wait();
    pdl_trigger();
    __shared__ double s_fp[MOE_MAX_EXPERTS];
    const int e = threadIdx.x;
    if (e < E) {
        const double fe = T > 0 ? (double)counts[e] / ((double)T * k) : 0.0;
        const double pe = T > 0 ? (double)probs_sum[e] / (double)T : 0.0;
        f[e] = (float)fe;
        P[e] = (float)pe;
        s_fp[e] = fe * pe;
    }
    __syncthreads();
    if (e == 0) {
        double s = 0.0;
        for (int i = 0; i < E; ++i)
            s += s_fp[i];
        loss[0] = (float)(lambda * s);
    }
}

cudaError_t launch_combine(const moe_params_t *p, const void *out, const int32_t *slot_row,
                           const float *w, void *y, cudaStream_t s, const void *resid)
{
    const float scale = p->rescale ? (float)p->E / (float)p->k : 1.0f;
    const int VN = p->dtype == MOE_BF16 ? 8 : 4;
    const int64_t items = (int64_t)p->T * ((p->d / VN + kCombineVPT - 1) / kCombineVPT);
    const int64_t blocks = (items + 255) / 256;
    const unsigned grid = (unsigned)(blocks < (1 << 30) ? blocks : (1 << 30));
#define MOE_COMBINE(KM)                                                                        \
    do {                                                                                       \
        if (p->dtype == MOE_BF16)                                                              \
            launch_pdl(combine_kernel<bf16, KM>, dim3(grid), dim3(256), 0, s, (const bf16 *)out, slot_row, w, p->T, \
                                                          p->d, p->k, scale, (bf16 *)y,        \
                       (const bf16 *)resid);                                                   \
        else                                                                                   \
            launch_pdl(combine_kernel<float, KM>, dim3(grid), dim3(256), 0, s, (const float *)out, slot_row, w,     \
                                                           p->T, p->d, p->k, scale, (float *)y, \
                       (const float *)resid);                                                  \
    } while (0)
    if (p->k <= 2)
        MOE_COMBINE(2);
    else if (p->k <= 4)
        MOE_COMBINE(4);
    else
        MOE_COMBINE(8);
#undef MOE_COMBINE
    count_launch();
    return cudaGetLastError();
}

__global__ void token_range_kernel(int32_t *offsets2, int T)
{
    pdl_wait();
    pdl_trigger();
    if (threadIdx.x == 0) {
        offsets2[0] = 0;
        offsets2[1] = T;
    }
}

cudaError_t launch_token_range(int32_t *offsets2, int T, cudaStream_t s)
{
    launch_pdl(token_range_kernel, dim3(1), dim3(32), 0, s, offsets2, T);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_gate_stats(const moe_params_t *p, const int32_t *counts,
                              const float *probs_sum, float *f, float *P, float *loss,
                              cudaStream_t s)
{
    launch_pdl(gate_stats_kernel, dim3(1), dim3(MOE_MAX_EXPERTS), 0, s, counts, probs_sum, p->T, p->E, p->k,
                                                    p->balance_lambda, f, P, loss);
    count_launch();
    return cudaGetLastError();
}

}  // namespace moe
