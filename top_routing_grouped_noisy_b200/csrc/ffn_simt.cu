// ffn_simt.cu -- a3/a4 for f32 layers on the CUDA cores (FFMA, no TF32, so the
// f32 layer keeps f32 accuracy).  SwiGLU expert ("LLaMA-MoE v2", code sample
// "代码实现示例", class Expert: down(silu(gate(x)) * up(x))).
//
// Grouped over experts without a host round trip: each CTA finds its (expert,
// 64-row tile) from the device-side offsets; CTAs past the last tile exit.
// Tiles: 64 rows x 32 neurons (64 packed W13 rows) for a3, 64 x 64 for a4;
// K slabs of 16 staged in shared memory; 4x(2+2) / 4x4 outputs per thread.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kSimtBM = 64;

// Finds the expert and row range of m-tile `tile` (over all experts in order).
__device__ __forceinline__ bool find_tile(const int32_t *offsets, int E, int tile, int BM,
                                          int &e_out, int &row0, int &row_end)
{
    for (int e = 0; e < E; ++e) {
        const int a = offsets[e], b = offsets[e + 1];
        const int nt = (b - a + BM - 1) / BM;
        if (tile < nt) {
            e_out = e;
            row0 = a + tile * BM;
            row_end = b;
            return true;
        }
        tile -= nt;
    }
    return false;
}

__global__ void __launch_bounds__(256) up_simt_kernel(const float *__restrict__ x_perm,
                                                      const int32_t *__restrict__ offsets,
                                                      const float *__restrict__ W13, int E,
                                                      int d, int m, float *__restrict__ h)
{
    pdl_wait();
    pdl_trigger();
    constexpr int BM = kSimtBM, BK = 16, BP = 64;  // BP packed rows = 32 neurons
    __shared__ float As[BK][BM + 4];
    __shared__ float Bs[BK][BP + 4];
    int e, row0, row_end;
    if (!find_tile(offsets, E, blockIdx.x, BM, e, row0, row_end))
        return;
    const int m16 = (m + 15) / 16 * 16, m8 = (m + 7) / 8 * 8;
    const int prow0 = blockIdx.y * BP;  // first packed row of this neuron tile
    const float *We = W13 + (int64_t)e * 2 * m16 * d;
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    float ag[4][2] = {}, au[4][2] = {};
    const int lr = tid / 4, lk = (tid % 4) * 4;
    for (int k0 = 0; k0 < d; k0 += BK) {
        float4 va = make_float4(0.f, 0.f, 0.f, 0.f), vb = va;
        if (row0 + lr < row_end && k0 + lk < d)
            va = *reinterpret_cast<const float4 *>(x_perm + (int64_t)(row0 + lr) * d + k0 + lk);
        if (prow0 + lr < 2 * m16 && k0 + lk < d)
            vb = *reinterpret_cast<const float4 *>(We + (int64_t)(prow0 + lr) * d + k0 + lk);
        As[lk + 0][lr] = va.x;
        As[lk + 1][lr] = va.y;
        As[lk + 2][lr] = va.z;
        As[lk + 3][lr] = va.w;
        Bs[lk + 0][lr] = vb.x;
        Bs[lk + 1][lr] = vb.y;
        Bs[lk + 2][lr] = vb.z;
        Bs[lk + 3][lr] = vb.w;
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float a[4], bg[2], bu[2];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                const int ln = tx * 2 + n;
                const int pr = (ln / 16) * 32 + (ln % 16);
                bg[n] = Bs[kk][pr];
                bu[n] = Bs[kk][pr + 16];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int n = 0; n < 2; ++n) {
                    ag[i][n] = fmaf(a[i], bg[n], ag[i][n]);
                    au[i][n] = fmaf(a[i], bu[n], au[i][n]);
                }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = row0 + ty * 4 + i;
        if (r >= row_end)
            continue;
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            const int neuron = blockIdx.y * 32 + tx * 2 + n;
            if (neuron < m) {
                const float g = ag[i][n];
                h[(int64_t)r * m8 + neuron] = g / (1.f + expf(-g)) * au[i][n];
            }
        }
    }
}

__global__ void __launch_bounds__(256) down_simt_kernel(const float *__restrict__ hbuf,
                                                        const int32_t *__restrict__ offsets,
                                                        const float *__restrict__ W2, int E,
                                                        int d, int m, float *__restrict__ out)
{
    pdl_wait();
    pdl_trigger();
    constexpr int BM = kSimtBM, BK = 16, BN = 64;
    __shared__ float As[BK][BM + 4];
    __shared__ float Bs[BK][BN + 4];
    int e, row0, row_end;
    if (!find_tile(offsets, E, blockIdx.x, BM, e, row0, row_end))
        return;
    const int m8 = (m + 7) / 8 * 8;
    const int n0 = blockIdx.y * BN;
    const float *We = W2 + (int64_t)e * d * m8;
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    float acc[4][4] = {};
    const int lr = tid / 4, lk = (tid % 4) * 4;
    for (int k0 = 0; k0 < m; k0 += BK) {
        float va[4] = {0.f, 0.f, 0.f, 0.f}, vb[4] = {0.f, 0.f, 0.f, 0.f};
        const int kc = k0 + lk;
        if (kc < m8) {
            if (row0 + lr < row_end) {
                const float4 t = *reinterpret_cast<const float4 *>(hbuf + (int64_t)(row0 + lr) * m8 + kc);
                va[0] = t.x; va[1] = t.y; va[2] = t.z; va[3] = t.w;
            }
            if (n0 + lr < d) {
                const float4 t = *reinterpret_cast<const float4 *>(We + (int64_t)(n0 + lr) * m8 + kc);
                vb[0] = t.x; vb[1] = t.y; vb[2] = t.z; vb[3] = t.w;
            }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const bool in = kc + q < m;  // h columns >= m are never written
            As[lk + q][lr] = in ? va[q] : 0.f;
            Bs[lk + q][lr] = in ? vb[q] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = As[kk][ty * 4 + i];
                b[i] = Bs[kk][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = row0 + ty * 4 + i;
        if (r >= row_end)
            continue;
        const int o = n0 + tx * 4;
        if (o + 3 < d) {
            *reinterpret_cast<float4 *>(out + (int64_t)r * d + o) =
                make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        } else {
            for (int j = 0; j < 4; ++j)
                if (o + j < d)
                    out[(int64_t)r * d + o + j] = acc[i][j];
        }
    }
}

static unsigned max_mtiles(const moe_params_t *p, int BM)
{
    // sum_e ceil(kept_e / BM) <= ceil(T*k / BM) + E
    return (unsigned)(ceil_div(p->T * p->k, BM) + p->E);
}

cudaError_t launch_up_simt(const moe_params_t *p, const float *x_perm, const int32_t *offsets,
                           const float *W13, float *h, cudaStream_t s)
{
    dim3 grid(max_mtiles(p, kSimtBM), ceil_div(p->m, 32));
    launch_pdl(up_simt_kernel, dim3(grid), dim3(256), 0, s, x_perm, offsets, W13, p->E, p->d, p->m, h);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_down_simt(const moe_params_t *p, const float *h, const int32_t *offsets,
                             const float *W2, float *out, cudaStream_t s)
{
    dim3 grid(max_mtiles(p, kSimtBM), ceil_div(p->d, 64));
    launch_pdl(down_simt_kernel, dim3(grid), dim3(256), 0, s, h, offsets, W2, p->E, p->d, p->m, out);
    count_launch();
    return cudaGetLastError();
}

}  // namespace moe
