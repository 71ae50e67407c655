// partition.cu -- a0: expert construction from a dense SwiGLU FFN
// ("LLaMA-MoE v2", section "专家构建方法": the intermediate neurons are split
// into E equal disjoint subsets, each subset one expert; "Llama 3 Meets MoE:
// Efficient Upcycling", section 2: every expert a copy of the FFN).
//
// Writes the packed layout the tensor-core expert GEMMs read:
//   W13_e [E][2*m16][d]: 32-row groups, rows 0..15 W1 (gate) of 16 neurons,
//                        rows 16..31 W3 (up) of the same neurons; zero rows for
//                        neurons >= m.
//   W2_e  [E][d][m8]:    W2 columns of the expert's neurons, zero-padded.
// A pure gather; off the per-batch path (once per weight set).
#include "common.cuh"
#include "kernels.h"

namespace moe {

// One CTA per packed W13 row; 16-byte copies along d.
template <typename E_T>
__global__ void __launch_bounds__(128) partition_w13_kernel(
    const E_T *__restrict__ W1, const E_T *__restrict__ W3, int d, int d_ff, int E, int m,
    int m16, int mode, const int32_t *__restrict__ perm, E_T *__restrict__ W13,
    int32_t *status)
{
    pdl_wait();
    pdl_trigger();
    const int64_t row = blockIdx.x;
    const int e = (int)(row / (2 * m16));
    const int r = (int)(row % (2 * m16));
    const int neuron = (r / 32) * 16 + (r & 15);
    const bool up = (r & 31) >= 16;
    const E_T *src = nullptr;
    if (neuron < m) {
        const E_T *base = up ? W3 : W1;
        if (mode == MOE_PARTITION_DISJOINT) {
            const int pidx = perm[(int64_t)e * m + neuron];
            if (pidx >= 0 && pidx < d_ff)
                src = base + (int64_t)pidx * d;
            else if (threadIdx.x == 0)
                set_status(status, MOE_ERR_DEVICE_BADINDEX);
        } else if (mode == MOE_PARTITION_COPY) {
            src = base + (int64_t)neuron * d;
        } else {
            src = base + ((int64_t)e * m + neuron) * d;
        }
    }
    constexpr int VN = 16 / sizeof(E_T);
    uint4 *dst = reinterpret_cast<uint4 *>(W13 + row * d);
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
    const int nv = d / VN;
    for (int v = threadIdx.x; v < nv; v += blockDim.x)
        dst[v] = src ? ld_nc_na(s4 + v) : make_uint4(0, 0, 0, 0);
}

// One CTA per (expert, output row o) of W2_e; element gather along the expert's columns.
template <typename E_T>
__global__ void __launch_bounds__(256) partition_w2_kernel(
    const E_T *__restrict__ W2, int d, int d_ff, int E, int m, int m8, int mode,
    const int32_t *__restrict__ perm, E_T *__restrict__ W2e, int32_t *status)
{
    pdl_wait();
    pdl_trigger();
    const int64_t row = blockIdx.x;  // e * d + o
    const int e = (int)(row / d);
    const int o = (int)(row % d);
    E_T *dst = W2e + row * m8;
    for (int i = threadIdx.x; i < m8; i += blockDim.x) {
        E_T v = E_T(0.0f);
        if (i < m) {
            if (mode == MOE_PARTITION_DISJOINT) {
                const int col = perm[(int64_t)e * m + i];
                if (col >= 0 && col < d_ff)
                    v = W2[(int64_t)o * d_ff + col];
                else
                    set_status(status, MOE_ERR_DEVICE_BADINDEX);
            } else if (mode == MOE_PARTITION_COPY) {
                v = W2[(int64_t)o * d_ff + i];
            } else {
                v = W2[((int64_t)e * d + o) * m + i];
            }
        }
        dst[i] = v;
    }
}

cudaError_t launch_partition(const void *W1, const void *W3, const void *W2, int d, int d_ff,
                             int E, int m, int mode, const int32_t *perm, int dtype,
                             void *W13_e, void *W2_e, int32_t *status, cudaStream_t s)
{
    const int m16 = round_up(m, 16), m8 = round_up(m, 8);
    const unsigned g13 = (unsigned)((int64_t)E * 2 * m16);
    const unsigned g2 = (unsigned)((int64_t)E * d);
    if (dtype == MOE_BF16) {
        launch_pdl(partition_w13_kernel<bf16>, dim3(g13), dim3(128), 0, s, 
            (const bf16 *)W1, (const bf16 *)W3, d, d_ff, E, m, m16, mode, perm, (bf16 *)W13_e,
            status);
        launch_pdl(partition_w2_kernel<bf16>, dim3(g2), dim3(256), 0, s, (const bf16 *)W2, d, d_ff, E, m, m8, mode,
                                                     perm, (bf16 *)W2_e, status);
    } else {
        launch_pdl(partition_w13_kernel<float>, dim3(g13), dim3(128), 0, s, 
            (const float *)W1, (const float *)W3, d, d_ff, E, m, m16, mode, perm,
            (float *)W13_e, status);
        launch_pdl(partition_w2_kernel<float>, dim3(g2), dim3(256), 0, s, (const float *)W2, d, d_ff, E, m, m8,
                                                      mode, perm, (float *)W2_e, status);
    }
    count_launch(2);
    return cudaGetLastError();
}

}  // namespace moe
