// decode.cu -- a3/a4 for decode-shaped bf16 batches (T <= 16 tokens): the expert
// FFN then reads each selected expert's weights once and does little arithmetic
// per byte, so it is bound by streaming weights from HBM.  SwiGLU expert as in
// "LLaMA-MoE v2", code sample "代码实现示例", class Expert.
//
// One CTA per (expert, block of weight rows): 16 neurons (32 packed W13 rows: 16
// W1 then 16 W3) for a3, 32 output rows of W2 for a4, so every SM streams
// weights.  CTAs of experts that received no rows return at once.  The product
// runs on the tensor cores (mma.sync m16n8k16, bf16 in, f32 accumulate) with the
// weight rows as the M = 16 operand and the expert's rows (in groups of up to 32,
// padded to n-tiles of 8) as N; K is split over the 8 warps and the partial sums are added
// in a fixed order through shared memory.  Each thread owns 8 consecutive K
// columns of every k32 block it visits (the same K map for both operands, as in
// the router), read with 16-byte loads; weights use non-allocating loads.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kDecodeWarps = 8;

// acc += W[0..32) . X[0..n_rows)^T over K; weight rows >= w_rows and activation
// columns >= k_valid_x read as zero.  Activation row r is Xrows + r x_ld, or,
// with a row table, Xrows + rtok[r] x_ld (rows of x gathered in dispatch order).
template <int NNT>
__device__ __forceinline__ void decode_mma_block(const bf16 *__restrict__ Wrows, int64_t w_ld,
                                                 int w_rows, const bf16 *__restrict__ Xrows,
                                                 int64_t x_ld, int n_rows, int K, int k_valid_x,
                                                 float (&acc)[2][NNT][4],
                                                 const int32_t *__restrict__ rtok = nullptr)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const int nkb = (K + 31) / 32;
    const bf16 *xrow[NNT];
#pragma unroll
    for (int nt = 0; nt < NNT; ++nt) {
        const int r = nt * 8 + g;
        xrow[nt] = r < n_rows ? Xrows + (rtok ? (int64_t)rtok[r] : (int64_t)r) * x_ld : nullptr;
    }
    // U k32 blocks per round: every load of the round is issued before its MMAs
    constexpr int U = NNT >= 4 ? 2 : 4;
    for (int kb0 = warp; kb0 < nkb; kb0 += kDecodeWarps * U) {
        uint4 wa[U][2][2];
        uint4 xb[U][NNT];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = (kb0 + u * kDecodeWarps) * 32 + 8 * q;
            const bool kv = c < K;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int ra = mt * 16 + g, rb = ra + 8;
                wa[u][mt][0] = (kv && ra < w_rows) ? ld_nc_na(Wrows + (int64_t)ra * w_ld + c)
                                                   : make_uint4(0, 0, 0, 0);
                wa[u][mt][1] = (kv && rb < w_rows) ? ld_nc_na(Wrows + (int64_t)rb * w_ld + c)
                                                   : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int nt = 0; nt < NNT; ++nt) {
                xb[u][nt] = (kv && xrow[nt] != nullptr) ? ld_nc(xrow[nt] + c)
                                                        : make_uint4(0, 0, 0, 0);
                if (c + 8 > k_valid_x) {  // activation columns past the valid K are not data
                    uint32_t *wv = reinterpret_cast<uint32_t *>(&xb[u][nt]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int c0 = c + 2 * i;
                        if (c0 >= k_valid_x)
                            wv[i] = 0u;
                        else if (c0 + 1 >= k_valid_x)
                            wv[i] &= 0x0000ffffu;
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < NNT; ++nt) {
                    if (nt * 8 < n_rows) {
                        mma_bf16_16816(acc[mt][nt], wa[u][mt][0].x, wa[u][mt][1].x,
                                       wa[u][mt][0].y, wa[u][mt][1].y, xb[u][nt].x,
                                       xb[u][nt].y);
                        mma_bf16_16816(acc[mt][nt], wa[u][mt][0].z, wa[u][mt][1].z,
                                       wa[u][mt][0].w, wa[u][mt][1].w, xb[u][nt].z,
                                       xb[u][nt].w);
                    }
                }
    }
}

// red[w][o][j]: warp w's partial sum of weight row o (0..31) and activation row j.
template <int NNT>
__device__ __forceinline__ void decode_store_partials(float *red, const float (&acc)[2][NNT][4])
{
    constexpr int NJ = NNT * 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NNT; ++nt) {
            const int o = mt * 16 + g, j = nt * 8 + 2 * q;
            float *b = red + ((size_t)warp * 32) * NJ;
            b[o * NJ + j] = acc[mt][nt][0];
            b[o * NJ + j + 1] = acc[mt][nt][1];
            b[(o + 8) * NJ + j] = acc[mt][nt][2];
            b[(o + 8) * NJ + j + 1] = acc[mt][nt][3];
        }
}

// x_rows: x_perm (expert-ordered rows), or, when row_token is given, x itself,
// whose rows are gathered through row_token; then CTA r < R also writes x_perm
// row r (x_perm_out) for inspection.
template <int NNT>
__global__ void __launch_bounds__(256) decode_up_kernel(const bf16 *__restrict__ x_rows,
                                                        const int32_t *__restrict__ offsets,
                                                        const bf16 *__restrict__ W13, int d,
                                                        int m, int blocks_per_expert,
                                                        bf16 *__restrict__ h,
                                                        const int32_t *__restrict__ row_token,
                                                        bf16 *__restrict__ x_perm_out, int E)
{
    pdl_wait();
    pdl_trigger();
    constexpr int NJ = NNT * 8;
    __shared__ float red[kDecodeWarps * 32 * NJ];
    if (row_token != nullptr && (int)blockIdx.x < offsets[E]) {
        const int r = blockIdx.x;
        const int64_t src = (int64_t)row_token[r] * d;
        for (int v = threadIdx.x; v < d / 8; v += blockDim.x)
            st_v4(x_perm_out + (int64_t)r * d + 8 * v, ld_nc(x_rows + src + 8 * v));
    }
    if ((int)blockIdx.x >= E * blocks_per_expert)  // extra CTAs of the copy only
        return;
    const int e = blockIdx.x / blocks_per_expert, blk = blockIdx.x % blocks_per_expert;
    const int r0 = offsets[e], n_rows = offsets[e + 1] - r0;
    if (n_rows <= 0)
        return;
    const int m16 = (m + 15) / 16 * 16, m8 = (m + 7) / 8 * 8;
    const bf16 *W = W13 + ((int64_t)e * 2 * m16 + (int64_t)blk * 32) * d;
    for (int rg = 0; rg < n_rows; rg += NJ) {  // more than NJ rows: the weights come from L2
        const int nr = min(NJ, n_rows - rg);
        float acc[2][NNT][4];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b = 0; b < NNT; ++b)
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    acc[a][b][c] = 0.f;
        if (row_token != nullptr)
            decode_mma_block<NNT>(W, d, 32, x_rows, d, nr, d, d, acc, row_token + r0 + rg);
        else
            decode_mma_block<NNT>(W, d, 32, x_rows + (int64_t)(r0 + rg) * d, d, nr, d, d, acc);
        if (rg > 0)
            __syncthreads();
        decode_store_partials<NNT>(red, acc);
        __syncthreads();
        // 16 neurons x nr outputs: gate row i, up row 16 + i
        for (int idx = threadIdx.x; idx < 16 * nr; idx += blockDim.x) {
            const int i = idx % 16, j = idx / 16;
            float gsum = 0.f, usum = 0.f;
#pragma unroll
            for (int w = 0; w < kDecodeWarps; ++w) {
                gsum += red[((size_t)w * 32 + i) * NJ + j];
                usum += red[((size_t)w * 32 + 16 + i) * NJ + j];
            }
            const int neuron = blk * 16 + i;
            if (neuron < m)
                h[(int64_t)(r0 + rg + j) * m8 + neuron] =
                    __float2bfloat16_rn(gsum / (1.0f + __expf(-gsum)) * usum);
        }
    }
}

template <int NNT>
__global__ void __launch_bounds__(256) decode_down_kernel(const bf16 *__restrict__ hbuf,
                                                          const int32_t *__restrict__ offsets,
                                                          const bf16 *__restrict__ W2, int d,
                                                          int m, int blocks_per_expert,
                                                          bf16 *__restrict__ out)
{
    pdl_wait();
    pdl_trigger();
    constexpr int NJ = NNT * 8;
    __shared__ float red[kDecodeWarps * 32 * NJ];
    const int e = blockIdx.x / blocks_per_expert, blk = blockIdx.x % blocks_per_expert;
    const int r0 = offsets[e], n_rows = offsets[e + 1] - r0;
    if (n_rows <= 0)
        return;
    const int m8 = (m + 7) / 8 * 8;
    const int o0 = blk * 32;  // output rows o0..o0+31 of W2_e [d][m8]
    const bf16 *W = W2 + ((int64_t)e * d + o0) * m8;
    for (int rg = 0; rg < n_rows; rg += NJ) {
        const int nr = min(NJ, n_rows - rg);
        float acc[2][NNT][4];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b = 0; b < NNT; ++b)
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    acc[a][b][c] = 0.f;
        decode_mma_block<NNT>(W, m8, d - o0, hbuf + (int64_t)(r0 + rg) * m8, m8, nr, m, m, acc);
        if (rg > 0)
            __syncthreads();
        decode_store_partials<NNT>(red, acc);
        __syncthreads();
        for (int idx = threadIdx.x; idx < 32 * nr; idx += blockDim.x) {
            const int i = idx % 32, j = idx / 32;
            const int o = o0 + i;
            if (o >= d)
                continue;
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < kDecodeWarps; ++w)
                sum += red[((size_t)w * 32 + i) * NJ + j];
            out[(int64_t)(r0 + rg + j) * d + o] = __float2bfloat16_rn(sum);
        }
    }
}

template <int NNT>
static void up_dispatch(const moe_params_t *p, const void *x_perm, const int32_t *offsets,
                        const void *W13, void *h, cudaStream_t s,
                        const int32_t *row_token = nullptr, void *x_perm_out = nullptr)
{
    const int bpe = (p->m + 15) / 16;
    const int grid = row_token ? max(p->E * bpe, p->T * p->k) : p->E * bpe;
    launch_pdl(decode_up_kernel<NNT>, dim3(grid), dim3(256), 0, s, (const bf16 *)x_perm, offsets,
               (const bf16 *)W13, p->d, p->m, bpe, (bf16 *)h, row_token, (bf16 *)x_perm_out,
               p->E);
}

template <int NNT>
static void down_dispatch(const moe_params_t *p, const void *h, const int32_t *offsets,
                          const void *W2, void *out, cudaStream_t s)
{
    const int bpe = (p->d + 31) / 32;
    launch_pdl(decode_down_kernel<NNT>, dim3(p->E * bpe), dim3(256), 0, s, (const bf16 *)h, offsets,
                                                      (const bf16 *)W2, p->d, p->m, bpe,
                                                      (bf16 *)out);
}

cudaError_t launch_up_decode(const moe_params_t *p, const void *x_perm, const int32_t *offsets,
                             const void *W13, void *h, cudaStream_t s)
{
    if (p->T <= 8)
        up_dispatch<1>(p, x_perm, offsets, W13, h, s);
    else
        up_dispatch<2>(p, x_perm, offsets, W13, h, s);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_up_decode_gather(const moe_params_t *p, const void *x, const int32_t *row_token,
                                    const int32_t *offsets, const void *W13, void *h,
                                    void *x_perm_out, cudaStream_t s)
{
    if (p->T <= 8)
        up_dispatch<1>(p, x, offsets, W13, h, s, row_token, x_perm_out);
    else
        up_dispatch<2>(p, x, offsets, W13, h, s, row_token, x_perm_out);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_down_decode(const moe_params_t *p, const void *h, const int32_t *offsets,
                               const void *W2, void *out, cudaStream_t s)
{
    if (p->T <= 8)
        down_dispatch<1>(p, h, offsets, W2, out, s);
    else
        down_dispatch<2>(p, h, offsets, W2, out, s);
    count_launch();
    return cudaGetLastError();
}

}  // namespace moe
