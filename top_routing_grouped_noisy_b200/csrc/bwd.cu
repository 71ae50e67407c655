// bwd.cu -- the layer's backward pass: the combine and router backward kernels,
// the input-gradient assembly, and the C-ABI entry points (moe_*_backward).
// The loss is l(y) + c L_balance; the caller passes dy = dl/dy and c.  Each kernel
// is the chain rule of one forward step ("Llama 3 Meets MoE", section 3 for the
// noisy Top-k router and the combine; "LLaMA-MoE v2", sections "门控机制设计"
// (L_balance) and "重新缩放机制" (the E/k scale)):
//   combine   d_out[r] = s G_tj dy_t,  dG_tj = s <dy_t, out_r>  (dropped: 0)
//   router    Mixtral  dH[idx_j] = G_j (dG_j - sum_l G_l dG_l)
//             ST       dH_e = p_e (g_e - sum_l p_l g_l), g = dG scattered to experts
//             balance  dH_e += p_e (b_e - sum_l p_l b_l), b_e = c lambda f_e / T
//             dL = dH, dN = dH eps sigmoid(N); dW_g = x^T dL, dW_noise = x^T dN,
//             db = sum_t dL
//   input     dx_t = sum_j dx_perm[slot_row[t][j]] + W_g dL_t + W_noise dN_t
// The expert GEMMs are in bwd_tc.cu.  bf16 layers only; every sum is f32 in a
// fixed order, so the results do not depend on scheduling.
#include <cstdio>

#include "common.cuh"
#include "kernels.h"

namespace moe {

cudaError_t launch_bwd_dh(const moe_params_t *p, const void *d_out, const int32_t *offsets,
                          const void *W2_e, void *dh, int32_t *status, cudaStream_t s);
cudaError_t launch_bwd_dgu(const moe_params_t *p, const void *x_perm, const int32_t *offsets,
                           const void *W13, const void *dh, void *dgu, int32_t *status,
                           cudaStream_t s);
cudaError_t launch_bwd_dx(const moe_params_t *p, const void *dgu, const int32_t *offsets,
                          const void *W13_e, void *dx_perm, int32_t *status, cudaStream_t s);
cudaError_t launch_bwd_wgrad(const moe_params_t *p, const void *A, int M, int a_ld, const void *B,
                             int n_cols, int b_ld, const int32_t *offsets, void *dW, int ld_dw,
                             int n_valid, int32_t *status, cudaStream_t s);


namespace {

constexpr int kPartChunks = 64;  // token chunks of the router weight-gradient partials

// Sections of the backward workspace (after the 256-byte header).
struct BwdLayout {
    size_t dgu, dln, wt, part, total;
};

size_t al256(size_t v) { return (v + 255) & ~(size_t)255; }

BwdLayout bwd_layout(const moe_params_t *p)
{
    BwdLayout L;
    const int64_t T = p->T, d = p->d, E = p->E, k = p->k;
    const int64_t m16 = round_up(p->m, 16);
    const int64_t rows = T * k;
    size_t o = kWsHeader;
    L.dgu = o;
    o = al256(o + (size_t)(rows * 2 * m16) * 2);
    L.dln = o;
    o = al256(o + (size_t)(T * 2 * E) * 4);
    L.wt = o;  // router weights transposed, [NE2 <= 128][d] bf16
    o = al256(o + (size_t)(128 * d) * 2);
    L.part = o;  // [chunks][d][2E] then [chunks][E]
    o = al256(o + (size_t)(kPartChunks * d * 2 * E + kPartChunks * E) * 4);
    L.total = o;
    return L;
}

}  // namespace

// ---------------------------------------------------------------- combine backward
// One warp per token; lanes stride over the 16-byte vectors of the row, two vectors
// per step so that the loads of both are in flight together.  KMAX = k rounded up
// to 2, 4 or 8 sizes the per-slot registers.
template <int KMAX>
__global__ void __launch_bounds__(256) combine_backward_kernel(
    const bf16 *__restrict__ dy, const bf16 *__restrict__ out, const int32_t *__restrict__ slot_row,
    const float *__restrict__ topk_w, int T, int d, int k, float scale, bf16 *__restrict__ d_out,
    float *__restrict__ dG)
{
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T)
        return;
    int row[KMAX];
    float w[KMAX], dot[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        row[j] = j < k ? slot_row[(int64_t)t * k + j] : -1;
        w[j] = j < k ? scale * topk_w[(int64_t)t * k + j] : 0.f;
        dot[j] = 0.f;
    }
    const int nv = d / 8;
    for (int v0 = lane; v0 < nv; v0 += 64) {
        const int v1 = v0 + 32;
        const bool has1 = v1 < nv;
        const uint4 y0 = ld_nc_na(dy + (int64_t)t * d + 8 * v0);
        const uint4 y1 = has1 ? ld_nc_na(dy + (int64_t)t * d + 8 * v1) : make_uint4(0, 0, 0, 0);
        uint4 o0[KMAX], o1[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            o0[j] = row[j] >= 0 ? ld_nc_na(out + (int64_t)row[j] * d + 8 * v0)
                                : make_uint4(0, 0, 0, 0);
            o1[j] = (row[j] >= 0 && has1) ? ld_nc_na(out + (int64_t)row[j] * d + 8 * v1)
                                          : make_uint4(0, 0, 0, 0);
        }
        float fy0[8], fy1[8];
        bf16x8_to_f32(y0, fy0);
        bf16x8_to_f32(y1, fy1);
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (row[j] < 0)
                continue;
            float fo[8], g[8];
            bf16x8_to_f32(o0[j], fo);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                dot[j] += fy0[i] * fo[i];
                g[i] = w[j] * fy0[i];
            }
            st_v4(d_out + (int64_t)row[j] * d + 8 * v0, f32x8_to_bf16(g));
            if (has1) {
                bf16x8_to_f32(o1[j], fo);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    dot[j] += fy1[i] * fo[i];
                    g[i] = w[j] * fy1[i];
                }
                st_v4(d_out + (int64_t)row[j] * d + 8 * v1, f32x8_to_bf16(g));
            }
        }
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        float s = dot[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0 && j < k)
            dG[(int64_t)t * k + j] = row[j] >= 0 ? scale * s : 0.f;
    }
}

// ---------------------------------------------------------------- router backward
// W^T packed for the logit recompute: WT [NE2][d] bf16, rows 0..E-1 = W_g^T, rows
// E..2E-1 = W_noise^T (zero without noise), the rest zero.
__global__ void __launch_bounds__(256) router_pack_wt_kernel(const bf16 *__restrict__ Wg,
                                                             const bf16 *__restrict__ Wn, int d,
                                                             int E, int ne2, bf16 *__restrict__ WT)
{
    pdl_wait();
    pdl_trigger();
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)ne2 * d)
        return;
    const int n = (int)(i / d), c = (int)(i % d);
    bf16 v = __float2bfloat16_rn(0.f);
    if (n < E)
        v = Wg[(int64_t)c * E + n];
    else if (n < 2 * E && Wn != nullptr)
        v = Wn[(int64_t)c * E + n - E];
    WT[i] = v;
}

// The logits L = x W_g + b and N = x W_noise are recomputed on the tensor cores
// (mma.sync m16n8k16, bf16 in, f32 accumulate).  CTA = 16 tokens, 4 warps; warp q
// takes the 32-column K blocks q, q+4, ... of d and all NE2 / 8 output tiles.  In
// each K block lane (g, t) = (lane / 4, lane % 4) loads columns 8t .. 8t+7 of rows
// g and g+8 of x and of WT row n0 + g as 16-byte vectors; the two MMAs of the
// block read words 0-1 and 2-3 of them.  That assigns K indices to the fragment
// slots in another order than the natural one, the same for A and B, so each
// product is still a sum over all 32 columns.  The four warps' partial tiles are
// added in warp order through shared memory.  Then warp w takes tokens 4w .. 4w+3:
// lane e handles expert e (and e + 32): softmax, the Mixtral / ST Jacobian, the
// balance term, dL and dN.
constexpr int kRbTok = 16;

template <int NE2>
__global__ void __launch_bounds__(128) router_backward_token_kernel(
    const bf16 *__restrict__ x, const bf16 *__restrict__ WT, const bool noisy,
    const float *__restrict__ eps, const float *__restrict__ bias, const int32_t *__restrict__ idx,
    const float *__restrict__ G, const float *__restrict__ dG, const int32_t *__restrict__ counts,
    int T, int d, int E, int k, int router_type, float lambda, float dLb,
    float *__restrict__ dLN)
{
    pdl_wait();
    pdl_trigger();
    constexpr int NT = NE2 / 8;  // output tiles of 8
    __shared__ float red[4][kRbTok][NE2];
    __shared__ float s_ln[kRbTok][NE2];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    const int t_base = blockIdx.x * kRbTok;
    const int r0 = t_base + g, r1 = t_base + g + 8;
    float c[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
        c[j][0] = c[j][1] = c[j][2] = c[j][3] = 0.f;
    const int nkb = (d + 31) / 32;
#pragma unroll 2
    for (int kb = warp; kb < nkb; kb += 4) {
        const int col = kb * 32 + 8 * t4;
        uint4 a0 = make_uint4(0, 0, 0, 0), a1 = make_uint4(0, 0, 0, 0);
        if (col < d) {  // d % 8 == 0: a vector is all in or all out
            if (r0 < T)
                a0 = ld_nc_na(x + (int64_t)r0 * d + col);
            if (r1 < T)
                a1 = ld_nc_na(x + (int64_t)r1 * d + col);
        }
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            uint4 bv = make_uint4(0, 0, 0, 0);
            if (col < d)
                bv = ld_nc(WT + (int64_t)(j * 8 + g) * d + col);
            mma_bf16_16816(c[j], a0.x, a1.x, a0.y, a1.y, bv.x, bv.y);
            mma_bf16_16816(c[j], a0.z, a1.z, a0.w, a1.w, bv.z, bv.w);
        }
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        red[warp][g][j * 8 + 2 * t4] = c[j][0];
        red[warp][g][j * 8 + 2 * t4 + 1] = c[j][1];
        red[warp][g + 8][j * 8 + 2 * t4] = c[j][2];
        red[warp][g + 8][j * 8 + 2 * t4 + 1] = c[j][3];
    }
    __syncthreads();
    for (int v = threadIdx.x; v < kRbTok * NE2; v += blockDim.x) {
        const int tt = v / NE2, n = v % NE2;
        s_ln[tt][n] = ((red[0][tt][n] + red[1][tt][n]) + red[2][tt][n]) + red[3][tt][n];
    }
    __syncthreads();
    const float inv_tk = 1.0f / ((float)T * (float)k);
#pragma unroll 1
    for (int tt = warp * 4; tt < warp * 4 + 4; ++tt) {
        const int t = t_base + tt;
        if (t >= T)
            break;
        const float *ln = s_ln[tt];
        float H[2], N[2], p[2], gsc[2], bterm[2];
        float hmax = -INFINITY;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int e = lane + 32 * h2;
            H[h2] = -INFINITY;
            N[h2] = 0.f;
            if (e < E) {
                const float L = ln[e] + (bias ? bias[e] : 0.f);
                N[h2] = ln[E + e];
                H[h2] = L;
                if (noisy) {
                    const float z = N[h2];
                    const float sp = fmaxf(z, 0.f) + log1pf(__expf(-fabsf(z)));
                    H[h2] = L + eps[(int64_t)t * E + e] * sp;
                }
                hmax = fmaxf(hmax, H[h2]);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            hmax = fmaxf(hmax, __shfl_xor_sync(0xffffffffu, hmax, o));
        float z = 0.f;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int e = lane + 32 * h2;
            p[h2] = e < E ? __expf(H[h2] - hmax) : 0.f;
            z += p[h2];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            z += __shfl_xor_sync(0xffffffffu, z, o);
        float Smix = 0.f;
        for (int j = 0; j < k; ++j)
            Smix += G[(int64_t)t * k + j] * dG[(int64_t)t * k + j];
        float sg = 0.f, sb = 0.f, dmix[2] = {0.f, 0.f};
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int e = lane + 32 * h2;
            p[h2] /= z;
            gsc[h2] = 0.f;
            for (int j = 0; j < k; ++j)
                if (idx[(int64_t)t * k + j] == e) {
                    gsc[h2] += dG[(int64_t)t * k + j];
                    dmix[h2] += G[(int64_t)t * k + j] * (dG[(int64_t)t * k + j] - Smix);
                }
            bterm[h2] = (e < E) ? dLb * lambda * ((float)counts[e] * inv_tk) / (float)T : 0.f;
            sg += p[h2] * gsc[h2];
            sb += p[h2] * bterm[h2];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            sg += __shfl_xor_sync(0xffffffffu, sg, o);
            sb += __shfl_xor_sync(0xffffffffu, sb, o);
        }
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int e = lane + 32 * h2;
            if (e >= E)
                continue;
            float dH = router_type == MOE_ROUTER_MIXTRAL ? dmix[h2] : p[h2] * (gsc[h2] - sg);
            dH += p[h2] * (bterm[h2] - sb);
            float dN = 0.f;
            if (noisy) {
                const float sig = 1.0f / (1.0f + __expf(-N[h2]));
                dN = dH * eps[(int64_t)t * E + e] * sig;
            }
            dLN[(int64_t)t * 2 * E + e] = dH;
            dLN[(int64_t)t * 2 * E + E + e] = dN;
        }
    }
}

// Router weight gradients, partial sums per token chunk.  Thread (column pair cp,
// group eg of 8 logits) sums x[t][c] dLN[t][e2] over the chunk's tokens for its 2
// columns and 8 logits; the CTA covers 2 * 256 / (NE2 / 8) columns.  The chunk's
// x columns and dLN rows pass through shared memory 64 tokens at a time.  CTA
// column-block 0 also sums dL for db.
constexpr int kWpTok = 64;

template <int NE2>
__global__ void __launch_bounds__(256) router_backward_wpart_kernel(
    const bf16 *__restrict__ x, const float *__restrict__ dLN, int T, int d, int E,
    float *__restrict__ part, float *__restrict__ part_b)
{
    pdl_wait();
    pdl_trigger();
    constexpr int NEG = NE2 / 8;         // logit groups
    constexpr int NCP = 256 / NEG;       // column pairs per CTA
    constexpr int COLS = 2 * NCP;        // columns per CTA
    __shared__ __align__(16) bf16 s_x[kWpTok][COLS];
    __shared__ __align__(16) float s_d[kWpTok][NE2];
    const int cp = threadIdx.x % NCP, eg = threadIdx.x / NCP;
    const int c = blockIdx.x * COLS + 2 * cp;
    const int ch = blockIdx.y;
    const int tpc = (T + kPartChunks - 1) / kPartChunks;
    const int t0 = ch * tpc, t1 = min(T, t0 + tpc);
    const int E2 = 2 * E;
    float acc[2][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        acc[0][i] = acc[1][i] = 0.f;
    float accb = 0.f;
    for (int tb = t0; tb < t1; tb += kWpTok) {
        const int nt = min(kWpTok, t1 - tb);
        __syncthreads();
        for (int v = threadIdx.x; v < kWpTok * (COLS / 8); v += blockDim.x) {
            const int r = v / (COLS / 8), cv = v % (COLS / 8);
            const int cg = blockIdx.x * COLS + 8 * cv;
            uint4 u = make_uint4(0, 0, 0, 0);
            if (r < nt && cg < d)  // d % 8 == 0
                u = ld_nc_na(x + (int64_t)(tb + r) * d + cg);
            *reinterpret_cast<uint4 *>(&s_x[r][8 * cv]) = u;
        }
        for (int v = threadIdx.x; v < kWpTok * NE2; v += blockDim.x) {
            const int r = v / NE2, e2 = v % NE2;
            s_d[r][e2] = (r < nt && e2 < E2) ? dLN[(int64_t)(tb + r) * E2 + e2] : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int r = 0; r < kWpTok; ++r) {
            const __nv_bfloat162 x2 = *reinterpret_cast<const __nv_bfloat162 *>(&s_x[r][2 * cp]);
            const float x0 = __low2float(x2), x1 = __high2float(x2);
            const float4 d0 = *reinterpret_cast<const float4 *>(&s_d[r][8 * eg]);
            const float4 d1 = *reinterpret_cast<const float4 *>(&s_d[r][8 * eg + 4]);
            const float dv[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                acc[0][i] += x0 * dv[i];
                acc[1][i] += x1 * dv[i];
            }
        }
        if (blockIdx.x == 0 && threadIdx.x < E)
            for (int r = 0; r < nt; ++r)
                accb += s_d[r][threadIdx.x];
    }
#pragma unroll
    for (int h = 0; h < 2; ++h)
        if (c + h < d)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e2 = 8 * eg + i;
                if (e2 < E2)
                    part[((int64_t)ch * d + c + h) * E2 + e2] = acc[h][i];
            }
    if (blockIdx.x == 0 && threadIdx.x < E)
        part_b[ch * E + threadIdx.x] = accb;
}

// Sums the partials over the chunks in order: dWg [d][E], dWn [d][E], db [E] (f32).
__global__ void __launch_bounds__(256) router_backward_wreduce_kernel(
    const float *__restrict__ part, const float *__restrict__ part_b, int d, int E,
    float *__restrict__ dWg, float *__restrict__ dWn, float *__restrict__ db)
{
    pdl_wait();
    pdl_trigger();
    const int E2 = 2 * E;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < (int64_t)d * E2) {
        float s = 0.f;
        for (int ch = 0; ch < kPartChunks; ++ch)
            s += part[(int64_t)ch * d * E2 + i];
        const int c = (int)(i / E2), e2 = (int)(i % E2);
        if (e2 < E)
            dWg[(int64_t)c * E + e2] = s;
        else if (dWn != nullptr)
            dWn[(int64_t)c * E + e2 - E] = s;
    }
    if (blockIdx.x == 0 && threadIdx.x < E && db != nullptr) {
        float s = 0.f;
        for (int ch = 0; ch < kPartChunks; ++ch)
            s += part_b[ch * E + threadIdx.x];
        db[threadIdx.x] = s;
    }
}

// Input gradient.  CTA = `cols` columns (512, or fewer for many experts) x 128
// tokens: the router weights of its columns are copied once from the packed WT
// [NE2][d] (16-byte loads) into Ws [ne][cols] bf16; thread (token group tg,
// column group ct) owns columns 8 ct .. 8 ct + 7 and tokens tg, tg + 256 / (cols
// / 8), ...  Per element: the k expert rows in slot order, then the router term
// over e2 ascending, then (residual layer) the shared block's input gradient; f32,
// rounded to bf16 once.
constexpr int kIgTokens = 128;

__host__ __device__ inline int input_grad_cols(int E) { return E <= 16 ? 512 : (E <= 32 ? 256 : 128); }

template <int KMAX>
__global__ void __launch_bounds__(256) input_grad_kernel(
    const bf16 *__restrict__ dx_perm, const int32_t *__restrict__ slot_row,
    const bf16 *__restrict__ WT, int ne, const float *__restrict__ dLN, int T, int d, int E,
    int k, const bf16 *__restrict__ resid, bf16 *__restrict__ dx)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(16) bf16 ig_ws[];  // [ne][cols], ne = E or 2E used rows
    const int E2 = 2 * E;
    const int cols = input_grad_cols(E);
    const int nct = cols / 8, ntg = blockDim.x / nct;
    const int c_base = blockIdx.x * cols;
    for (int v = threadIdx.x; v < ne * nct; v += blockDim.x) {
        const int e2 = v / nct, cv = v % nct;
        const int c = c_base + 8 * cv;
        uint4 u = make_uint4(0, 0, 0, 0);
        if (c < d)  // d % 8 == 0
            u = ld_nc(WT + (int64_t)e2 * d + c);
        *reinterpret_cast<uint4 *>(ig_ws + (size_t)e2 * cols + 8 * cv) = u;
    }
    __syncthreads();
    const int ct = threadIdx.x % nct, tg = threadIdx.x / nct;
    const int c = c_base + 8 * ct;
    if (c >= d)
        return;
    const int t0 = blockIdx.y * kIgTokens;
    const int t1 = min(T, t0 + kIgTokens);
    // two tokens per step: all their expert rows are requested before any is summed,
    // and each weight vector read from shared memory serves both
    for (int tp = t0 + tg; tp < t1; tp += 2 * ntg) {
        const int tt[2] = {tp, tp + ntg};
        const bool v1 = tt[1] < t1;
        uint4 rv[2][KMAX];
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                const int r = (j < k && tt[q] < t1) ? slot_row[(int64_t)tt[q] * k + j] : -1;
                rv[q][j] = r >= 0 ? ld_nc_na(dx_perm + (int64_t)r * d + c) : make_uint4(0, 0, 0, 0);
            }
        float a[2][8];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
#pragma unroll
            for (int u = 0; u < 8; ++u)
                a[q][u] = 0.f;
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (j >= k)
                    break;
                float f[8];
                bf16x8_to_f32(rv[q][j], f);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    a[q][u] += f[u];
            }
        }
        const float *dl0 = dLN + (int64_t)tt[0] * E2;
        const float *dl1 = dLN + (int64_t)(v1 ? tt[1] : tt[0]) * E2;
        for (int e2 = 0; e2 < ne; ++e2) {
            const float g0 = dl0[e2], g1 = dl1[e2];
            float wf[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4 *>(ig_ws + (size_t)e2 * cols + 8 * ct),
                          wf);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                a[0][u] += g0 * wf[u];
                a[1][u] += g1 * wf[u];
            }
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            if (q == 1 && !v1)
                break;
            const int t = tt[q];
            if (resid != nullptr) {  // the shared block's input gradient (residual layer)
                float f[8];
                bf16x8_to_f32(ld_nc_na(resid + (int64_t)t * d + c), f);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    a[q][u] += f[u];
            }
            st_v4(dx + (int64_t)t * d + c, f32x8_to_bf16(a[q]));
        }
    }
}

template <int NE2>
static cudaError_t launch_router_bwd_t(const moe_params_t *p, const void *x, const void *Wg,
                                       const void *Wn, const float *eps, const float *bias,
                                       const int32_t *idx, const float *G, const float *dG,
                                       const int32_t *counts, float dLb, float *dLN, bf16 *WT,
                                       float *part, float *part_b, cudaStream_t s)
{
    count_launch(3);
    const int64_t nw = (int64_t)NE2 * p->d;
    cudaError_t e = launch_pdl(router_pack_wt_kernel, dim3((unsigned)((nw + 255) / 256)),
                               dim3(256), 0, s, (const bf16 *)Wg, (const bf16 *)Wn, p->d, p->E,
                               NE2, WT);
    if (e == cudaSuccess)
        e = launch_pdl(router_backward_token_kernel<NE2>, dim3((p->T + kRbTok - 1) / kRbTok),
                       dim3(128), 0, s, (const bf16 *)x, (const bf16 *)WT, Wn != nullptr, eps,
                       bias, idx, G, dG, counts, p->T, p->d, p->E, p->k, p->router_type,
                       p->balance_lambda, dLb, dLN);
    if (e == cudaSuccess)
        e = launch_pdl(router_backward_wpart_kernel<NE2>,
                       dim3((p->d + 2 * 256 / (NE2 / 8) - 1) / (2 * 256 / (NE2 / 8)), kPartChunks),
                       dim3(256), 0, s, (const bf16 *)x, (const float *)dLN, p->T, p->d, p->E,
                       part, part_b);
    return e;
}

static cudaError_t launch_router_bwd(const moe_params_t *p, const void *x, const void *Wg,
                                     const void *Wn, const float *eps, const float *bias,
                                     const int32_t *idx, const float *G, const float *dG,
                                     const int32_t *counts, float dLb, float *dLN, bf16 *WT,
                                     float *part, float *part_b, cudaStream_t s)
{
    const int e2 = 2 * p->E;
    if (e2 <= 16)
        return launch_router_bwd_t<16>(p, x, Wg, Wn, eps, bias, idx, G, dG, counts, dLb, dLN, WT,
                                       part, part_b, s);
    if (e2 <= 32)
        return launch_router_bwd_t<32>(p, x, Wg, Wn, eps, bias, idx, G, dG, counts, dLb, dLN, WT,
                                       part, part_b, s);
    if (e2 <= 64)
        return launch_router_bwd_t<64>(p, x, Wg, Wn, eps, bias, idx, G, dG, counts, dLb, dLN, WT,
                                       part, part_b, s);
    return launch_router_bwd_t<128>(p, x, Wg, Wn, eps, bias, idx, G, dG, counts, dLb, dLN, WT,
                                    part, part_b, s);
}

}  // namespace moe

using namespace moe;

// ------------------------------------------------------------------------ C ABI

namespace {

thread_local char g_msg[320];  // per host thread, like the library's last-error string

int fail_msg(int code, const char *fmt, const char *fn, const char *what)
{
    snprintf(g_msg, sizeof g_msg, fmt, fn, what);
    return report_error(code, g_msg);
}

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define NEED(ptr)                                                                           \
    do {                                                                                    \
        if ((ptr) == nullptr)                                                               \
            return fail_msg(MOE_ERR_INVALID_ARG, "%s: argument '%s' is NULL", fn, #ptr);    \
        if (!al16(ptr))                                                                     \
            return fail_msg(MOE_ERR_ALIGN, "%s: argument '%s' is not 16-byte aligned", fn, \
                            #ptr);                                                          \
    } while (0)

#define MAYBE(ptr)                                                                          \
    do {                                                                                    \
        if ((ptr) != nullptr && !al16(ptr))                                                 \
            return fail_msg(MOE_ERR_ALIGN, "%s: argument '%s' is not 16-byte aligned", fn, \
                            #ptr);                                                          \
    } while (0)

int check_bwd(const char *fn, const moe_params_t *p)
{
    int rc = validate_params(fn, p);
    if (rc != MOE_OK)
        return rc;
    if (p->dtype != MOE_BF16)
        return fail_msg(MOE_ERR_DTYPE, "%s: %s", fn, "the backward pass takes bf16 layers");
    if (p->T < 1)
        return fail_msg(MOE_ERR_INVALID_ARG, "%s: %s", fn, "the backward pass needs T >= 1");
    return MOE_OK;
}

int check_ws(const char *fn, const moe_params_t *p, void *ws, size_t ws_bytes)
{
    NEED(ws);
    if (ws_bytes < bwd_layout(p).total)
        return fail_msg(MOE_ERR_WORKSPACE, "%s: %s", fn,
                        "workspace smaller than moe_backward_workspace_size()");
    return MOE_OK;
}

int finish(const char *fn, cudaError_t e)
{
    if (e == cudaSuccess)
        e = cudaGetLastError();
    if (e != cudaSuccess)
        return report_cuda(e, fn);
    return report_ok();
}

}  // namespace

extern "C" size_t moe_backward_workspace_size(const moe_params_t *p)
{
    if (validate_params("moe_backward_workspace_size", p) != MOE_OK || p->T < 1)
        return 0;
    return bwd_layout(p).total;
}

extern "C" int moe_combine_backward(const moe_params_t *p, const void *dy, const void *out,
                                    const int32_t *slot_row, const float *topk_w, void *d_out,
                                    float *dG, void *stream)
{
    const char *fn = "moe_combine_backward";
    int rc = check_bwd(fn, p);
    if (rc != MOE_OK)
        return rc;
    NEED(dy);
    NEED(out);
    NEED(slot_row);
    NEED(topk_w);
    NEED(d_out);
    NEED(dG);
    const float scale = p->rescale ? (float)p->E / (float)p->k : 1.0f;
    count_launch();
    auto kern = p->k <= 2 ? combine_backward_kernel<2>
                          : (p->k <= 4 ? combine_backward_kernel<4> : combine_backward_kernel<8>);
    return finish(fn, launch_pdl(kern, dim3((p->T + 7) / 8), dim3(256), 0, (cudaStream_t)stream,
                                 (const bf16 *)dy, (const bf16 *)out, slot_row, topk_w, p->T,
                                 p->d, p->k, scale, (bf16 *)d_out, dG));
}

extern "C" int moe_expert_down_backward(const moe_params_t *p, const void *d_out, const void *h,
                                        const int32_t *offsets, const void *W2_e, void *dh,
                                        void *dW2_e, void *ws, size_t ws_bytes, void *stream)
{
    const char *fn = "moe_expert_down_backward";
    int rc = check_bwd(fn, p);
    if (rc != MOE_OK || (rc = check_ws(fn, p, ws, ws_bytes)) != MOE_OK)
        return rc;
    NEED(d_out);
    NEED(h);
    NEED(offsets);
    NEED(W2_e);
    NEED(dh);
    NEED(dW2_e);
    int32_t *status = reinterpret_cast<int32_t *>(ws);  // the workspace holds the status only
    cudaStream_t s = (cudaStream_t)stream;
    const int d = p->d, m = p->m, m8 = round_up(m, 8);
    cudaError_t e = launch_bwd_dh(p, d_out, offsets, W2_e, dh, status, s);
    if (e == cudaSuccess)  // dW2_e = d_out_e^T h_e (h columns past m read as zero)
        e = launch_bwd_wgrad(p, d_out, d, d, h, m, m8, offsets, dW2_e, m8, m8, status, s);
    return finish(fn, e);
}

extern "C" int moe_expert_up_backward(const moe_params_t *p, const void *x_perm, const void *dh,
                                      const int32_t *offsets, const void *W13_e, void *dx_perm,
                                      void *dW13_e, void *ws, size_t ws_bytes, void *stream)
{
    const char *fn = "moe_expert_up_backward";
    int rc = check_bwd(fn, p);
    if (rc != MOE_OK || (rc = check_ws(fn, p, ws, ws_bytes)) != MOE_OK)
        return rc;
    NEED(x_perm);
    NEED(dh);
    NEED(offsets);
    NEED(W13_e);
    NEED(dx_perm);
    NEED(dW13_e);
    const BwdLayout L = bwd_layout(p);
    char *w = static_cast<char *>(ws);
    int32_t *status = reinterpret_cast<int32_t *>(ws);
    cudaStream_t s = (cudaStream_t)stream;
    const int d = p->d, m16 = round_up(p->m, 16);
    cudaError_t e = launch_bwd_dgu(p, x_perm, offsets, W13_e, dh, w + L.dgu, status, s);
    if (e == cudaSuccess)
        e = launch_bwd_dx(p, w + L.dgu, offsets, W13_e, dx_perm, status, s);
    if (e == cudaSuccess)  // dW13_e = dGU_e^T x_e
        e = launch_bwd_wgrad(p, w + L.dgu, 2 * m16, 2 * m16, x_perm, d, d, offsets, dW13_e, d, d,
                             status, s);
    return finish(fn, e);
}

namespace {

static int route_backward(const char *fn, const moe_params_t *p, const void *x, const void *Wg,
                          const void *Wnoise, const float *noise, const float *bias,
                          const int32_t *topk_idx, const float *topk_w, const float *dG,
                          const int32_t *counts, float dLb, const void *dx_perm,
                          const int32_t *slot_row, const void *resid, void *dx, float *dWg,
                          float *dWnoise, float *dbias, void *ws, size_t ws_bytes, void *stream)
{
    int rc = check_bwd(fn, p);
    if (rc != MOE_OK || (rc = check_ws(fn, p, ws, ws_bytes)) != MOE_OK)
        return rc;
    NEED(x);
    NEED(Wg);
    NEED(topk_idx);
    NEED(topk_w);
    NEED(dG);
    NEED(counts);
    NEED(dx_perm);
    NEED(slot_row);
    NEED(dx);
    NEED(dWg);
    MAYBE(resid);
    MAYBE(Wnoise);
    MAYBE(noise);
    MAYBE(bias);
    MAYBE(dWnoise);
    MAYBE(dbias);
    if ((Wnoise == nullptr) != (noise == nullptr) || (Wnoise == nullptr) != (dWnoise == nullptr))
        return fail_msg(MOE_ERR_INVALID_ARG, "%s: %s", fn,
                        "Wnoise, noise and dWnoise are given together or not at all");
    if ((bias == nullptr) != (dbias == nullptr))
        return fail_msg(MOE_ERR_INVALID_ARG, "%s: %s", fn, "bias and dbias go together");
    const BwdLayout L = bwd_layout(p);
    char *w = static_cast<char *>(ws);
    float *dLN = reinterpret_cast<float *>(w + L.dln);
    float *part = reinterpret_cast<float *>(w + L.part);
    float *part_b = part + (size_t)kPartChunks * p->d * 2 * p->E;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = launch_router_bwd(p, x, Wg, Wnoise, noise, bias, topk_idx, topk_w, dG, counts,
                                      dLb, dLN, reinterpret_cast<bf16 *>(w + L.wt), part, part_b,
                                      s);
    if (e == cudaSuccess) {
        count_launch(2);
        const int64_t n = (int64_t)p->d * 2 * p->E;
        e = launch_pdl(router_backward_wreduce_kernel, dim3((unsigned)((n + 255) / 256)),
                       dim3(256), 0, s, (const float *)part, (const float *)part_b, p->d, p->E,
                       dWg, dWnoise, dbias);
        if (e == cudaSuccess) {
            const int cols = input_grad_cols(p->E);
            const int ne = Wnoise != nullptr ? 2 * p->E : p->E;
            const size_t smem = (size_t)ne * cols * sizeof(bf16);
            auto kern = p->k <= 2 ? input_grad_kernel<2>
                                  : (p->k <= 4 ? input_grad_kernel<4> : input_grad_kernel<8>);
            if (smem > 48 * 1024)
                e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
            if (e == cudaSuccess)
                e = launch_pdl(kern,
                               dim3((p->d + cols - 1) / cols, (p->T + kIgTokens - 1) / kIgTokens),
                               dim3(256), smem, s, (const bf16 *)dx_perm, slot_row,
                               (const bf16 *)(w + L.wt), ne, (const float *)dLN, p->T, p->d,
                               p->E, p->k, (const bf16 *)resid, (bf16 *)dx);
        }
    }
    return finish(fn, e);
}

}  // namespace

extern "C" int moe_route_backward(const moe_params_t *p, const void *x, const void *Wg,
                                  const void *Wnoise, const float *noise, const float *bias,
                                  const int32_t *topk_idx, const float *topk_w, const float *dG,
                                  const int32_t *counts, float dLb, const void *dx_perm,
                                  const int32_t *slot_row, void *dx, float *dWg, float *dWnoise,
                                  float *dbias, void *ws, size_t ws_bytes, void *stream)
{
    return route_backward("moe_route_backward", p, x, Wg, Wnoise, noise, bias, topk_idx, topk_w,
                          dG, counts, dLb, dx_perm, slot_row, nullptr, dx, dWg, dWnoise, dbias,
                          ws, ws_bytes, stream);
}

extern "C" int moe_backward(const moe_params_t *p, const moe_buffers_t *b,
                            const moe_bwd_buffers_t *g, float dLb, void *ws, size_t ws_bytes,
                            void *stream)
{
    const char *fn = "moe_backward";
    if (b == nullptr || g == nullptr)
        return fail_msg(MOE_ERR_INVALID_ARG, "%s: %s", fn, "buffers are NULL");
    int rc = moe_combine_backward(p, g->dy, b->out, b->slot_row, b->topk_w, g->d_out, g->dG,
                                  stream);
    if (rc == MOE_OK)
        rc = moe_expert_down_backward(p, g->d_out, b->h, b->offsets, b->W2_e, g->dh, g->dW2_e, ws,
                                      ws_bytes, stream);
    if (rc == MOE_OK)
        rc = moe_expert_up_backward(p, b->x_perm, g->dh, b->offsets, b->W13_e, g->dx_perm,
                                    g->dW13_e, ws, ws_bytes, stream);
    if (rc == MOE_OK)
        rc = moe_route_backward(p, b->x, b->Wg, b->Wnoise, b->noise, b->bias, b->topk_idx,
                                b->topk_w, g->dG, b->counts, dLb, g->dx_perm, b->slot_row, g->dx,
                                g->dWg, g->dWnoise, g->dbias, ws, ws_bytes, stream);
    return rc;
}

// ---------------------------------------------------------------- residual layer
// y = FFN_S(x) + s sum_j G_j E_j(x): the shared block's output gradient is dy
// itself; its backward is the expert backward of a one-expert layer over all T
// tokens (offsets {0, T}), and its input gradient joins dx in the input-gradient
// kernel.

namespace {

moe_params_t shared_params(const moe_params_t *p, int32_t m_s)
{
    moe_params_t ps = *p;
    ps.E = 1;
    ps.k = 1;
    ps.m = m_s;
    ps.capacity = -1;
    ps.rescale = 0;
    return ps;
}

// words 8-9 of the backward workspace header: the offsets {0, T} of the shared block
constexpr int kBwdTokenRangeWord = 8;

}  // namespace

extern "C" size_t moe_backward_residual_workspace_size(const moe_params_t *p, int32_t m_s)
{
    if (validate_params("moe_backward_residual_workspace_size", p) != MOE_OK || p->T < 1 ||
        m_s < 1)
        return 0;
    const moe_params_t ps = shared_params(p, m_s);
    const size_t a = bwd_layout(p).total, b = bwd_layout(&ps).total;
    return a > b ? a : b;
}

extern "C" int moe_backward_residual(const moe_params_t *p, const moe_buffers_t *b,
                                     const moe_bwd_buffers_t *g, const void *W13_s,
                                     const void *W2_s, int32_t m_s, const void *h_s, void *dh_s,
                                     void *dx_s, void *dW13_s, void *dW2_s, float dLb, void *ws,
                                     size_t ws_bytes, void *stream)
{
    const char *fn = "moe_backward_residual";
    if (b == nullptr || g == nullptr)
        return fail_msg(MOE_ERR_INVALID_ARG, "%s: %s", fn, "buffers are NULL");
    int rc = check_bwd(fn, p);
    if (rc != MOE_OK)
        return rc;
    if (m_s < 1)
        return fail_msg(MOE_ERR_SHAPE, "%s: %s", fn, "m_s must be >= 1");
    NEED(ws);
    if (ws_bytes < moe_backward_residual_workspace_size(p, m_s))
        return fail_msg(MOE_ERR_WORKSPACE, "%s: %s", fn,
                        "workspace smaller than moe_backward_residual_workspace_size()");
    NEED(W13_s);
    NEED(W2_s);
    NEED(h_s);
    NEED(dh_s);
    NEED(dx_s);
    NEED(dW13_s);
    NEED(dW2_s);
    const moe_params_t ps = shared_params(p, m_s);
    int32_t *tok = reinterpret_cast<int32_t *>(ws) + kBwdTokenRangeWord;
    cudaError_t e = launch_token_range(tok, p->T, (cudaStream_t)stream);
    if (e != cudaSuccess)
        return finish(fn, e);
    rc = moe_expert_down_backward(&ps, g->dy, h_s, tok, W2_s, dh_s, dW2_s, ws, ws_bytes, stream);
    if (rc == MOE_OK)
        rc = moe_expert_up_backward(&ps, b->x, dh_s, tok, W13_s, dx_s, dW13_s, ws, ws_bytes,
                                    stream);
    if (rc == MOE_OK)
        rc = moe_combine_backward(p, g->dy, b->out, b->slot_row, b->topk_w, g->d_out, g->dG,
                                  stream);
    if (rc == MOE_OK)
        rc = moe_expert_down_backward(p, g->d_out, b->h, b->offsets, b->W2_e, g->dh, g->dW2_e, ws,
                                      ws_bytes, stream);
    if (rc == MOE_OK)
        rc = moe_expert_up_backward(p, b->x_perm, g->dh, b->offsets, b->W13_e, g->dx_perm,
                                    g->dW13_e, ws, ws_bytes, stream);
    if (rc == MOE_OK)
        rc = route_backward(fn, p, b->x, b->Wg, b->Wnoise, b->noise, b->bias, b->topk_idx,
                            b->topk_w, g->dG, b->counts, dLb, g->dx_perm, b->slot_row, dx_s, g->dx,
                            g->dWg, g->dWnoise, g->dbias, ws, ws_bytes, stream);
    return rc;
}
