// decode.cu -- a3/a4 for decode-shaped bf16 batches (T <= 16 tokens): the expert
// FFN then reads each selected expert's weights once and does little arithmetic
// per byte, so it is bound by streaming weights from HBM.  SwiGLU expert as in
// "LLaMA-MoE v2", code sample "代码实现示例", class Expert; the combine that the
// moe_forward form fuses into GEMM 2 is that of "Llama 3 Meets MoE: Efficient
// Upcycling", section 3 (y = sum_i G(x)_i E_i(x)).
//
// The weights of the experts that received rows are cut into equal units of 16
// weight rows x one K slice, and the units are spread over every warp of a grid
// that fills the device once, so every SM streams the same number of bytes
// whatever the routing picked.  A warp issues all 16-byte loads of a round of its
// unit (16 rows x 8 blocks of 32 columns) before it multiplies them with the
// expert's token rows on the tensor cores (mma.sync m16n8k16, bf16 in, f32 out),
// and writes its 16 x tokens partial sums to the workspace.  The K slices of a row
// block are added in slice order by whichever warp finishes the block's last unit
// (a ticket per block, reset by that warp): no warp ever waits for another, and
// the sums do not depend on which warp came last.
//   GEMM 1: a block is one 32-row group of the packed W13 (16 W1 rows, 16 W3 rows);
//           its last warp writes h = silu(g) * u, rounded to bf16.
//   GEMM 2: a block is 16 output columns of every selected expert; its last warp
//           writes out (rounded to bf16) and, in the fused form, y for those
//           columns: s * sum_j G_tj out_{row(t,j)} in slot order, f32, one rounding
//           -- the arithmetic of combine_kernel.
// The number of K slices is chosen on the device from the routing (fewer selected
// experts, more slices), identically in every warp.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kDecKB = 8;                    // 32-column blocks per load round
constexpr int kDecTargetUnits = 148 * 16 * 2; // units aimed at (two per warp of a full grid)
constexpr int kDecTok = kDecodeMaxTokens;     // token slots of a partial block
constexpr int kDecMaxSlices = 8;              // slice partials loaded together in a reduction

// K slices for nsel experts of nb row blocks: as many as give about
// kDecTargetUnits units, in whole load rounds where possible.
__host__ __device__ inline int dec_slices(int nsel, int nb, int nk32)
{
    const int s0 = (nk32 + kDecKB - 1) / kDecKB;
    const long long base = (long long)nsel * nb * s0;
    int f = (int)(base / kDecTargetUnits);
    if (f < 1)
        f = 1;
    int S = (s0 + f - 1) / f;
    return S < 1 ? 1 : S;
}

// Partial-sum floats the decode kernels may use for a layer (upper bound over
// every routing): units <= 2 * target + nsel_max * nb, 16 rows x kDecTok each.
size_t decode_partial_floats(const moe_params_t *p)
{
    const int tm = p->T < kDecTok ? (p->T > 0 ? p->T : 1) : kDecTok;
    const int esel = p->E < tm * p->k ? p->E : tm * p->k;
    const int m16 = round_up(p->m, 16);
    const int nb_up = m16 / 8;
    const int nb_dn = ceil_div(p->d, 16);
    const int nb = nb_up > nb_dn ? nb_up : nb_dn;
    return ((size_t)2 * kDecTargetUnits + (size_t)esel * nb) * 16 * kDecTok;
}
size_t decode_ticket_ints(const moe_params_t *p)
{
    const int tm = p->T < kDecTok ? (p->T > 0 ? p->T : 1) : kDecTok;
    const int esel = p->E < tm * p->k ? p->E : tm * p->k;
    return (size_t)esel * (round_up(p->m, 16) / 16) + (size_t)ceil_div(p->d, 16);
}
bool decode_fits(const moe_params_t *p)
{
    return p->dtype == MOE_BF16 && p->T >= 1 && p->T <= kDecodeMaxTokens &&
           decode_ticket_ints(p) <= (size_t)kDecTickets;
}

// offsets of every expert and the list of experts with rows (expert order) into
// shared memory; called by all threads.
__device__ __forceinline__ int dec_selected(const int32_t *__restrict__ offsets, int E,
                                            int32_t *s_off, int32_t *s_sel)
{
    __shared__ int s_n;
    for (int e = threadIdx.x; e <= E; e += blockDim.x)
        s_off[e] = offsets[e];
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int base = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const bool has = e < E && s_off[e + 1] > s_off[e];
            const unsigned b = __ballot_sync(0xffffffffu, has);
            if (has)
                s_sel[base + __popc(b & ((1u << lane) - 1u))] = e;
            base += __popc(b);
        }
        if (lane == 0)
            s_n = base;
    }
    __syncthreads();
    return s_n;
}

// acc[nt] += W[16 rows] . X[rows nt*8 .. nt*8+7]^T over the 32-column blocks
// [kb0, kb1).  Lane (g = lane/4, q = lane%4) loads 8 consecutive columns of weight
// rows g and g + 8 and of token rows nt*8 + g; the same K permutation on both
// operands, so the dot products are exact sums over the blocks' columns.  Weight
// rows >= w_rows and token rows >= nr read as zero; columns >= kcols (a multiple
// of 8) are not loaded, and token columns >= kvalid (<= kcols) are zeroed.
template <int NNT, typename RowPtr, typename AfterLoads>
__device__ __forceinline__ void dec_unit(const bf16 *__restrict__ W, int64_t w_ld, int w_rows,
                                         RowPtr xrow, int nr, int kb0, int kb1, int kcols,
                                         int kvalid, float (&acc)[NNT][4], AfterLoads after_loads)
{
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const bf16 *xr[NNT];
#pragma unroll
    for (int nt = 0; nt < NNT; ++nt)
        xr[nt] = nt * 8 + g < nr ? xrow(nt * 8 + g) : nullptr;
    for (int kb = kb0; kb < kb1; kb += kDecKB) {
        uint4 wa[kDecKB][2], xb[kDecKB][NNT];
#pragma unroll
        for (int u = 0; u < kDecKB; ++u) {
            const int c = (kb + u) * 32 + 8 * q;
            const bool kv = kb + u < kb1 && c < kcols;
            wa[u][0] = (kv && g < w_rows) ? ld_nc_na(W + (int64_t)g * w_ld + c)
                                          : make_uint4(0, 0, 0, 0);
            wa[u][1] = (kv && g + 8 < w_rows) ? ld_nc_na(W + (int64_t)(g + 8) * w_ld + c)
                                              : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int nt = 0; nt < NNT; ++nt) {
                xb[u][nt] = (kv && xr[nt] != nullptr) ? ld_nc(xr[nt] + c) : make_uint4(0, 0, 0, 0);
                if (c + 8 > kvalid) {  // columns past the valid K are not data
                    uint32_t *wv = reinterpret_cast<uint32_t *>(&xb[u][nt]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int c0 = c + 2 * i;
                        if (c0 >= kvalid)
                            wv[i] = 0u;
                        else if (c0 + 1 >= kvalid)
                            wv[i] &= 0x0000ffffu;
                    }
                }
            }
        }
        if (kb == kb0)  // work that overlaps the first round's loads
            after_loads();
#pragma unroll
        for (int u = 0; u < kDecKB; ++u)
#pragma unroll
            for (int nt = 0; nt < NNT; ++nt)
                if (nt * 8 < nr) {
                    mma_bf16_16816(acc[nt], wa[u][0].x, wa[u][1].x, wa[u][0].y, wa[u][1].y,
                                   xb[u][nt].x, xb[u][nt].y);
                    mma_bf16_16816(acc[nt], wa[u][0].z, wa[u][1].z, wa[u][0].w, wa[u][1].w,
                                   xb[u][nt].z, xb[u][nt].w);
                }
    }
}

// A unit's partial block [16 rows][kDecTok token slots]: the slots of the NNT
// n-tiles are written (the reductions read only the expert's rows).
template <int NNT>
__device__ __forceinline__ void dec_store(float *__restrict__ blk, const float (&acc)[NNT][4])
{
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NNT; ++nt) {
        const int j = nt * 8 + 2 * q;
        __stcg(reinterpret_cast<float2 *>(blk + g * kDecTok + j), make_float2(acc[nt][0], acc[nt][1]));
        __stcg(reinterpret_cast<float2 *>(blk + (g + 8) * kDecTok + j),
               make_float2(acc[nt][2], acc[nt][3]));
    }
}

// Block tickets.  After a unit's partial block is stored, lane 0 adds one to the
// block's ticket with release-acquire semantics at GPU scope (the warp barrier before
// it orders every lane's stores); the old value is looked at only after the warp's
// next unit has issued its loads, so the atomic's round trip overlaps them.  The warp
// that sees target - 1 finished the block last: it resets the ticket and adds the
// slices (every other unit's partials were released before its ticket increment).
__device__ __forceinline__ int ticket_add(int32_t *ticket)
{
    int old = 0;
    __syncwarp();
    if ((threadIdx.x & 31) == 0)
        asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;"
                     : "=r"(old)
                     : "l"(ticket)
                     : "memory");
    return old;
}
__device__ __forceinline__ bool ticket_last(int old, int32_t *ticket, int target)
{
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old != target - 1)
        return false;
    if ((threadIdx.x & 31) == 0)
        *ticket = 0;
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    __syncwarp();
    return true;
}

// GEMM 1 + SwiGLU.  x_rows: x_perm (rows in expert order), or with row_token, x
// itself (rows gathered through row_token; then the CTAs also write x_perm).
template <int NNT, int WARPS>
__global__ void __launch_bounds__(WARPS * 32, 1) decode_up_kernel(
    const bf16 *__restrict__ x_rows, const int32_t *__restrict__ row_token,
    bf16 *__restrict__ x_perm_out, const int32_t *__restrict__ offsets,
    const bf16 *__restrict__ W13, int d, int m, int E, bf16 *__restrict__ h,
    float *__restrict__ pre, int32_t *__restrict__ tickets)
{
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1], s_sel[MOE_MAX_EXPERTS];
    const int nsel = dec_selected(offsets, E, s_off, s_sel);
    if (row_token != nullptr) {  // x_perm for inspection: row r = x[row_token[r]]
        const int R = s_off[E];
        for (int r = blockIdx.x; r < R; r += gridDim.x) {
            const int64_t src = (int64_t)row_token[r] * d;
            for (int v = threadIdx.x; v < d / 8; v += blockDim.x)
                st_v4(x_perm_out + (int64_t)r * d + 8 * v, ld_nc(x_rows + src + 8 * v));
        }
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m16 = round_up(m, 16), m8 = round_up(m, 8);
    const int nb = m16 / 8;  // 16-row blocks: 2b = W1 rows of group b, 2b+1 = its W3 rows
    const int nk32 = (d + 31) / 32;
    const int S = dec_slices(nsel, nb, nk32);
    const int units = nsel * nb * S;
    const int gw = blockIdx.x * WARPS + warp, nw = gridDim.x * WARPS;
    // the group's last unit: add the slices in order, h = silu(g) * u
    auto reduce_group = [&](int is, int grp) {
        const int e = s_sel[is], r0 = s_off[e], nr = s_off[e + 1] - r0;
        const float *gp = pre + (int64_t)(is * nb + 2 * grp) * S * 16 * kDecTok;
        const float *up = gp + (int64_t)S * 16 * kDecTok;
        for (int o = lane; o < 16 * nr; o += 32) {
            const int i = o % 16, j = o / 16;
            float gs = 0.f, us = 0.f;
            for (int s0 = 0; s0 < S; s0 += kDecMaxSlices) {
                // every load of a batch of slices is issued before the first add
                float gv[kDecMaxSlices], uv[kDecMaxSlices];
#pragma unroll
                for (int s2 = 0; s2 < kDecMaxSlices; ++s2) {
                    const bool ok = s0 + s2 < S;
                    const int64_t off = ((int64_t)(s0 + s2) * 16 + i) * kDecTok + j;
                    gv[s2] = ok ? __ldcg(gp + off) : 0.f;
                    uv[s2] = ok ? __ldcg(up + off) : 0.f;
                }
#pragma unroll
                for (int s2 = 0; s2 < kDecMaxSlices; ++s2)
                    if (s0 + s2 < S) {
                        gs += gv[s2];
                        us += uv[s2];
                    }
            }
            const int neuron = grp * 16 + i;
            if (neuron < m)
                h[(int64_t)(r0 + j) * m8 + neuron] = __float2bfloat16_rn(gs / (1.0f + __expf(-gs)) * us);
        }
    };
    int pend_old = 0, pend_is = -1, pend_grp = 0;  // the previous unit's ticket
    auto settle = [&]() {
        if (pend_is < 0)
            return;
        int32_t *tk = tickets + pend_is * (nb / 2) + pend_grp;
        if (ticket_last(pend_old, tk, 2 * S))
            reduce_group(pend_is, pend_grp);
        pend_is = -1;
    };
    for (int u = gw; u < units; u += nw) {
        const int s = u % S, blk = (u / S) % nb, is = u / (S * nb);
        const int e = s_sel[is], r0 = s_off[e], nr = s_off[e + 1] - r0;
        const bf16 *W = W13 + ((int64_t)e * 2 * m16 + (int64_t)blk * 16) * d;
        float acc[NNT][4];
#pragma unroll
        for (int a = 0; a < NNT; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                acc[a][c] = 0.f;
        const int kb0 = (int)((int64_t)s * nk32 / S), kb1 = (int)((int64_t)(s + 1) * nk32 / S);
        if (row_token != nullptr)
            dec_unit<NNT>(W, d, 16, [&](int j) { return x_rows + (int64_t)row_token[r0 + j] * d; },
                          nr, kb0, kb1, d, d, acc, settle);
        else
            dec_unit<NNT>(W, d, 16, [&](int j) { return x_rows + (int64_t)(r0 + j) * d; }, nr,
                          kb0, kb1, d, d, acc, settle);
        float *blkp = pre + ((int64_t)(is * nb + blk) * S + s) * 16 * kDecTok;
        dec_store<NNT>(blkp, acc);
        pend_old = ticket_add(tickets + is * (nb / 2) + (blk >> 1));
        pend_is = is;
        pend_grp = blk >> 1;
    }
    settle();
}

// GEMM 2 (+ the combine when y != NULL).
template <int NNT, int WARPS>
__global__ void __launch_bounds__(WARPS * 32, 1) decode_down_kernel(
    const bf16 *__restrict__ hbuf, const int32_t *__restrict__ offsets,
    const bf16 *__restrict__ W2, int d, int m, int E, bf16 *__restrict__ out,
    float *__restrict__ pre, int32_t *__restrict__ tickets, int T, int k,
    const int32_t *__restrict__ slot_row, const float *__restrict__ gw_in, float scale,
    bf16 *__restrict__ y)
{
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1], s_sel[MOE_MAX_EXPERTS];
    const int nsel = dec_selected(offsets, E, s_off, s_sel);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m8 = round_up(m, 8);
    const int nob = (d + 15) / 16;  // 16 output columns per block
    const int nk32 = (m8 + 31) / 32;
    const int S = dec_slices(nsel, nob, nk32);
    const int units = nsel * nob * S;
    const int R = s_off[E];
    const int gw = blockIdx.x * WARPS + warp, nw = gridDim.x * WARPS;
    // the block's last unit: out of every kept row (slices in order), then y
    auto reduce_block = [&](int ob) {
        const float *bp = pre + (int64_t)ob * nsel * S * 16 * kDecTok;
        for (int o = lane; o < 16 * R; o += 32) {
            const int i = o % 16, r = o / 16, col = ob * 16 + i;
            if (col >= d)
                continue;
            int isr = 0;  // selected-expert index of row r
            while (s_off[s_sel[isr] + 1] <= r)
                ++isr;
            const int j = r - s_off[s_sel[isr]];
            const float *rp = bp + (int64_t)isr * S * 16 * kDecTok;
            float v = 0.f;
            for (int s0 = 0; s0 < S; s0 += kDecMaxSlices) {
                float pv[kDecMaxSlices];  // loads first, then the adds in slice order
#pragma unroll
                for (int s2 = 0; s2 < kDecMaxSlices; ++s2)
                    pv[s2] = s0 + s2 < S ? __ldcg(rp + ((int64_t)(s0 + s2) * 16 + i) * kDecTok + j)
                                         : 0.f;
#pragma unroll
                for (int s2 = 0; s2 < kDecMaxSlices; ++s2)
                    if (s0 + s2 < S)
                        v += pv[s2];
            }
            out[(int64_t)r * d + col] = __float2bfloat16_rn(v);
        }
        if (y == nullptr)
            return;
        __threadfence();  // this warp's out values, read back below by other lanes
        __syncwarp();
        for (int o = lane; o < 16 * T; o += 32) {
            const int i = o % 16, t = o / 16, col = ob * 16 + i;
            if (col >= d)
                continue;
            float ov[MOE_MAX_TOPK], gv[MOE_MAX_TOPK];  // loads first, then the sum in slot order
            bool kept[MOE_MAX_TOPK];
#pragma unroll
            for (int j = 0; j < MOE_MAX_TOPK; ++j) {
                const int32_t row = j < k ? slot_row[t * k + j] : -1;
                kept[j] = row >= 0;
                ov[j] = kept[j] ? __bfloat162float(__ldcg(out + (int64_t)row * d + col)) : 0.f;
                gv[j] = kept[j] ? gw_in[t * k + j] : 0.f;
            }
            float a = 0.f;
#pragma unroll
            for (int j = 0; j < MOE_MAX_TOPK; ++j)
                if (kept[j])
                    a = fmaf(gv[j], ov[j], a);
            a *= scale;
            y[(int64_t)t * d + col] = __float2bfloat16_rn(a);
        }
    };
    int pend_old = 0, pend_ob = -1;  // the previous unit's ticket
    auto settle = [&]() {
        if (pend_ob < 0)
            return;
        if (ticket_last(pend_old, tickets + pend_ob, nsel * S))
            reduce_block(pend_ob);
        pend_ob = -1;
    };
    for (int u = gw; u < units; u += nw) {
        // output block fastest across the selected experts: a block's units spread
        const int s = u % S, is = (u / S) % nsel, ob = u / (S * nsel);
        const int e = s_sel[is], r0 = s_off[e], nr = s_off[e + 1] - r0;
        const bf16 *W = W2 + ((int64_t)e * d + (int64_t)ob * 16) * m8;
        float acc[NNT][4];
#pragma unroll
        for (int a = 0; a < NNT; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                acc[a][c] = 0.f;
        const int kb0 = (int)((int64_t)s * nk32 / S), kb1 = (int)((int64_t)(s + 1) * nk32 / S);
        dec_unit<NNT>(W, m8, d - ob * 16, [&](int j) { return hbuf + (int64_t)(r0 + j) * m8; },
                      nr, kb0, kb1, m8, m, acc, settle);
        float *blkp = pre + ((int64_t)(ob * nsel + is) * S + s) * 16 * kDecTok;
        dec_store<NNT>(blkp, acc);
        pend_old = ticket_add(tickets + ob);
        pend_ob = ob;
    }
    settle();
}

// ------------------------------------------------------------------ row-block kernels
// For at most kRbMaxTok tokens per expert (decode batches of up to 8 tokens) the
// weights are cut into blocks whose sums all end in one CTA, so no partial sum ever
// leaves the CTA that made it:
//   GEMM 1: a block is 4 neurons of one selected expert -- their 4 W1 rows and 4 W3
//           rows (two runs of 4 contiguous rows of the packed W13) -- so the CTA
//           finishes h = silu(g) * u of those neurons itself;
//   GEMM 2: a block is 4 output columns (4 rows of W2_e) of every selected expert,
//           so the CTA finishes out for those columns and, in the fused form, y.
// Each CTA takes an equal contiguous run of blocks (whatever the routing picked,
// every SM streams the same bytes, within one block).  Its 16 warps split K: lane
// l of warp w multiplies the 16-byte vectors w * nvw + l (+ 32 i) of every row of
// the block with the same vectors of the expert's token rows (f32 FMA in column
// order), the lanes' sums are added by a butterfly and the warps' sums in warp
// order.  The first vector of the next block's rows is loaded before the current
// block's sums are reduced, so a CTA keeps two blocks' loads in flight.  The GEMM 1
// kernel also asks L2 to prefetch the W2 rows that the GEMM 2 CTA of the same index
// will read, so GEMM 2 streams from L2 while GEMM 1 still runs.
constexpr int kRbWarps = 16;
constexpr int kRbMaxTok = 8;

__device__ __forceinline__ float warp_sum_f(float v)
{
#pragma unroll
    for (int s = 16; s > 0; s >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, s);
    return v;
}

__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)),
                 "r"(bytes)
                 : "memory");
}

// The GEMM 2 blocks of CTA c of a grid of g CTAs: [c nblk / g, (c+1) nblk / g).
__device__ __forceinline__ void rb_range(int nblk, int c, int g, int &b0, int &b1)
{
    b0 = (int)((int64_t)c * nblk / g);
    b1 = (int)((int64_t)(c + 1) * nblk / g);
}

template <int TM>
__global__ void __launch_bounds__(kRbWarps * 32, 1) decode_up_rows_kernel(
    const bf16 *__restrict__ x_rows, const int32_t *__restrict__ row_token,
    bf16 *__restrict__ x_perm_out, const int32_t *__restrict__ offsets,
    const bf16 *__restrict__ W13, int d, int m, int E, bf16 *__restrict__ h,
    const bf16 *__restrict__ W2)
{
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1], s_sel[MOE_MAX_EXPERTS];
    __shared__ float red[kRbWarps][8][TM];
    const int nsel = dec_selected(offsets, E, s_off, s_sel);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m16 = round_up(m, 16), m8 = round_up(m, 8);
    if (W2 != nullptr && threadIdx.x < nsel) {  // the GEMM 2 rows of this CTA index, into L2
        int o0, o1;
        rb_range((d + 3) / 4, blockIdx.x, gridDim.x, o0, o1);
        o0 *= 4;
        o1 = min(d, o1 * 4);
        if (o1 > o0)
            prefetch_l2(W2 + ((int64_t)s_sel[threadIdx.x] * d + o0) * m8,
                        (uint32_t)((int64_t)(o1 - o0) * m8 * 2));
    }
    if (row_token != nullptr) {  // x_perm for inspection: row r = x[row_token[r]]
        const int R = s_off[E];
        for (int r = blockIdx.x; r < R; r += gridDim.x) {
            const int64_t src = (int64_t)row_token[r] * d;
            for (int v = threadIdx.x; v < d / 8; v += blockDim.x)
                st_v4(x_perm_out + (int64_t)r * d + 8 * v, ld_nc(x_rows + src + 8 * v));
        }
    }
    const int nq = m16 / 4;  // neuron quads per expert
    int b0, b1;
    rb_range(nsel * nq, blockIdx.x, gridDim.x, b0, b1);
    const int nv = d / 8, nvw = (nv + kRbWarps - 1) / kRbWarps;
    const int v0 = warp * nvw, v1 = min(nv, v0 + nvw);
    // weight row rr (0..7) of block b: rows 0-3 W1, 4-7 W3 of its 4 neurons
    auto wrow = [&](int b, int rr) {
        const int is = b / nq, qd = b % nq;
        const int e = s_sel[is];
        const int row = (qd >> 2) * 32 + (qd & 3) * 4 + (rr & 3) + (rr >> 2) * 16;
        return W13 + ((int64_t)e * 2 * m16 + row) * d;
    };
    uint4 wn[8];  // the first vector of the next block's rows
    const bool first = v0 + lane < v1;
    if (b0 < b1 && first)
#pragma unroll
        for (int rr = 0; rr < 8; ++rr)
            wn[rr] = ld_nc_na(wrow(b0, rr) + (int64_t)(v0 + lane) * 8);
    for (int b = b0; b < b1; ++b) {
        const int is = b / nq, qd = b % nq;
        const int e = s_sel[is], r0 = s_off[e], nr = min(s_off[e + 1] - r0, TM);
        float acc[8][TM];
#pragma unroll
        for (int rr = 0; rr < 8; ++rr)
#pragma unroll
            for (int j = 0; j < TM; ++j)
                acc[rr][j] = 0.f;
        for (int v = v0 + lane; v < v1; v += 32) {
            uint4 w[8];
#pragma unroll
            for (int rr = 0; rr < 8; ++rr)
                w[rr] = v == v0 + lane ? wn[rr] : ld_nc_na(wrow(b, rr) + (int64_t)v * 8);
#pragma unroll
            for (int j = 0; j < TM; ++j) {
                if (j >= nr)
                    break;
                const int64_t xr = row_token != nullptr ? (int64_t)row_token[r0 + j] : (int64_t)(r0 + j);
                float xf[8];
                bf16x8_to_f32(ld_nc(x_rows + xr * d + (int64_t)v * 8), xf);
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    float wf[8];
                    bf16x8_to_f32(w[rr], wf);
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        acc[rr][j] = fmaf(wf[c], xf[c], acc[rr][j]);
                }
            }
        }
        if (b + 1 < b1 && first)  // the next block's loads overlap this block's sums
#pragma unroll
            for (int rr = 0; rr < 8; ++rr)
                wn[rr] = ld_nc_na(wrow(b + 1, rr) + (int64_t)(v0 + lane) * 8);
#pragma unroll
        for (int rr = 0; rr < 8; ++rr)
#pragma unroll
            for (int j = 0; j < TM; ++j) {
                const float sm = warp_sum_f(acc[rr][j]);
                if (lane == 0)
                    red[warp][rr][j] = sm;
            }
        __syncthreads();
        if ((int)threadIdx.x < 4 * nr) {
            const int qq = threadIdx.x & 3, j = threadIdx.x >> 2;
            float g = 0.f, u = 0.f;
#pragma unroll
            for (int w = 0; w < kRbWarps; ++w) {
                g += red[w][qq][j];
                u += red[w][4 + qq][j];
            }
            const int neuron = (qd >> 2) * 16 + (qd & 3) * 4 + qq;
            if (neuron < m)
                h[(int64_t)(r0 + j) * m8 + neuron] = __float2bfloat16_rn(g / (1.0f + __expf(-g)) * u);
        }
        __syncthreads();
    }
}

template <int TM>
__global__ void __launch_bounds__(kRbWarps * 32, 1) decode_down_rows_kernel(
    const bf16 *__restrict__ hbuf, const int32_t *__restrict__ offsets,
    const bf16 *__restrict__ W2, int d, int m, int E, bf16 *__restrict__ out, int T, int k,
    const int32_t *__restrict__ slot_row, const float *__restrict__ gw_in, float scale,
    bf16 *__restrict__ y)
{
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1], s_sel[MOE_MAX_EXPERTS];
    __shared__ float red[MOE_MAX_EXPERTS * 4][TM];   // per (item, K part) pair (<= 256)
    __shared__ float outs[MOE_MAX_EXPERTS * 4][TM];  // the block's out, rounded
    const int nsel = dec_selected(offsets, E, s_off, s_sel);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m8 = round_up(m, 8);
    const int nv = m8 / 8;
    const int items = nsel * 4;  // (selected expert, output row of the block)
    // K parts per item so that items x parts fill the 16 warps (1, 2 or 4)
    const int parts = items >= kRbWarps ? 1 : (items * 2 >= kRbWarps ? 2 : 4);
    const int pairs = items * parts;
    int b0, b1;
    rb_range((d + 3) / 4, blockIdx.x, gridDim.x, b0, b1);
    for (int b = b0; b < b1; ++b) {
        for (int pr = warp; pr < pairs; pr += kRbWarps) {
            const int item = pr / parts, part = pr % parts;
            const int is = item >> 2, o = b * 4 + (item & 3);
            const int e = s_sel[is], r0 = s_off[e], nr = min(s_off[e + 1] - r0, TM);
            float acc[TM];
#pragma unroll
            for (int j = 0; j < TM; ++j)
                acc[j] = 0.f;
            if (o < d) {
                const bf16 *W = W2 + ((int64_t)e * d + o) * m8;
                const int va = (int)((int64_t)part * nv / parts), vb = (int)((int64_t)(part + 1) * nv / parts);
                for (int v = va + lane; v < vb; v += 32) {
                    float wf[8];
                    bf16x8_to_f32(ld_nc_na(W + (int64_t)v * 8), wf);
#pragma unroll
                    for (int j = 0; j < TM; ++j) {
                        if (j >= nr)
                            break;
                        float hf[8];
                        bf16x8_to_f32(ld_nc(hbuf + (int64_t)(r0 + j) * m8 + (int64_t)v * 8), hf);
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            if (v * 8 + c < m)  // h columns past m are not data
                                acc[j] = fmaf(wf[c], hf[c], acc[j]);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < TM; ++j) {
                const float sm = warp_sum_f(acc[j]);
                if (lane == 0)
                    red[pr][j] = sm;
            }
        }
        __syncthreads();
        for (int i = threadIdx.x; i < items * TM; i += blockDim.x) {
            const int item = i / TM, j = i % TM;
            const int is = item >> 2, o = b * 4 + (item & 3);
            const int e = s_sel[is], r0 = s_off[e], nr = s_off[e + 1] - r0;
            if (o >= d || j >= nr)
                continue;
            float sum = 0.f;
            for (int pt = 0; pt < parts; ++pt)
                sum += red[item * parts + pt][j];
            const bf16 ob = __float2bfloat16_rn(sum);
            out[(int64_t)(r0 + j) * d + o] = ob;
            outs[item][j] = __bfloat162float(ob);
        }
        __syncthreads();
        if (y != nullptr)  // the combine of this block's columns (combine_kernel's arithmetic)
            for (int i = threadIdx.x; i < T * 4; i += blockDim.x) {
                const int t = i >> 2, o = b * 4 + (i & 3);
                if (o >= d)
                    continue;
                float a = 0.f;
                for (int jj = 0; jj < k; ++jj) {
                    const int32_t row = slot_row[t * k + jj];
                    if (row < 0)
                        continue;
                    int is = 0;
                    while (s_off[s_sel[is] + 1] <= row)
                        ++is;
                    a = fmaf(gw_in[t * k + jj], outs[is * 4 + (i & 3)][row - s_off[s_sel[is]]], a);
                }
                a *= scale;
                y[(int64_t)t * d + o] = __float2bfloat16_rn(a);
            }
        __syncthreads();
    }
}

// CTAs of a one-wave grid (one per SM; each fills its SM's registers).
static int dec_grid()
{
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 148;
    if (cached[dev] == 0) {
        int sms = 0;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = sms > 0 ? sms : 148;
    }
    return cached[dev];
}

static void dec_ws(const moe_params_t *p, char *ws, float **pre, int32_t **t_up, int32_t **t_dn)
{
    const WsLayout L = ws_layout(p);
    *pre = reinterpret_cast<float *>(ws + L.dpre);
    *t_up = reinterpret_cast<int32_t *>(ws + L.dtick);
    const int tm = p->T < kDecTok ? (p->T > 0 ? p->T : 1) : kDecTok;
    const int esel = p->E < tm * p->k ? p->E : tm * p->k;
    *t_dn = *t_up + (size_t)esel * (round_up(p->m, 16) / 16);
}

static cudaError_t up_launch(const moe_params_t *p, const void *x_rows, const int32_t *row_token,
                             void *x_perm_out, const int32_t *offsets, const void *W13, void *h,
                             char *ws, const void *W2_prefetch, cudaStream_t s)
{
    float *pre;
    int32_t *tu, *td;
    dec_ws(p, ws, &pre, &tu, &td);
    const dim3 grid(dec_grid());
    const bf16 *xr = (const bf16 *)x_rows, *w13 = (const bf16 *)W13, *w2 = (const bf16 *)W2_prefetch;
    bf16 *xo = (bf16 *)x_perm_out, *hh = (bf16 *)h;
    const dim3 rb(kRbWarps * 32);
    if (p->T <= 1)
        launch_pdl(decode_up_rows_kernel<1>, grid, rb, 0, s, xr, row_token, xo, offsets, w13, p->d,
                   p->m, p->E, hh, w2);
    else if (p->T <= 2)
        launch_pdl(decode_up_rows_kernel<2>, grid, rb, 0, s, xr, row_token, xo, offsets, w13, p->d,
                   p->m, p->E, hh, w2);
    else if (p->T <= 4)
        launch_pdl(decode_up_rows_kernel<4>, grid, rb, 0, s, xr, row_token, xo, offsets, w13, p->d,
                   p->m, p->E, hh, w2);
    else if (p->T <= kRbMaxTok)
        launch_pdl(decode_up_rows_kernel<8>, grid, rb, 0, s, xr, row_token, xo, offsets, w13, p->d,
                   p->m, p->E, hh, w2);
    else
        launch_pdl(decode_up_kernel<2, 12>, grid, dim3(12 * 32), 0, s, xr, row_token, xo, offsets,
                   w13, p->d, p->m, p->E, hh, pre, tu);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_up_decode(const moe_params_t *p, const void *x_perm, const int32_t *offsets,
                             const void *W13, void *h, char *ws, cudaStream_t s)
{
    return up_launch(p, x_perm, nullptr, nullptr, offsets, W13, h, ws, nullptr, s);
}

cudaError_t launch_up_decode_gather(const moe_params_t *p, const void *x, const int32_t *row_token,
                                    const int32_t *offsets, const void *W13, void *h,
                                    void *x_perm_out, char *ws, const void *W2_prefetch,
                                    cudaStream_t s)
{
    return up_launch(p, x, row_token, x_perm_out, offsets, W13, h, ws, W2_prefetch, s);
}

cudaError_t launch_down_decode(const moe_params_t *p, const void *h, const int32_t *offsets,
                               const void *W2, void *out, char *ws, cudaStream_t s,
                               const int32_t *slot_row, const float *topk_w, void *y)
{
    float *pre;
    int32_t *tu, *td;
    dec_ws(p, ws, &pre, &tu, &td);
    const float scale = p->rescale ? (float)p->E / (float)p->k : 1.0f;
    const dim3 grid(dec_grid());
    const bf16 *hh = (const bf16 *)h, *w2 = (const bf16 *)W2;
    bf16 *o = (bf16 *)out, *yy = (bf16 *)y;
    const dim3 rb(kRbWarps * 32);
    if (p->T <= 1)
        launch_pdl(decode_down_rows_kernel<1>, grid, rb, 0, s, hh, offsets, w2, p->d, p->m, p->E,
                   o, p->T, p->k, slot_row, topk_w, scale, yy);
    else if (p->T <= 2)
        launch_pdl(decode_down_rows_kernel<2>, grid, rb, 0, s, hh, offsets, w2, p->d, p->m, p->E,
                   o, p->T, p->k, slot_row, topk_w, scale, yy);
    else if (p->T <= 4)
        launch_pdl(decode_down_rows_kernel<4>, grid, rb, 0, s, hh, offsets, w2, p->d, p->m, p->E,
                   o, p->T, p->k, slot_row, topk_w, scale, yy);
    else if (p->T <= kRbMaxTok)
        launch_pdl(decode_down_rows_kernel<8>, grid, rb, 0, s, hh, offsets, w2, p->d, p->m, p->E,
                   o, p->T, p->k, slot_row, topk_w, scale, yy);
    else
        launch_pdl(decode_down_kernel<2, 12>, grid, dim3(12 * 32), 0, s, hh, offsets, w2, p->d,
                   p->m, p->E, o, pre, td, p->T, p->k, slot_row, topk_w, scale, yy);
    count_launch();
    return cudaGetLastError();
}

}  // namespace moe
