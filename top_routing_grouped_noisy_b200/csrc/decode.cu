// decode.cu -- the layer for decode-shaped bf16 batches (1 <= T <= 16 tokens).  The
// expert FFN then reads each selected expert's weights once and does little
// arithmetic per byte, so the layer is bound by streaming those weights from HBM.
// Router of "Llama 3 Meets MoE: Efficient Upcycling", section 3 "核心公式" (noisy
// Top-k routing, KeepTopK; section 5 for the Mixtral and ST routers); capacity
// dispatch of its section 3 "容量因子"; SwiGLU expert of "LLaMA-MoE v2", code
// sample "代码实现示例", class Expert; the combine y = sum_i G(x)_i E_i(x) of
// "Llama 3 Meets MoE", section 3; the balance loss of "LLaMA-MoE v2", section
// "门控机制设计".
//
// One kernel shape serves four modes:
//   route   (one CTA)  the router logits and the gate of every token (moe_route);
//   up      (grid)     GEMM 1 with the SwiGLU epilogue from x_perm (moe_expert_up);
//   down    (grid)     GEMM 2 (moe_expert_down);
//   forward (grid, cooperative launch: every CTA resident)  the whole layer in one
//           launch.  Every CTA computes the logits and the gate itself (x and
//           [W_g | W_noise] are a few ten KB, read from L2 by all but the first
//           CTA), so no CTA waits for a router CTA; CTA 0 alone writes the routing,
//           the dispatch tables and the gate statistics.  Then GEMM 1, a grid
//           barrier (h complete), GEMM 2, and the combine of the output columns
//           each CTA owns.
//
// Weight streaming.  Warp 0 is the loader: it walks the CTA's work items and copies
// their weight rows with untiled bulk copies (cp.async.bulk) into a ring of stages
// (one mbarrier pair per stage), each lane issuing one copy so that the copies of a
// stage go out together.  A copy moves a 4 KB row chunk, or a run of consecutive
// whole rows at once: an SM's bulk-copy engine spends a roughly fixed time per copy,
// so copies of 1-2 KB cannot keep up with the SM's share of HBM bandwidth.  The
// ring spans ~130-200 KB and the loader runs ahead across the grid barrier: GEMM 2's
// weights stream in while GEMM 1 finishes elsewhere.
// Warps 1..8 multiply: a stage's rows are the A operand of mma.sync m16n8k16 (bf16
// in, f32 out), the expert's token rows (at most 16, in shared memory) are B.  Lane
// (g, c) loads 8 consecutive K of A rows g (and g + 8) and of B row g; the two mma
// of a 32-column step take those 8 K in the same order for A and B, so the product
// is the plain dot product with K permuted inside the step.  A warp issues every
// fragment load of a stage before its first mma (the loop is bound by shared-memory
// latency otherwise).  Warp w takes the 32-column steps s = w, w + 8, ... of every
// row and the 8 warps' sums are added in warp order: the order depends only on the
// column index, so the sums do not depend on the grid, the ring depth or which CTA
// owns a row.
//   GEMM 1 item: up to 8 neurons of one expert; a stage holds their W1 rows (A rows
//                0..7) and W3 rows (A rows 8..15) for 2048 columns, so one lane ends
//                with g and u of a neuron and writes h = silu(g) * u (bf16).
//   GEMM 2 item: up to 8 output columns of one expert (8 W2 rows, A rows 0..7).
// Balance: GEMM 1 splits the selected experts' neurons evenly over the CTAs and
// GEMM 2 their output columns, so every SM streams the same bytes within a row.
#include <type_traits>

#include "common.cuh"
#include "gate.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace moe {

using tc::bulk_load;
using tc::mbar_arrive;
using tc::mbar_drain;
using tc::mbar_expect_tx;
using tc::mbar_init;
using tc::mbar_wait;
using tc::smem_u32;

enum : int { kDsRoute = 1, kDsUp = 2, kDsDown = 4, kDsForward = 8 };

constexpr int kDsCw = 8;                     // multiplying warps (1..8); warp 0 loads
constexpr int kDsThreads = 32 * (kDsCw + 1);
// GEMM 1: K columns per stage (16 rows): 2048 (4 KB copies) where two such stages fit
// beside the rest, else 1024
constexpr int kDsKc1 = 2048, kDsKc1Small = 1024;
constexpr int kDsKc2 = 2048;                 // GEMM 2: K columns per stage (8 rows)
constexpr int kDsRows = 8;                   // neurons (GEMM 1) or output columns (GEMM 2) per item
constexpr int kDsMaxStages = 16;
constexpr int kDsMinStages = 2;
constexpr int kDsBarBytes = 512;                     // full[16], empty[16], x, W
// two buffers of the warps' sums, 4 NB floats per lane
__host__ __device__ constexpr int ds_red_bytes(int nb) { return 2 * kDsCw * 32 * 4 * nb * 4; }
constexpr int kDsRouterRed = kDsCw * 16 * 32 * 4;    // the warps' partial logits
constexpr int kDsRouterLg = 16 * 32 * 4;             // logits [T][nout]
constexpr int kDsRouterGate = 2 * 16 * 32 * 4;       // gate scratch [T][E] x 2
constexpr int kDsRouterScratch = kDsRouterRed + kDsRouterLg + kDsRouterGate;
constexpr size_t kDsSmemCap = 222 * 1024;            // dynamic (the static tables apart)
constexpr int kDsMaxRows = kDecodeMaxTokens * MOE_MAX_TOPK;

// Staged row pitch (bytes) of a matrix with K columns: whole rows as they lie in
// memory (runs of rows copied at once) when K fits a stage of kc columns, else
// chunks of kc columns with a 16-byte pad (16 mod 128: conflict-free fragment loads).
__host__ __device__ inline int ds_pitch(int K, int kc) { return K <= kc ? 2 * K : 2 * kc + 16; }

struct DsArgs {
    const bf16 *x;              // [T][d]       route, forward
    const bf16 *x_perm;         // [R][d]       up
    const bf16 *Wg, *Wn;        // [d][E]       route, forward (Wn may be NULL)
    const float *noise;         // [T][E]
    const float *bias;          // [E] or NULL
    const bf16 *W13;            // packed [E][2 m16][d]
    const bf16 *W2;             // packed [E][d][m8]
    const int32_t *offsets_in;  // [E+1]        up, down
    const bf16 *h_in;           // [R][m8]      down
    int32_t *idx;               // [T][k]       route, forward
    float *w;                   // [T][k]
    float *probs_sum, *importance;                            // [E]
    int32_t *counts, *kept, *offsets, *row_token, *slot_row;  // forward
    float *f, *P, *loss;                                      // forward
    bf16 *x_perm_out;           // forward
    bf16 *h;                    // [R][m8]      up, forward
    bf16 *out;                  // [R][d]       down, forward
    bf16 *y;                    // [T][d]       forward
    int32_t *status;
    int32_t *gbar;              // grid barrier: arrival count (zero between calls), generation
    uint64_t wait_ns;
    float lambda, scale;
    int T, d, m, E, k, C, router_type;
    int stages, stage_bytes, bpitch, hpitch, bbytes, obytes, kc1;
    int split13;  // GEMM 1 stages of 8 rows (W1 rows, then W3 rows) instead of 16
};

__device__ __forceinline__ uint4 lds128(const char *p) { return *reinterpret_cast<const uint4 *>(p); }

// barrier of the multiplying warps (named barrier 1, warps 1..8)
__device__ __forceinline__ void cw_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kDsCw * 32) : "memory"); }

__device__ __forceinline__ uint32_t lds32_s(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t bf16_pair_s(const bf16 *lo, const bf16 *hi)
{
    return (uint32_t)__bfloat16_as_ushort(*lo) | ((uint32_t)__bfloat16_as_ushort(*hi) << 16);
}

// --------------------------------------------------------------------- work items
// GEMM 1: neurons [c N1 / G, (c+1) N1 / G) of the selected experts' nsel * m
// neurons (expert-major), cut into items of at most 8 neurons of one expert, each
// once per group of at most rg rows of that expert: f(e, j0, nv, r0, nr).
template <class F>
__device__ __forceinline__ void ds_walk_up(int nsel, const int32_t *s_sel, const int32_t *s_off,
                                           int m, int rg, F f)
{
    const int64_t N1 = (int64_t)nsel * m;
    int64_t n = (int64_t)blockIdx.x * N1 / gridDim.x;
    const int64_t n_hi = (int64_t)(blockIdx.x + 1) * N1 / gridDim.x;
    while (n < n_hi) {
        const int is = (int)(n / m), j0 = (int)(n - (int64_t)is * m);
        const int nv = (int)min((int64_t)min(kDsRows, m - j0), n_hi - n);
        const int e = s_sel[is], r0 = s_off[e], nr = s_off[e + 1] - r0;
        for (int g0 = 0; g0 < nr; g0 += rg)
            f(e, j0, nv, r0 + g0, min(rg, nr - g0));
        n += nv;
    }
}

// GEMM 2: output columns [c d / G, (c+1) d / G) of every selected expert, items of
// at most 8 columns, each once per group of at most rg rows: f(e, oc, nv, r0, nr).
template <class F>
__device__ __forceinline__ void ds_walk_down(int nsel, const int32_t *s_sel, const int32_t *s_off,
                                             int d, int rg, F f)
{
    const int o_lo = (int)((int64_t)blockIdx.x * d / gridDim.x);
    const int o_hi = (int)((int64_t)(blockIdx.x + 1) * d / gridDim.x);
    for (int is = 0; is < nsel; ++is) {
        const int e = s_sel[is], r0 = s_off[e], nr = s_off[e + 1] - r0;
        for (int oc = o_lo; oc < o_hi; oc += kDsRows)
            for (int g0 = 0; g0 < nr; g0 += rg)
                f(e, oc, min(kDsRows, o_hi - oc), r0 + g0, min(rg, nr - g0));
    }
}

// --------------------------------------------------------------------- the ring
struct DsRing {
    char *base;
    uint64_t *full, *empty;
    int stages, stage_bytes;
    int it;      // stages handed out (loader) or taken (multiplying warps) so far
    int issued;  // loader: stages whose copies were issued (all of them, or up to an abort)
};

// Loader (all lanes of warp 0): waits until the next stage is free, then copies
// `nrows` (<= 32) rows of `len` columns of a matrix with K columns (row i from
// global row(i), column k0 on, to stage row slot(i)) at `pitch`
// (ds_pitch(K, kc)): a run of consecutive whole rows into consecutive stage rows
// in one copy, else one copy per row; lane i issues the copy that starts at row i,
// so the copies of a stage go out together.
template <class RowPtr, class Slot>
__device__ __forceinline__ void ds_issue(DsRing &r, int nrows, int len, int K, int pitch,
                                         RowPtr row, Slot slot, const DsArgs &a,
                                         volatile int32_t *abort_flag)
{
    const int lane = threadIdx.x & 31;
    const int s = r.it % r.stages;
    const uint32_t use = (uint32_t)(r.it / r.stages);
    ++r.it;
    bool go = true;
    if (lane == 0) {
        if (use > 0)
            go = mbar_wait(smem_u32(&r.empty[s]), (use - 1) & 1, a.wait_ns, abort_flag, a.status);
        go = go && !*abort_flag;
        if (go)
            mbar_expect_tx(smem_u32(&r.full[s]), (uint32_t)(nrows * len * 2));
    }
    if (!__shfl_sync(0xffffffffu, go ? 1 : 0, 0))
        return;
    const uint32_t bar = smem_u32(&r.full[s]);
    char *st = r.base + (size_t)s * r.stage_bytes;
    if (lane < nrows) {
        const bf16 *p = row(lane);
        const int sl = slot(lane);
        if (len == K) {  // whole rows: lane i copies the run of consecutive rows from i
            if (lane == 0 || row(lane - 1) + K != p || slot(lane - 1) + 1 != sl) {
                int n = 1;
                while (lane + n < nrows && row(lane + n) == p + (size_t)n * K &&
                       slot(lane + n) == sl + n)
                    ++n;
                bulk_load(smem_u32(st + (size_t)sl * pitch), p, (uint32_t)(n * K * 2), bar);
            }
        } else {
            bulk_load(smem_u32(st + (size_t)sl * pitch), p, (uint32_t)(len * 2), bar);
        }
    }
    r.issued = r.it;
}

// Loader, on exit: waits for the copies of the last stages issued (only after an
// abort can some still be in flight).
__device__ __forceinline__ void ds_drain(const DsRing &r)
{
    for (int i = r.issued > r.stages ? r.issued - r.stages : 0; i < r.issued; ++i)
        mbar_drain(smem_u32(&r.full[i % r.stages]), (uint32_t)(i / r.stages) & 1);
}

// --------------------------------------------------------------------- the multiply
__device__ __forceinline__ uint4 lds128_s(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

// acc[.][nb] += A * B over this warp's 32-column steps of a stage: A rows 0..7 are
// the stage's rows at `pitch` from st, and with ROWS16 rows 8..15 those from st8 (the
// next 8 rows of the same stage, or the rows of a second stage); `len` columns; B at
// the shared addresses bp[nb] of this lane's B row (0 for none), columns k0 + ....
// Even steps add into acc[0], odd ones into acc[1] (two independent mma chains; the
// split depends only on the column index).  Every fragment load of the stage is
// issued before the first mma: the loop is bound by shared-memory latency otherwise.
template <int NB, int KS, bool ROWS16>
__device__ __forceinline__ void ds_stage_mma(float (&acc)[2][NB][4], uint32_t st, uint32_t st8,
                                             int pitch, int len, int k0,
                                             const uint32_t (&bp)[NB], int cw, int g, int c)
{
    const uint4 zero = make_uint4(0, 0, 0, 0);
    const uint32_t arow = st + (uint32_t)(g * pitch + 16 * c);
    const uint32_t arow8 = st8 + (uint32_t)(g * pitch + 16 * c);
    uint4 A[KS], A8[KS], B[KS][NB];
#pragma unroll
    for (int j = 0; j < KS; ++j) {
        const int kk = (cw + j * kDsCw) * 32;
        const bool valid = kk + 8 * c < len;  // len is a multiple of 8
        A[j] = valid ? lds128_s(arow + kk * 2) : zero;
        A8[j] = (ROWS16 && valid) ? lds128_s(arow8 + kk * 2) : zero;
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
            B[j][nb] = (valid && bp[nb] != 0u) ? lds128_s(bp[nb] + (uint32_t)(k0 + kk) * 2) : zero;
    }
#pragma unroll
    for (int j = 0; j < KS; ++j)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            mma_bf16_16816(acc[j & 1][nb], A[j].x, A8[j].x, A[j].y, A8[j].y, B[j][nb].x,
                           B[j][nb].y);
            mma_bf16_16816(acc[j & 1][nb], A[j].z, A8[j].z, A[j].w, A8[j].w, B[j][nb].z,
                           B[j][nb].w);
        }
}

// Copies rows [0, n) of the B region (pitch bp) from global rows src(j) (ncols bf16
// in 16-byte vectors, read at L2), zeroing columns >= valid.  Called by the
// multiplying warps between two cw_sync().
template <class Src>
__device__ __forceinline__ void ds_load_rows(char *breg, int bp, int n, int ncols, int valid,
                                             Src src, int ct)
{
    const int nv8 = ncols / 8;
    const int total = n * nv8;
    constexpr int U = 4;
    for (int i0 = ct; i0 < total; i0 += U * kDsCw * 32) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * kDsCw * 32;
            v[u] = i < total ? __ldcg(reinterpret_cast<const uint4 *>(src(i / nv8)) + i % nv8)
                             : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * kDsCw * 32;
            if (i >= total)
                continue;
            const int j = i / nv8, col0 = (i % nv8) * 8;
            if (col0 + 8 > valid) {
                uint16_t *hv = reinterpret_cast<uint16_t *>(&v[u]);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (col0 + q >= valid)
                        hv[q] = 0;
            }
            *reinterpret_cast<uint4 *>(breg + (size_t)j * bp + col0 * 2) = v[u];
        }
    }
}

// --------------------------------------------------------------------- the router
// Logits lg[T][nout] of the T tokens whose rows sit in the B region (pitch bp)
// against [W_g | W_noise], staged through `wst` in rounds of kr rows (kr a multiple
// of 256); round 0 was issued by the caller.  Warp w (1..8) takes the 16-column
// steps s = w-1, w-1 + 8, ..., alternating two accumulators; the warps' partial sums
// are added in warp order -- the same bits whatever kr is.  Called by every thread.
template <int NT>
__device__ void ds_router_logits(const char *breg, int bp, const DsArgs &a, char *wst, int kr,
                                 float *red, float *lg, uint64_t *wbar,
                                 volatile int32_t *abort_flag)
{
    const int T = a.T, d = a.d, E = a.E;
    const int nout = a.Wn != nullptr ? 2 * E : E;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const bf16 *gs = reinterpret_cast<const bf16 *>(wst);
    const bf16 *ns = gs + (size_t)kr * E;
    float acc[2][NT][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q)
                acc[h][nt][q] = 0.f;
    int round = 0, last_issued = 0;
    for (int k0 = 0; k0 < d; k0 += kr, ++round) {
        const int kc = min(kr, d - k0);
        if (round > 0 && threadIdx.x == 0 && !*abort_flag) {
            last_issued = round;
            tc::fence_proxy_async_smem();  // after the previous round's reads
            const uint32_t bar = smem_u32(wbar);
            const uint32_t bytes = (uint32_t)kc * E * 2;
            mbar_expect_tx(bar, a.Wn != nullptr ? 2 * bytes : bytes);
            bulk_load(smem_u32(wst), a.Wg + (size_t)k0 * E, bytes, bar);
            if (a.Wn != nullptr)
                bulk_load(smem_u32(ns), a.Wn + (size_t)k0 * E, bytes, bar);
        }
        const bool ok = mbar_wait(smem_u32(wbar), round & 1, a.wait_ns, abort_flag, a.status);
        if (warp >= 1 && ok) {
            // groups of 4 steps: every load of a group before its mma (even steps
            // into acc[0], odd ones into acc[1]; kr is a multiple of 256)
            const uint32_t xs = smem_u32(breg), gsa = smem_u32(gs), nsa = smem_u32(ns);
            const bool vec = (E & 7) == 0;  // rows of 8 experts 16-byte aligned: ldmatrix
            for (int kb = k0 + (warp - 1) * 16; kb < k0 + kc; kb += 4 * 16 * kDsCw) {
                uint32_t A[4][4], B[4][NT][2];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int kk = kb + j * 16 * kDsCw;
                    const bool in = kk < k0 + kc;
                    const bool hi = in && kk + 8 < d;  // d % 8 == 0: 8 more columns or none
                    const uint32_t x0 = xs + (uint32_t)(g * bp + (kk + 2 * c) * 2);
                    const uint32_t x1 = x0 + (uint32_t)(8 * bp);
                    A[j][0] = (in && g < T) ? lds32_s(x0) : 0u;
                    A[j][1] = (in && g + 8 < T) ? lds32_s(x1) : 0u;
                    A[j][2] = (hi && g < T) ? lds32_s(x0 + 16) : 0u;
                    A[j][3] = (hi && g + 8 < T) ? lds32_s(x1 + 16) : 0u;
                    const int r = kk - k0 + 2 * c;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        B[j][nt][0] = B[j][nt][1] = 0u;
                        if (!in || nt * 8 >= nout)
                            continue;
                        if (vec) {
                            // rows kk - k0 + 0..15 of the 8 experts of this tile, transposed
                            const bool noise_tile = nt * 8 >= E;
                            const uint32_t base = noise_tile ? nsa : gsa;
                            const int col = noise_tile ? nt * 8 - E : nt * 8;
                            const int row = kk - k0 + (lane & 15);
                            uint32_t b0, b1;
                            ldsm_x2_trans(base + (uint32_t)((row * E + col) * 2), b0, b1);
                            B[j][nt][0] = b0;
                            B[j][nt][1] = hi ? b1 : 0u;
                        } else {
                            const int n = nt * 8 + g;
                            const bf16 *src = n < E ? gs + n : (n < nout ? ns + (n - E) : nullptr);
                            if (src != nullptr) {
                                B[j][nt][0] =
                                    bf16_pair_s(src + (size_t)r * E, src + (size_t)(r + 1) * E);
                                if (hi)
                                    B[j][nt][1] = bf16_pair_s(src + (size_t)(r + 8) * E,
                                                              src + (size_t)(r + 9) * E);
                            }
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (kb + j * 16 * kDsCw >= k0 + kc)
                        break;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_bf16_16816(acc[j & 1][nt], A[j][0], A[j][1], A[j][2], A[j][3],
                                       B[j][nt][0], B[j][nt][1]);
                }
            }
        }
        __syncthreads();
    }
    if (threadIdx.x == 0)  // copies still in flight after an abort
        mbar_drain(smem_u32(wbar), (uint32_t)last_issued & 1);
    constexpr int NP = NT * 8;
    if (warp >= 1) {
        float *rw = red + (size_t)(warp - 1) * 16 * NP;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int n = nt * 8 + 2 * c;
            rw[g * NP + n] = acc[0][nt][0] + acc[1][nt][0];
            rw[g * NP + n + 1] = acc[0][nt][1] + acc[1][nt][1];
            rw[(g + 8) * NP + n] = acc[0][nt][2] + acc[1][nt][2];
            rw[(g + 8) * NP + n + 1] = acc[0][nt][3] + acc[1][nt][3];
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < T * nout; i += blockDim.x) {
        const int t = i / nout, o = i % nout;
        float sum = 0.f;
        for (int w = 0; w < kDsCw; ++w)
            sum += red[((size_t)w * 16 + t) * NP + o];
        lg[i] = sum;
    }
    __syncthreads();
}

// The gate of every token (gate_token_warp, one warp per token; E <= 32), then the
// token sums probs_sum, importance in token order.  gsm: [T][E] probabilities, then
// [T][E] gate weights.  Called by every thread of the CTA.
__device__ void ds_gate(const float *lg, const DsArgs &a, int32_t *idx_out, float *w_out,
                        float *probs_sum, float *importance, float *gsm)
{
    const int T = a.T, E = a.E, k = a.k;
    const int noisy = a.Wn != nullptr ? 1 : 0, nout = noisy ? 2 * E : E;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    float *prob_s = gsm, *gw_s = gsm + (size_t)T * E;
    for (int t = warp; t < T; t += nwarps) {
        const float *l = lg + (size_t)t * nout;
        const bool on = lane < E;
        float h = 0.f;
        if (on) {
            h = l[lane];
            if (a.bias)
                h += a.bias[lane];
            if (noisy)
                h += a.noise[(size_t)t * E + lane] * softplus_f(l[E + lane]);
        }
        const bool bad = __any_sync(0xffffffffu, on && !isfinite(h));
        if (bad) {
            if (lane == 0)
                set_status(a.status, MOE_ERR_DEVICE_BADINDEX);
            if (lane < k) {
                idx_out[t * k + lane] = -1;
                w_out[t * k + lane] = 0.f;
            }
            if (on) {
                prob_s[t * E + lane] = 0.f;
                gw_s[t * E + lane] = 0.f;
            }
            continue;
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
        if (a.router_type == MOE_ROUTER_MIXTRAL) {
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
            prob_s[t * E + lane] = p;
            gw_s[t * E + lane] = taken ? wsel : 0.f;
        }
#pragma unroll
        for (int j = 0; j < MOE_MAX_TOPK; ++j) {
            if (j >= k)
                break;
            const float wj = __shfl_sync(0xffffffffu, wsel, sel[j]);
            if (lane == j) {
                idx_out[t * k + j] = sel[j];
                w_out[t * k + j] = wj;
            }
        }
    }
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

// --------------------------------------------------------------------- the kernel
template <int NB, int MODE>
__global__ void __launch_bounds__(kDsThreads, 1) decode_stream_kernel(const __grid_constant__ DsArgs a)
{
    extern __shared__ __align__(128) char sm[];
    __shared__ int32_t s_off[MOE_MAX_EXPERTS + 1], s_sel[MOE_MAX_EXPERTS];
    __shared__ int32_t s_cnt[MOE_MAX_EXPERTS], s_kept[MOE_MAX_EXPERTS];
    __shared__ int32_t s_idx[kDsMaxRows], s_slot[kDsMaxRows], s_rtok[kDsMaxRows];
    __shared__ float s_w[kDsMaxRows], s_psum[MOE_MAX_EXPERTS], s_imp[MOE_MAX_EXPERTS];
    __shared__ int s_nsel;
    __shared__ int32_t s_abort_mem;
    volatile int32_t *abort_flag = &s_abort_mem;

    constexpr int RG = 8 * NB;  // token rows of one B group
    constexpr bool kUp = (MODE & (kDsUp | kDsForward)) != 0;
    constexpr bool kDown = (MODE & (kDsDown | kDsForward)) != 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm);
    float *red = reinterpret_cast<float *>(sm + kDsBarBytes);
    char *breg = sm + kDsBarBytes + ds_red_bytes(NB);
    float *outs = reinterpret_cast<float *>(breg + a.bbytes);  // forward: rounded out values
    DsRing ring{breg + a.bbytes + a.obytes, bars, bars + kDsMaxStages, a.stages, a.stage_bytes,
                0, 0};
    uint64_t *xbar = bars + 2 * kDsMaxStages, *wbar = xbar + 1;
    const int bp = a.bpitch;
    if (threadIdx.x == 0) {
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(smem_u32(&ring.full[s]), 1);
            mbar_init(smem_u32(&ring.empty[s]), kDsCw);
        }
        mbar_init(smem_u32(xbar), 1);
        mbar_init(smem_u32(wbar), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    pdl_wait();
    const int T = a.T, E = a.E, k = a.k, m = a.m, d = a.d;
    const int m8 = round_up(m, 8), m16 = round_up(m, 16);
    // forward: the grid barrier's generation before this launch's barrier (it changes
    // only once every CTA has arrived, this one included)
    int32_t gen = 0;
    if constexpr (MODE == kDsForward)
        if (threadIdx.x == 32)
            gen = ld_acquire_gpu(a.gbar + 1);

    if constexpr ((MODE & (kDsRoute | kDsForward)) != 0) {
        // ---- router: the token rows of x into the B region and the first round of
        // [W_g | W_noise] into the ring, both in flight at once; logits; gate
        const int nout = a.Wn != nullptr ? 2 * E : E;
        const int ring_bytes = a.stages * a.stage_bytes;
        char *scratch = ring.base + ring_bytes - kDsRouterScratch;
        float *rred = reinterpret_cast<float *>(scratch);
        float *lg = reinterpret_cast<float *>(scratch + kDsRouterRed);
        float *gsm = reinterpret_cast<float *>(scratch + kDsRouterRed + kDsRouterLg);
        int kr = (ring_bytes - kDsRouterScratch) / (nout * 2) / 256 * 256;
        kr = min(kr, round_up(d, 256));
        if (threadIdx.x == 0) {
            const uint32_t xb = smem_u32(xbar);
            mbar_expect_tx(xb, (uint32_t)(T * d * 2));
            for (int t = 0; t < T; ++t)
                bulk_load(smem_u32(breg + (size_t)t * bp), a.x + (size_t)t * d, (uint32_t)d * 2,
                          xb);
            const uint32_t wb = smem_u32(wbar);
            const uint32_t bytes = (uint32_t)min(kr, d) * E * 2;
            mbar_expect_tx(wb, a.Wn != nullptr ? 2 * bytes : bytes);
            bulk_load(smem_u32(ring.base), a.Wg, bytes, wb);
            if (a.Wn != nullptr)
                bulk_load(smem_u32(ring.base + (size_t)kr * E * 2), a.Wn, bytes, wb);
        }
        if (!mbar_wait(smem_u32(xbar), 0, a.wait_ns, abort_flag, a.status) && threadIdx.x == 0)
            mbar_drain(smem_u32(xbar), 0);
        switch ((nout + 7) / 8) {
        case 1: ds_router_logits<1>(breg, bp, a, ring.base, kr, rred, lg, wbar, abort_flag); break;
        case 2: ds_router_logits<2>(breg, bp, a, ring.base, kr, rred, lg, wbar, abort_flag); break;
        case 3: ds_router_logits<3>(breg, bp, a, ring.base, kr, rred, lg, wbar, abort_flag); break;
        default: ds_router_logits<4>(breg, bp, a, ring.base, kr, rred, lg, wbar, abort_flag); break;
        }
        if constexpr (MODE == kDsRoute) {
            ds_gate(lg, a, a.idx, a.w, a.probs_sum, a.importance, gsm);
            pdl_trigger();
            return;
        } else {
            ds_gate(lg, a, s_idx, s_w, s_psum, s_imp, gsm);
            __syncthreads();
            // ---- the dispatch tables (those of the count and scatter kernels:
            // stable by token, assignments past the capacity dropped)
            for (int e = threadIdx.x; e < E; e += blockDim.x) {
                int cnt = 0;
                for (int i = 0; i < T * k; ++i)
                    cnt += s_idx[i] == e;
                s_cnt[e] = cnt;
                s_kept[e] = a.C < 0 ? cnt : min(cnt, a.C);
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                int acc = 0, ns = 0;
                for (int e = 0; e < E; ++e) {
                    s_off[e] = acc;
                    acc += s_kept[e];
                    if (s_kept[e] > 0)
                        s_sel[ns++] = e;
                }
                s_off[E] = acc;
                s_nsel = ns;
            }
            __syncthreads();
            for (int i = threadIdx.x; i < T * k; i += blockDim.x) {
                const int t = i / k, e = s_idx[i];
                int row = -1;
                if (e < 0 || e >= E) {
                    set_status(a.status, MOE_ERR_DEVICE_BADINDEX);
                } else {
                    int rank = 0;  // the expert's assignments of earlier tokens
                    for (int i2 = 0; i2 < t * k; ++i2)
                        rank += s_idx[i2] == e;
                    if (rank < s_kept[e]) {
                        row = s_off[e] + rank;
                        s_rtok[row] = t;
                    }
                }
                s_slot[i] = row;
            }
            __syncthreads();
        }
    } else {
        // ---- step calls: the dispatch tables from offsets
        for (int e = threadIdx.x; e <= E; e += blockDim.x)
            s_off[e] = __ldcg(a.offsets_in + e);
        __syncthreads();
        if (threadIdx.x == 0) {
            int ns = 0;
            for (int e = 0; e < E; ++e)
                if (s_off[e + 1] > s_off[e])
                    s_sel[ns++] = e;
            s_nsel = ns;
        }
        __syncthreads();
    }
    const int nsel = s_nsel;
    const int kc1 = a.kc1, pitch1 = ds_pitch(d, kc1), pitch2 = ds_pitch(m8, kDsKc2);

    if (warp == 0) {
        // ---------------------------------------------------------------- loader
        {
            tc::fence_proxy_async_smem();  // the router's reads of the ring come first
            if constexpr (kUp) {
                ds_walk_up(nsel, s_sel, s_off, m, RG, [&](int e, int j0, int nv, int, int) {
                    const bf16 *base = a.W13 + (size_t)e * 2 * m16 * d;
                    for (int k0 = 0; k0 < d; k0 += kc1) {
                        if (a.split13) {  // a stage of W1 rows, then one of W3 rows
                            for (int half = 0; half < 2; ++half)
                                ds_issue(
                                    ring, nv, min(kc1, d - k0), d, pitch1,
                                    [&](int i) {
                                        const int n = j0 + i;
                                        const int row = (n >> 4) * 32 + (n & 15) + 16 * half;
                                        return base + (size_t)row * d + k0;
                                    },
                                    [&](int i) { return i; }, a, abort_flag);
                        } else {  // W1 rows to stage rows 0.., W3 rows to 8..
                            ds_issue(
                                ring, 2 * nv, min(kc1, d - k0), d, pitch1,
                                [&](int i) {
                                    const int n = j0 + (i < nv ? i : i - nv);
                                    const int row = (n >> 4) * 32 + (n & 15) + (i < nv ? 0 : 16);
                                    return base + (size_t)row * d + k0;
                                },
                                [&](int i) { return i < nv ? i : 8 + i - nv; }, a, abort_flag);
                        }
                    }
                });
            }
            if constexpr (kDown) {
                ds_walk_down(nsel, s_sel, s_off, d, RG, [&](int e, int oc, int nv, int, int) {
                    const bf16 *base = a.W2 + ((size_t)e * d + oc) * m8;
                    for (int k0 = 0; k0 < m8; k0 += kDsKc2)
                        ds_issue(
                            ring, nv, min(kDsKc2, m8 - k0), m8, pitch2,
                            [&](int i) { return base + (size_t)i * m8 + k0; },
                            [&](int i) { return i; }, a, abort_flag);
                });
            }
            ds_drain(ring);
        }
    } else {
        // ---------------------------------------------------------------- multiply
        const int cw = warp - 1, ct = threadIdx.x - 32, g = lane >> 2, c = lane & 3;
        int rb = 0;
        int loaded = -1;  // first row of the expert rows held in the B region
        const uint32_t ring_s = smem_u32(ring.base), breg_s = smem_u32(breg);
        int ss = 0;          // the ring stage taken next
        uint32_t phase = 0;  // its phase parity
        // Takes the next stage of the ring (GEMM 1 with paired 8-row stages: the next two,
        // W1 rows then W3 rows) and adds its rows * B into acc.  kind: 2 = GEMM 1 with
        // 16-row stages of kc1 columns, 1 = GEMM 1 with paired 8-row stages, 0 = GEMM 2
        // (8 rows, kDsKc2 columns).
        auto take_stage = [&](auto kind, float (&acc)[2][NB][4], int pitch, int len, int k0,
                              const uint32_t (&bpt)[NB]) {
            constexpr int KIND = decltype(kind)::value;
            constexpr int NS = KIND == 1 ? 2 : 1;
            int sl[NS];
            bool ok = true;
#pragma unroll
            for (int i = 0; i < NS; ++i) {
                sl[i] = ss;
                ok = ok && mbar_wait(smem_u32(&ring.full[ss]), phase, a.wait_ns, abort_flag,
                                     a.status);
                if (++ss == ring.stages) {
                    ss = 0;
                    phase ^= 1u;
                }
            }
            const uint32_t st = ring_s + (uint32_t)(sl[0] * ring.stage_bytes);
            const uint32_t st8 = KIND == 1 ? ring_s + (uint32_t)(sl[NS - 1] * ring.stage_bytes)
                                           : st + (uint32_t)(8 * pitch);
            if (ok) {
                if constexpr (KIND > 0) {
                    if (kc1 == kDsKc1)
                        ds_stage_mma<NB, kDsKc1 / (32 * kDsCw), true>(acc, st, st8, pitch, len, k0,
                                                                      bpt, cw, g, c);
                    else
                        ds_stage_mma<NB, kDsKc1Small / (32 * kDsCw), true>(acc, st, st8, pitch,
                                                                           len, k0, bpt, cw, g, c);
                } else
                    ds_stage_mma<NB, kDsKc2 / (32 * kDsCw), false>(acc, st, st8, pitch, len, k0,
                                                                   bpt, cw, g, c);
            }
            __syncwarp();
            if (lane == 0)
#pragma unroll
                for (int i = 0; i < NS; ++i)
                    mbar_arrive(smem_u32(&ring.empty[sl[i]]));
        };
        // The warps' sums of an item: v[0..nv) into red, then epi(sum) with sum(L, q)
        // = value q of lane L added over the warps in warp order.
        auto reduce = [&](const float *v, int nv, auto epi) {
            constexpr int RS = 4 * NB;  // floats per lane
            float *rw = red + (size_t)rb * kDsCw * 32 * RS + ((size_t)cw * 32 + lane) * RS;
            for (int q = 0; q < nv; ++q)
                rw[q] = v[q];
            cw_sync();
            const float *rr = red + (size_t)rb * kDsCw * 32 * RS;
            epi([&](int L, int q) {
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < kDsCw; ++w)
                    sum += rr[((size_t)w * 32 + L) * RS + q];
                return sum;
            });
            rb ^= 1;
        };

        if constexpr (kUp) {
            ds_walk_up(nsel, s_sel, s_off, m, RG, [&](int, int j0, int nv, int r0, int nr) {
                uint32_t bpt[NB];
                if constexpr (MODE == kDsUp) {
                    if (loaded != r0) {  // this item's rows of x_perm into the B region
                        cw_sync();
                        ds_load_rows(breg, bp, nr, d, d,
                                     [&](int j) { return a.x_perm + (size_t)(r0 + j) * d; }, ct);
                        cw_sync();
                        loaded = r0;
                    }
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) {
                        const int j = nb * 8 + g;
                        bpt[nb] = j < nr ? breg_s + (uint32_t)(j * bp + 16 * c) : 0u;
                    }
                } else {  // forward: every token row of x is in the B region
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) {
                        const int j = nb * 8 + g;
                        bpt[nb] = j < nr ? breg_s + (uint32_t)(s_rtok[r0 + j] * bp + 16 * c) : 0u;
                    }
                }
                // A row g is the W1 row of neuron g (acc 0, 1), row g + 8 its W3 row (acc 2, 3)
                float acc[2][NB][4];
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            acc[h][nb][q] = 0.f;
                for (int k0 = 0; k0 < d; k0 += kc1) {
                    if (a.split13)
                        take_stage(std::integral_constant<int, 1>(), acc, pitch1, min(kc1, d - k0),
                                   k0, bpt);
                    else
                        take_stage(std::integral_constant<int, 2>(), acc, pitch1, min(kc1, d - k0),
                                   k0, bpt);
                }
                float v[8];
#pragma unroll
                for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        v[nb * 4 + q] = acc[0][nb][q] + acc[1][nb][q];
                reduce(v, 4 * NB, [&](auto sum) {
                    for (int i = ct; i < 32 * 2 * NB; i += kDsCw * 32) {
                        const int L = i & 31, q = i >> 5, nb = q >> 1, jj = q & 1;
                        const int neuron = L >> 2, tok = nb * 8 + 2 * (L & 3) + jj;
                        if (neuron < nv && tok < nr) {
                            const float gv = sum(L, nb * 4 + jj), uv = sum(L, nb * 4 + 2 + jj);
                            a.h[(size_t)(r0 + tok) * m8 + j0 + neuron] =
                                __float2bfloat16_rn(__fdividef(gv, 1.0f + __expf(-gv)) * uv);
                        }
                    }
                });
            });
        }

        if constexpr (MODE == kDsForward) {
            // ---- h of every CTA complete: a grid barrier (its wait overlaps the loader
            // streaming GEMM 2's weights).  One thread arrives and waits; meanwhile the
            // others write x_perm and, in CTA 0, the routing, the tables and the gate
            // statistics (outputs that nothing in this launch reads).
            cw_sync();
            const int R = s_off[E];
            if (ct == 0) {
                const int G = (int)gridDim.x;
                __threadfence();  // this CTA's h, ordered before by the barrier above
                if (atomicAdd(a.gbar, 1) == G - 1) {  // the last to arrive releases the others
                    __threadfence();
                    atomicAdd(a.gbar + 1, 1);
                    asm volatile("red.relaxed.gpu.global.and.b32 [%0], 0;" ::"l"(a.gbar) : "memory");
                } else {
                    const uint64_t t0 = globaltimer_ns();
                    while (!*abort_flag && ld_acquire_gpu(a.gbar + 1) == gen) {
                        if (globaltimer_ns() - t0 > a.wait_ns) {
                            set_status(a.status, MOE_ERR_DEVICE_TIMEOUT);
                            *abort_flag = 1;
                            break;
                        }
                        __nanosleep(32);
                    }
                }
            } else {
                const int nt = kDsCw * 32 - 1, t1 = ct - 1;
                for (int r = blockIdx.x; r < R; r += gridDim.x)
                    for (int v = t1; v < d / 8; v += nt)
                        st_v4(a.x_perm_out + (size_t)r * d + 8 * v,
                              ld_nc(a.x + (size_t)s_rtok[r] * d + 8 * v));
                if (blockIdx.x == 0) {
                    for (int i = t1; i < T * k; i += nt) {
                        a.idx[i] = s_idx[i];
                        a.w[i] = s_w[i];
                        a.slot_row[i] = s_slot[i];
                    }
                    for (int r = t1; r < R; r += nt)
                        a.row_token[r] = s_rtok[r];
                    for (int e = t1; e <= E; e += nt)
                        a.offsets[e] = s_off[e];
                    // the gate statistics, in gate_stats_kernel's arithmetic
                    for (int e = t1; e < E; e += nt) {
                        a.counts[e] = s_cnt[e];
                        a.kept[e] = s_kept[e];
                        a.probs_sum[e] = s_psum[e];
                        a.importance[e] = s_imp[e];
                        a.f[e] = (float)((double)s_cnt[e] / ((double)T * k));
                        a.P[e] = (float)((double)s_psum[e] / (double)T);
                    }
                    if (t1 == nt - 1) {
                        double sfp = 0.0;
                        for (int e = 0; e < E; ++e)
                            sfp += ((double)s_cnt[e] / ((double)T * k)) *
                                   ((double)s_psum[e] / (double)T);
                        a.loss[0] = (float)(a.lambda * sfp);
                    }
                }
            }
            cw_sync();
            // every row of h into the B region (at most one row per token and expert)
            ds_load_rows(breg, a.hpitch, R, m8, m, [&](int j) { return a.h + (size_t)j * m8; }, ct);
            cw_sync();
        }

        if constexpr (kDown) {
            const int o_lo = (int)((int64_t)blockIdx.x * d / gridDim.x);
            const int o_hi = (int)((int64_t)(blockIdx.x + 1) * d / gridDim.x);
            const int ncol = o_hi - o_lo;
            ds_walk_down(nsel, s_sel, s_off, d, RG, [&](int, int oc, int nv, int r0, int nr) {
                int rb0 = r0;  // forward: every row of h is in the B region already
                if constexpr (MODE == kDsDown) {
                    if (loaded != r0) {  // this item's rows of h into the B region
                        cw_sync();
                        ds_load_rows(breg, a.hpitch, nr, m8, m,
                                     [&](int j) { return a.h_in + (size_t)(r0 + j) * m8; }, ct);
                        cw_sync();
                        loaded = r0;
                    }
                    rb0 = 0;
                }
                uint32_t bpt[NB];
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    const int j = nb * 8 + g;
                    bpt[nb] = j < nr ? breg_s + (uint32_t)((rb0 + j) * a.hpitch + 16 * c) : 0u;
                }
                float acc[2][NB][4];
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            acc[h][nb][q] = 0.f;
                for (int k0 = 0; k0 < m8; k0 += kDsKc2)
                    take_stage(std::integral_constant<int, 0>(), acc, pitch2, min(kDsKc2, m8 - k0),
                               k0, bpt);
                float v[8];
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    v[nb * 2 + 0] = acc[0][nb][0] + acc[1][nb][0];
                    v[nb * 2 + 1] = acc[0][nb][1] + acc[1][nb][1];
                }
                reduce(v, 2 * NB, [&](auto sum) {
                    for (int i = ct; i < 32 * 2 * NB; i += kDsCw * 32) {
                        const int L = i & 31, q = i >> 5, nb = q >> 1, jj = q & 1;
                        const int row = L >> 2, tok = nb * 8 + 2 * (L & 3) + jj;
                        if (row < nv && tok < nr) {
                            const bf16 ob = __float2bfloat16_rn(sum(L, q));
                            a.out[(size_t)(r0 + tok) * d + oc + row] = ob;
                            if constexpr (MODE == kDsForward)
                                outs[(size_t)(r0 + tok) * ncol + oc - o_lo + row] =
                                    __bfloat162float(ob);
                        }
                    }
                });
            });
            if constexpr (MODE == kDsForward) {
                // ---- the combine of this CTA's columns, in combine_kernel's arithmetic
                cw_sync();
                for (int i = ct; i < T * ncol; i += kDsCw * 32) {
                    const int t = i / ncol, o = i % ncol;
                    float acc = 0.f;
                    for (int j = 0; j < k; ++j) {
                        const int32_t row = s_slot[t * k + j];
                        if (row < 0)
                            continue;
                        acc = fmaf(s_w[t * k + j], outs[(size_t)row * ncol + o], acc);
                    }
                    acc *= a.scale;
                    a.y[(size_t)t * d + o_lo + o] = __float2bfloat16_rn(acc);
                }
            }
        }
    }
    pdl_trigger();
}

// --------------------------------------------------------------------- host side
struct DsGeom {
    int nb, bpitch, hpitch, bbytes, obytes, stage_bytes, stages, kc1, split13;
    size_t smem;
};

static int ds_grid()
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

static bool ds_geom_kc(const moe_params_t *p, int mode, bool noisy, int kc1, int split13,
                       DsGeom *g)
{
    g->nb = p->T <= 8 ? 1 : 2;
    g->kc1 = kc1;
    g->split13 = split13;
    const int m8 = round_up(p->m, 8);
    const int xp = round_up(p->d * 2, 128) + 16;
    const int hp = round_up(m8 * 2, 128) + 16;
    // B region: token rows of x (pitch xp) and / or rows of h (pitch hp).  Rows held:
    // router and forward, the T token rows and every row of h (an expert has at most
    // one row per token); step calls, one group of an expert's rows.
    const int group = 8 * g->nb < p->T * p->k ? 8 * g->nb : p->T * p->k;
    int sp = 0, xbytes = 0, hbytes = 0;
    g->bpitch = g->hpitch = 0;
    if (mode & (kDsRoute | kDsUp | kDsForward)) {
        g->bpitch = xp;
        sp = (split13 ? 1 : 2) * ds_pitch(p->d, kc1);  // 8 or 16 rows
        xbytes = ((mode & kDsUp) ? group : p->T) * xp;
    }
    if (mode & (kDsDown | kDsForward)) {
        g->hpitch = hp;
        sp = sp > ds_pitch(m8, kDsKc2) ? sp : ds_pitch(m8, kDsKc2);
        hbytes = ((mode & kDsDown) ? group : p->T * p->k) * hp;
    }
    g->bbytes = round_up(xbytes > hbytes ? xbytes : hbytes, 128);
    // forward: the rounded out values of this CTA's columns for the combine
    const int ncol = (p->d + ds_grid() - 1) / ds_grid() + 1;
    g->obytes = (mode & kDsForward) ? round_up(p->T * p->k * ncol * 4, 128) : 0;
    g->stage_bytes = round_up(kDsRows * sp, 128);
    const size_t fixed = (size_t)kDsBarBytes + ds_red_bytes(g->nb) + g->bbytes + g->obytes;
    if (fixed + (size_t)kDsMinStages * g->stage_bytes > kDsSmemCap)
        return false;
    const int st = (int)((kDsSmemCap - fixed) / g->stage_bytes);
    g->stages = st < kDsMaxStages ? st : kDsMaxStages;
    g->smem = fixed + (size_t)g->stages * g->stage_bytes;
    if (mode & (kDsRoute | kDsForward)) {
        const int nout = noisy ? 2 * p->E : p->E;
        if (nout > 32)
            return false;
        // a round of 256 router rows must fit beside the router's scratch
        if ((size_t)g->stages * g->stage_bytes < (size_t)kDsRouterScratch + 256 * nout * 2)
            return false;
    }
    return true;
}

static bool ds_geom(const moe_params_t *p, int mode, bool noisy, DsGeom *g)
{
    if (p->dtype != MOE_BF16 || p->T < 1 || p->T > kDecodeMaxTokens)
        return false;
    // GEMM 1 stages: 16 rows x 2048 columns while the forward layout fits 3 of them, else
    // 8 rows (W1 and W3 rows in alternate stages) x 2048, else 8 rows x 1024 -- decided on
    // the forward layout for every mode, so the step calls stream like the forward
    DsGeom f;
    int split = 0, kc = kDsKc1;
    if (!(ds_geom_kc(p, kDsForward, false, kDsKc1, 0, &f) && f.stages >= 3)) {
        split = 1;
        if (!ds_geom_kc(p, kDsForward, false, kDsKc1, 1, &f))
            kc = kDsKc1Small;
    }
    return ds_geom_kc(p, mode, noisy, kc, split, g);
}

template <int NB, int MODE>
static cudaError_t ds_launch(const DsGeom &g, int grid, const DsArgs &a, cudaStream_t s)
{
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    if (!attr_done[dev]) {
        e = cudaFuncSetAttribute(decode_stream_kernel<NB, MODE>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDsSmemCap);
        if (e != cudaSuccess)
            return e;
        attr_done[dev] = true;
    }
    if (MODE == kDsForward) {
        // every CTA must be resident for the grid barrier: a cooperative launch
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(kDsThreads);
        cfg.dynamicSmemBytes = g.smem;
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, decode_stream_kernel<NB, MODE>, a);
    } else {
        e = launch_pdl(decode_stream_kernel<NB, MODE>, dim3(grid), dim3(kDsThreads), g.smem, s, a);
    }
    count_launch();
    return e == cudaSuccess ? cudaGetLastError() : e;
}

template <int MODE>
static cudaError_t ds_dispatch(const DsGeom &g, int grid, DsArgs &a, cudaStream_t s)
{
    a.stages = g.stages;
    a.stage_bytes = g.stage_bytes;
    a.bpitch = g.bpitch;
    a.hpitch = g.hpitch;
    a.bbytes = g.bbytes;
    a.obytes = g.obytes;
    a.kc1 = g.kc1;
    a.split13 = g.split13;
    a.wait_ns = wait_limit_ns();
    return g.nb == 1 ? ds_launch<1, MODE>(g, grid, a, s) : ds_launch<2, MODE>(g, grid, a, s);
}

static DsArgs ds_args(const moe_params_t *p, int32_t *status)
{
    DsArgs a = {};
    a.T = p->T;
    a.d = p->d;
    a.m = p->m;
    a.E = p->E;
    a.k = p->k;
    a.C = p->capacity;
    a.router_type = p->router_type;
    a.lambda = p->balance_lambda;
    a.scale = p->rescale ? (float)p->E / (float)p->k : 1.0f;
    a.status = status;
    return a;
}

bool decode_route_fits(const moe_params_t *p, bool noisy)
{
    DsGeom g;
    return ds_geom(p, kDsRoute, noisy, &g);
}

bool decode_fits(const moe_params_t *p)
{
    DsGeom g;
    return ds_geom(p, kDsUp, false, &g) && ds_geom(p, kDsDown, false, &g);
}

bool decode_forward_fits(const moe_params_t *p, bool noisy)
{
    DsGeom g;
    return decode_route_fits(p, noisy) && decode_fits(p) && ds_geom(p, kDsForward, noisy, &g);
}

cudaError_t launch_route_decode(const moe_params_t *p, const void *x, const void *Wg,
                                const void *Wn, const float *noise, const float *bias,
                                int32_t *idx, float *w, float *probs_sum, float *importance,
                                int32_t *status, cudaStream_t s)
{
    DsGeom g;
    if (!ds_geom(p, kDsRoute, Wn != nullptr, &g))
        return cudaErrorInvalidValue;
    DsArgs a = ds_args(p, status);
    a.x = (const bf16 *)x;
    a.Wg = (const bf16 *)Wg;
    a.Wn = (const bf16 *)Wn;
    a.noise = noise;
    a.bias = bias;
    a.idx = idx;
    a.w = w;
    a.probs_sum = probs_sum;
    a.importance = importance;
    return ds_dispatch<kDsRoute>(g, 1, a, s);
}

cudaError_t launch_up_decode(const moe_params_t *p, const void *x_perm, const int32_t *offsets,
                             const void *W13, void *h, char *ws, cudaStream_t s)
{
    DsGeom g;
    if (!ds_geom(p, kDsUp, false, &g))
        return cudaErrorInvalidValue;
    DsArgs a = ds_args(p, reinterpret_cast<int32_t *>(ws));
    a.x_perm = (const bf16 *)x_perm;
    a.offsets_in = offsets;
    a.W13 = (const bf16 *)W13;
    a.h = (bf16 *)h;
    return ds_dispatch<kDsUp>(g, ds_grid(), a, s);
}

cudaError_t launch_down_decode(const moe_params_t *p, const void *h, const int32_t *offsets,
                               const void *W2, void *out, char *ws, cudaStream_t s)
{
    DsGeom g;
    if (!ds_geom(p, kDsDown, false, &g))
        return cudaErrorInvalidValue;
    DsArgs a = ds_args(p, reinterpret_cast<int32_t *>(ws));
    a.h_in = (const bf16 *)h;
    a.offsets_in = offsets;
    a.W2 = (const bf16 *)W2;
    a.out = (bf16 *)out;
    return ds_dispatch<kDsDown>(g, ds_grid(), a, s);
}

cudaError_t launch_forward_decode(const moe_params_t *p, const moe_buffers_t *b, char *ws,
                                  cudaStream_t s)
{
    DsGeom g;
    if (!ds_geom(p, kDsForward, b->Wnoise != nullptr, &g))
        return cudaErrorInvalidValue;
    DsArgs a = ds_args(p, reinterpret_cast<int32_t *>(ws));
    a.gbar = reinterpret_cast<int32_t *>(ws) + kWsDecodeBarrierWord;
    a.x = (const bf16 *)b->x;
    a.Wg = (const bf16 *)b->Wg;
    a.Wn = (const bf16 *)b->Wnoise;
    a.noise = b->noise;
    a.bias = b->bias;
    a.W13 = (const bf16 *)b->W13_e;
    a.W2 = (const bf16 *)b->W2_e;
    a.idx = b->topk_idx;
    a.w = b->topk_w;
    a.probs_sum = b->probs_sum;
    a.importance = b->importance;
    a.counts = b->counts;
    a.kept = b->kept;
    a.offsets = b->offsets;
    a.row_token = b->row_token;
    a.slot_row = b->slot_row;
    a.f = b->f;
    a.P = b->P;
    a.loss = b->loss;
    a.x_perm_out = (bf16 *)b->x_perm;
    a.h = (bf16 *)b->h;
    a.out = (bf16 *)b->out;
    a.y = (bf16 *)b->y;
    return ds_dispatch<kDsForward>(g, ds_grid(), a, s);
}

}  // namespace moe
