// kernels.h -- internal interface between the C-ABI layer (api.cu) and the
// kernel translation units of libmoe.so.  Not installed, not part of the ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// Tokens handled by one dispatch CTA (one warp ballot per expert).
constexpr int kDispatchChunk = 32;
// Smallest number of tokens one router CTA handles (sizes the partial sums).
constexpr int kRouterMinTokens = 8;
// Warps of a router CTA (bf16: split-K over the warps; f32: one token per warp).
constexpr int kRouterWarps = 8;
// Rows of the transposed router weights [W_g | W_noise | 0]^T in the workspace.
constexpr int kWtRows = 128;
// Batches up to this many tokens use the split-K router (partials in `rsmall`).
constexpr int kRouterSmallTokens = 64;
constexpr int kRouterSmallSplit = 32;
// Columns of x per split-K slice: d / kRouterSmallSplit rounded up to a multiple of 8,
// so every slice starts on a 16-byte boundary of a row (d % 8 == 0).
__host__ __device__ inline int router_small_kc(int d)
{
    return ((d + kRouterSmallSplit - 1) / kRouterSmallSplit + 7) / 8 * 8;
}

// Shared memory of one split-K router slice (bytes): bf16 stages the slice's x rows
// [round16(T)][round16(kc) + 8] and weight columns [round16(kc)][round8(nout) + 8] as bf16
// tiles for mma.sync; f32 stages x [T][kc] and the columns [kc][nout] as f32.
__host__ __device__ inline size_t router_small_slice_smem(int T, int d, int nout, int dtype)
{
    const int kc = router_small_kc(d);
    if (dtype == MOE_BF16) {
        const int kp = (kc + 15) / 16 * 16, np = (nout + 7) / 8 * 8;
        return 2 * ((size_t)(T + 15) / 16 * 16 * (kp + 8) + (size_t)kp * (np + 8));
    }
    return sizeof(float) * ((size_t)T * kc + (size_t)kc * nout);
}

// Byte offsets of the sections of the caller's workspace.
struct WsLayout {
    size_t wt;     // router weights transposed to [nout_pad][d] (dtype; backward, f32 router)
    size_t rpart;  // router per-CTA partial sums [blocks][2][E] f32
    size_t hist;   // dispatch per-chunk counts, then bases, [E][chunks] int32
    size_t dcounts;// routed count of every expert [E] int32 (next to the chunk bases)
    size_t rsmall; // small-batch router partial logits [32][T][2E] f32 (T <= 64)
    size_t gsmall; // small-batch forward: softmax and gate weight rows [2][T][E] f32
    size_t total;
};
WsLayout ws_layout(const moe_params_t *p);

__host__ __device__ inline int round_up(int v, int m) { return (v + m - 1) / m * m; }
__host__ __device__ inline int ceil_div(int v, int m) { return (v + m - 1) / m; }

// Error reporting of the C ABI, for entry points outside api.cu.
int validate_params(const char *fn, const moe_params_t *p);
int report_error(int code, const char *msg);
int report_cuda(cudaError_t e, const char *where);
int report_ok();

// Launches `kern` with programmatic stream serialization allowed: the kernel
// may be scheduled while the previous kernel on `s` finishes (it waits for that
// kernel with griddepcontrol.wait before touching memory).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Launch counter shared by every launch site.
void count_launch(int n = 1);
// Current time limit of bounded device waits (ns).
uint64_t wait_limit_ns();
// Rows of A that the 2-SM grouped GEMM's concurrent clusters sweep N over (0: all
// of an expert's rows).
int gemm_band_rows();

// Every launcher returns cudaSuccess or the launch error.
cudaError_t launch_partition(const void *W1, const void *W3, const void *W2, int d, int d_ff,
                             int E, int m, int mode, const int32_t *perm, int dtype,
                             void *W13_e, void *W2_e, int32_t *status, cudaStream_t s);

// a1; Wt: the router weights packed by launch_router_pack (used by the tensor-core
// router), or NULL to pack them into the workspace first
cudaError_t launch_route(const moe_params_t *p, const void *x, const void *Wg,
                         const void *Wnoise, const void *Wt, const float *noise,
                         const float *bias, int32_t *idx, float *w, float *probs_sum,
                         float *importance, char *ws, int32_t *status, cudaStream_t s);

// Rows of the packed router weights [rows][d]: 2E (noisy) or E, padded to 16..128.
int router_packed_rows(int E, bool noisy);
cudaError_t launch_router_pack(const moe_params_t *p, const void *Wg, const void *Wnoise, void *Wt,
                               cudaStream_t s);
// a1 on the tcgen05 tensor cores (bf16), token sums included (per-CTA partials in
// `part`, added by the CTA that finishes last; `counter` is zero between calls).
// The gate epilogue also counts the chunks of a2 (hist), which the last CTA scans
// into chunk bases and routed counts (dcounts).
cudaError_t launch_route_tc(const moe_params_t *p, const void *x, const void *Wt, bool noisy,
                            const float *noise, const float *bias, int32_t *idx, float *w,
                            float *probs_sum, float *importance, float *part, int32_t *counter,
                            int32_t *hist, int32_t *dcounts, int32_t *status, cudaStream_t s);

// a2 count step: chunk histogram of idx, scanned into bases (hist) and routed
// counts (dcounts) by the CTA that finishes last (`counter` zero between calls).
cudaError_t launch_count(const moe_params_t *p, const int32_t *idx, int32_t *hist,
                         int32_t *counter, int32_t *dcounts, int32_t *status, cudaStream_t s);
// a2 scatter step: kept, offsets, slot_row, row_token and x_perm (NULL: tables only)
// from the bases and counts of the count step (or of the router).
cudaError_t launch_scatter(const moe_params_t *p, const void *x, const int32_t *idx,
                           const int32_t *bases, const int32_t *dcounts, void *x_perm,
                           int32_t *row_token, int32_t *slot_row, int32_t *counts,
                           int32_t *kept, int32_t *offsets, cudaStream_t s);
// count + scatter; routed: skip the count (the router of the same workspace left
// the bases and counts of these indices)
cudaError_t launch_dispatch(const moe_params_t *p, const void *x, const int32_t *idx,
                            void *x_perm, int32_t *row_token, int32_t *slot_row,
                            int32_t *counts, int32_t *kept, int32_t *offsets, char *ws,
                            int32_t *status, bool routed, cudaStream_t s);

// moe_forward's a1 + a2 + a6 for 1 <= T <= 64 (cooperative, 32 CTAs): the indices,
// weights, token sums, tables, x_perm, counts / kept / offsets and f, P, L_balance
cudaError_t launch_front_small(const moe_params_t *p, const moe_buffers_t *b, char *ws,
                               cudaStream_t s);
bool front_small_fits(const moe_params_t *p, bool noisy);

// a3 / a4 for f32 (CUDA-core FMA)
cudaError_t launch_up_simt(const moe_params_t *p, const float *x_perm, const int32_t *offsets,
                           const float *W13, float *h, cudaStream_t s);
cudaError_t launch_down_simt(const moe_params_t *p, const float *h, const int32_t *offsets,
                             const float *W2, float *out, cudaStream_t s);

// a3 / a4 for bf16 (tcgen05 tensor cores, TMA, TMEM)
cudaError_t launch_up_tc(const moe_params_t *p, const void *x_perm, const int32_t *offsets,
                         const void *W13, void *h, int32_t *status, cudaStream_t s);
cudaError_t launch_up_tc_gather(const moe_params_t *p, const void *x, const int32_t *row_token,
                                const int32_t *offsets, const void *W13, void *h,
                                int32_t *status, cudaStream_t s);
cudaError_t launch_down_tc(const moe_params_t *p, const void *h, const int32_t *offsets,
                           const void *W2, void *out, int32_t *status, cudaStream_t s);

// Decode-shaped bf16 batches (1 <= T <= kDecodeMaxTokens): the weight-streaming
// kernel of decode.cu.  Larger batches run the tcgen05 grouped GEMMs.
constexpr int kDecodeMaxTokens = 16;
// a1 (logits and gate, one CTA) for such a batch: nout <= 32 and the token rows fit
bool decode_route_fits(const moe_params_t *p, bool noisy);
cudaError_t launch_route_decode(const moe_params_t *p, const void *x, const void *Wg,
                                const void *Wn, const float *noise, const float *bias,
                                int32_t *idx, float *w, float *probs_sum, float *importance,
                                int32_t *status, cudaStream_t s);
// a3 / a4 for such a batch (the step calls)
bool decode_fits(const moe_params_t *p);
cudaError_t launch_up_decode(const moe_params_t *p, const void *x_perm, const int32_t *offsets,
                             const void *W13, void *h, char *ws, cudaStream_t s);
cudaError_t launch_down_decode(const moe_params_t *p, const void *h, const int32_t *offsets,
                               const void *W2, void *out, char *ws, cudaStream_t s);
// the whole layer (a1..a6) in one cooperative launch
bool decode_forward_fits(const moe_params_t *p, bool noisy);
cudaError_t launch_forward_decode(const moe_params_t *p, const moe_buffers_t *b, char *ws,
                                  cudaStream_t s);

cudaError_t launch_combine(const moe_params_t *p, const void *out, const int32_t *slot_row,
                           const float *w, void *y, cudaStream_t s, const void *resid = nullptr);
// offsets {0, T} of a one-expert grouped GEMM over all tokens (the shared block)
cudaError_t launch_token_range(int32_t *offsets2, int T, cudaStream_t s);

cudaError_t launch_gate_stats(const moe_params_t *p, const int32_t *counts,
                              const float *probs_sum, float *f, float *P, float *loss,
                              cudaStream_t s);

}  // namespace moe
