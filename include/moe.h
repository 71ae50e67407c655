/*
 * moe.h -- C ABI of libmoe.so: the forward pass of a sparse Mixture-of-Experts
 * SwiGLU FFN layer on NVIDIA B200 (sm_100a).
 *
 * The layer (notation: T tokens, model width d, dense FFN width d_ff, E experts,
 * k experts per token, m neurons per expert, R kept (token, expert) rows):
 *
 *   a0  experts are equal disjoint random subsets of the dense FFN's
 *       intermediate neurons, or whole copies of it
 *         ["LLaMA-MoE v2: 基于后训练混合专家模型的稀疏性探索与技术突破",
 *          section "专家构建方法"; "Llama 3 Meets MoE: Efficient Upcycling",
 *          section 2 "解决方案概述"]
 *   a1  H = x W_g (+ b) + eps * Softplus(x W_noise);  idx = KeepTopK(H, k);
 *       Mixtral type G = Softmax over the k kept logits, ST type G = the full
 *       softmax at the kept experts
 *         ["Llama 3 Meets MoE", section 3 "核心公式" (Noisy Top-k routing) and
 *          section 5 "路由器算法消融实验"]
 *   a2  expert capacity C = tokens per batch / E * CF; assignments past an
 *       expert's capacity are dropped (lower token index wins)
 *         ["Llama 3 Meets MoE", section 3 "容量因子"]
 *   a3  h = silu(x W1_e^T) * (x W3_e^T)        (SwiGLU expert, first half)
 *   a4  out = h W2_e^T                           (second half)
 *         ["LLaMA-MoE v2", code sample "代码实现示例", class Expert]
 *   a5  y_t = s * sum_j G_tj out_{row(t,j)},  s = E/k with rescale, else 1
 *         ["Llama 3 Meets MoE", section 3, y = sum_i G(x)_i E_i(x);
 *          "LLaMA-MoE v2", section "重新缩放机制与负载均衡"]
 *   a6  gate load, gate importance, f_e, P_e, L_balance = lambda sum f_e P_e
 *         ["LLaMA-MoE v2", section "门控机制设计"; "从大炼到巧炼：LLaMA-MoE 如何用
 *          MoE 架构让 LLM 变快变省", section "持续预训练" (monitored metrics)]
 *
 * Conventions
 *  - Every entry point returns MOE_OK (0) or a negative moe_status_t.  On error
 *    nothing was launched and moe_last_error_string() describes the problem.
 *  - Pointers named as device pointers must be CUDA device memory of the
 *    current device; the caller owns every buffer.  The library allocates no
 *    device memory: internal scratch lives in the caller's workspace, sized by
 *    moe_workspace_size() and zeroed once by moe_workspace_init().
 *  - Every compute call is asynchronous on `stream` (a cudaStream_t passed as
 *    void*; NULL is the legacy default stream).  Calls never synchronise the
 *    host with the device, except moe_get_device_status().
 *  - Errors found by kernels (an expert index outside [0,E), a NaN routing
 *    logit, a wait that ran out) are recorded in a status word inside the
 *    workspace; the first one sticks until read with clear=1.
 *  - Device pointers must be 16-byte aligned (MOE_ERR_ALIGN otherwise).
 *  - Row-major everywhere; "[A][B]" means B is the contiguous dimension.
 *  - Element type of activations and expert/router weights is `dtype`
 *    (MOE_BF16 or MOE_F32); gate weights, noise, bias and statistics are f32;
 *    indices are int32.  bf16 paths accumulate in f32.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,    /* null pointer, k < 1, k > E, E > 64, T < 0, ... */
    MOE_ERR_SHAPE = -2,          /* d % 8 != 0, d_ff % E != 0 (disjoint), too large */
    MOE_ERR_ALIGN = -3,          /* device pointer not 16-byte aligned */
    MOE_ERR_DTYPE = -4,          /* dtype not MOE_BF16 / MOE_F32, or unsupported mix */
    MOE_ERR_CUDA = -5,           /* a CUDA runtime/driver call or launch failed */
    MOE_ERR_DEVICE_TIMEOUT = -6, /* a kernel wait ran past its limit (device status) */
    MOE_ERR_DEVICE_BADINDEX = -7,/* expert index out of range or NaN logit (device status) */
    MOE_ERR_WORKSPACE = -8,      /* workspace smaller than moe_workspace_size() */
    MOE_ERR_UNSUPPORTED = -9     /* no kernel for this device or configuration */
} moe_status_t;

enum { MOE_F32 = 0, MOE_BF16 = 1 };
enum { MOE_ROUTER_MIXTRAL = 0, MOE_ROUTER_ST = 1 };
enum { MOE_PARTITION_DISJOINT = 0, MOE_PARTITION_COPY = 1, MOE_PARTITION_STACKED = 2 };

#define MOE_MAX_EXPERTS 64
#define MOE_MAX_TOPK 8

/* Layer description, passed by pointer, read only during the call. */
typedef struct {
    int32_t T;             /* tokens in the batch (>= 0) */
    int32_t d;             /* model width (multiple of 8) */
    int32_t E;             /* experts, 1..64 */
    int32_t k;             /* experts per token, 1..min(E, 8) */
    int32_t m;             /* neurons per expert (d_ff/E disjoint, d_ff copies) */
    int32_t dtype;         /* MOE_BF16 or MOE_F32 */
    int32_t router_type;   /* MOE_ROUTER_MIXTRAL or MOE_ROUTER_ST */
    int32_t capacity;      /* rows kept per expert; < 0 means no limit */
    int32_t rescale;       /* nonzero: combine scales by E/k */
    float balance_lambda;  /* lambda of L_balance */
} moe_params_t;

/* Library version string (static storage). */
const char *moe_version(void);

/* Message of the last error returned on the calling thread (thread-local storage). */
const char *moe_last_error_string(void);

/* Number of kernels this process has launched through the library so far. */
uint64_t moe_launch_count(void);

/* Expert capacity ["Llama 3 Meets MoE", section 3 "容量因子"]: tokens per batch
 * divided by the number of experts times the capacity factor, rounded up to a
 * whole token: ceil(T * cf / E).  cf < 0 returns -1 (no limit).  Host-only. */
int32_t moe_capacity(int32_t T, int32_t E, double cf);

/* ---- packed expert weight layout (a0 output, a3/a4 input) ----------------
 * W13_e [E][2*m16][d], m16 = m rounded up to a multiple of 16.  Rows come in
 *   groups of 32: rows 32b..32b+15 are the W1 (gate, inside silu) rows of
 *   expert neurons 16b..16b+15, rows 32b+16..32b+31 their W3 (up) rows.  Rows
 *   of neurons >= m are zero.
 * W2_e  [E][d][m8], m8 = m rounded up to a multiple of 8; columns >= m are zero.
 * h     [rows][m8] (the SwiGLU activations; columns >= m are never read). */
int64_t moe_packed_w13_elems(int32_t E, int32_t m, int32_t d);
int64_t moe_packed_w2_elems(int32_t E, int32_t m, int32_t d);
int32_t moe_h_ld(int32_t m);

/* a0. Builds the packed expert weights from a dense SwiGLU FFN
 * ["LLaMA-MoE v2", section "专家构建方法" (IndependentRandom: the index set of
 * intermediate neurons split into E equal disjoint subsets);
 * "Llama 3 Meets MoE", section 2 (upcycling: E copies of the FFN)].
 *   mode DISJOINT: W1, W3 [d_ff][d], W2 [d][d_ff] (nn.Linear out x in);
 *                  m = d_ff / E; expert e owns neurons perm[e*m .. e*m+m);
 *                  perm [d_ff] int32 device, a permutation of 0..d_ff-1.
 *   mode COPY:     same inputs, m = d_ff, every expert is the whole FFN; perm unused.
 *   mode STACKED:  already-built experts (e.g. perturbed copies): W1, W3 [E][d_ff][d],
 *                  W2 [E][d][d_ff]; m = d_ff; perm unused.
 * Outputs W13_e, W2_e in the packed layout above (device, caller-allocated with
 * moe_packed_*_elems elements of dtype).  A perm entry outside [0, d_ff) writes
 * a zero neuron and sets MOE_ERR_DEVICE_BADINDEX in the status word of `ws`
 * (ws may be NULL, then such entries are only zeroed).
 * Errors: MOE_ERR_INVALID_ARG, MOE_ERR_SHAPE (d % 8, d_ff % E in DISJOINT),
 * MOE_ERR_DTYPE, MOE_ERR_ALIGN, MOE_ERR_CUDA. */
int moe_partition_experts(const void *W1, const void *W3, const void *W2,
                          int32_t d, int32_t d_ff, int32_t E, int32_t mode,
                          const int32_t *perm, int32_t dtype,
                          void *W13_e, void *W2_e, void *ws, void *stream);

/* Bytes of workspace the calls below need for `p` (covers every call with the
 * same dtype and the same or smaller T, E, d, m).  Host-only, never fails
 * (returns 0 on bad params). */
size_t moe_workspace_size(const moe_params_t *p);

/* Zeroes a freshly allocated workspace (status word and counters).  Call once
 * after allocation; the library keeps it consistent afterwards. */
int moe_workspace_init(void *ws, size_t ws_bytes, void *stream);

/* a1. Router ["Llama 3 Meets MoE", section 3 "Noisy Top-k 路由", section 5].
 *   x [T][d] (dtype), Wg [d][E] (dtype), Wnoise [d][E] (dtype, NULL: no noise),
 *   noise [T][E] f32 (the StandardNormal() draws; required iff Wnoise given),
 *   bias [E] f32 (NULL: none; added to the clean logits).
 * Outputs (device): topk_idx [T][k] int32 (slot j holds the j-th largest H;
 *   ties go to the lower expert index), topk_w [T][k] f32 (gate weights),
 *   probs_sum [E] f32 (sum over tokens of the full softmax of H),
 *   importance [E] f32 (sum over tokens of the gate weight of each expert).
 * A NaN logit sets MOE_ERR_DEVICE_BADINDEX and writes idx -1, weight 0. */
int moe_route(const moe_params_t *p, const void *x, const void *Wg, const void *Wnoise,
              const float *noise, const float *bias, int32_t *topk_idx, float *topk_w,
              float *probs_sum, float *importance, void *ws, size_t ws_bytes, void *stream);

/* The router weights W_g (and W_noise) as the tensor-core router reads them: one
 * K-major row per logit ([rows][d] bf16: row 2e = W_g[:, e], row 2e+1 = W_noise[:, e]
 * with noise, row e = W_g[:, e] without; rows = 2E or E rounded up to 16, 32, 64 or
 * 128; the other rows zero).  moe_route rebuilds them in the workspace on every call;
 * a caller whose router weights do not change between calls (inference, or until the
 * next optimizer step) packs them once with moe_router_pack and passes them to
 * moe_route_packed or moe_forward (moe_buffers_t.router_packed), and must pack them
 * again after changing W_g or W_noise.
 * moe_router_packed_bytes: bytes of the packed buffer for p (bf16), noisy = whether
 * W_noise is part of the router; 0 on bad params.  Host-only.
 * moe_router_pack: writes the packed buffer Wt (device, 16-byte aligned) from Wg and
 * Wnoise (NULL: none) [d][E] bf16.  Errors: MOE_ERR_INVALID_ARG, MOE_ERR_ALIGN,
 * MOE_ERR_DTYPE (f32), MOE_ERR_CUDA. */
size_t moe_router_packed_bytes(const moe_params_t *p, int32_t noisy);
int moe_router_pack(const moe_params_t *p, const void *Wg, const void *Wnoise, void *Wt,
                    void *stream);

/* a1 with the router weights packed by moe_router_pack (Wt, for the same Wg/Wnoise
 * and E): the same outputs as moe_route, without the packing pass.  Wg and Wnoise
 * are still required: batches that do not run on the tensor-core router (f32, up to
 * 64 tokens) read them directly. */
int moe_route_packed(const moe_params_t *p, const void *x, const void *Wg, const void *Wnoise,
                     const void *Wt, const float *noise, const float *bias, int32_t *topk_idx,
                     float *topk_w, float *probs_sum, float *importance, void *ws,
                     size_t ws_bytes, void *stream);

/* a2. Dispatch with capacity ["Llama 3 Meets MoE", section 3 "容量因子"].
 * Stable counting sort of the T*k assignments by expert, token-ascending inside
 * an expert; assignment (t,j) is dropped iff its rank inside its expert is
 * >= p->capacity (no limit when < 0).  Outputs (device):
 *   counts [E] (routed, pre-drop = gate load), kept [E] = min(counts, C),
 *   offsets [E+1] exclusive prefix sum of kept (offsets[E] = R),
 *   row_token [T*k] (first R entries: token of each kept row),
 *   slot_row [T][k] (row of each assignment, -1 if dropped),
 *   x_perm [T*k][d] (dtype; first R rows: x of row_token, grouped by expert).
 * topk_idx entries outside [0,E) are dropped and set MOE_ERR_DEVICE_BADINDEX. */
int moe_dispatch(const moe_params_t *p, const void *x, const int32_t *topk_idx,
                 void *x_perm, int32_t *row_token, int32_t *slot_row, int32_t *counts,
                 int32_t *kept, int32_t *offsets, void *ws, size_t ws_bytes, void *stream);

/* a2 right after moe_route ["Llama 3 Meets MoE", section 3 "容量因子"]: the same
 * outputs as moe_dispatch for the indices that the last moe_route call on this
 * workspace wrote, without counting them again.  moe_route leaves, in the
 * workspace, how many tokens of each 32-token chunk it sent to each expert (the
 * tensor-core router counts them in its gate epilogue), scanned into the chunks'
 * rank bases; this call only ranks, writes the tables and copies x.  Requirements:
 * the same workspace, the same p (T, E, k), topk_idx as written by that moe_route
 * call and not changed since, and no other moe_route / moe_dispatch on this
 * workspace in between; otherwise the results are undefined (use moe_dispatch).
 * p->capacity may differ from the routing call's (it is applied here). */
int moe_dispatch_routed(const moe_params_t *p, const void *x, const int32_t *topk_idx,
                        void *x_perm, int32_t *row_token, int32_t *slot_row, int32_t *counts,
                        int32_t *kept, int32_t *offsets, void *ws, size_t ws_bytes,
                        void *stream);

/* a2, tables only: moe_dispatch without the permuted copy of x (x_perm).  Same
 * counts, kept, offsets, row_token and slot_row.  For moe_expert_up_gather, which
 * reads the rows of x through row_token itself. */
int moe_dispatch_rows(const moe_params_t *p, const int32_t *topk_idx, int32_t *row_token,
                      int32_t *slot_row, int32_t *counts, int32_t *kept, int32_t *offsets,
                      void *ws, size_t ws_bytes, void *stream);

/* a2 without a workspace.  The pages have no counterpart: this is a service
 * for callers that cannot allocate device memory or pass a workspace (for
 * example a host engine whose plugin interface hands a layer only its input and
 * output tensors and forbids allocation while work is enqueued).  Same inputs,
 * outputs and results as moe_dispatch; `status` (device int32, 4-byte aligned)
 * receives MOE_ERR_DEVICE_BADINDEX like the workspace status word (set only,
 * never cleared: the caller zeroes it).  It is required when T > 0, since it is
 * the only place a bad expert index is reported (MOE_ERR_INVALID_ARG if NULL);
 * with T = 0 it may be NULL.
 * Scratch: a fixed 256 KiB array inside the library image, reserved on every
 * GPU that loads libmoe.so until the process exits; limit E * ceil(T/32) <=
 * 65536 (T <= 32768 at E = 64), larger sizes return MOE_ERR_SHAPE.  The first
 * call on a device looks up that array's device address (make it before any
 * stream capture).  All calls share the array: calls that overlap on the GPU
 * race, so serialise them.  Allocates nothing. */
int moe_dispatch_noalloc(const moe_params_t *p, const void *x, const int32_t *topk_idx,
                         void *x_perm, int32_t *row_token, int32_t *slot_row, int32_t *counts,
                         int32_t *kept, int32_t *offsets, int32_t *status, void *stream);

/* a3. First half of every expert's SwiGLU FFN on its kept rows
 * ["LLaMA-MoE v2", code sample, class Expert: down(silu(gate(x)) * up(x))]:
 *   h[r] = silu(x_perm[r] W1_e^T) * (x_perm[r] W3_e^T) for rows r in
 *   [offsets[e], offsets[e+1]).  x_perm [T*k][d], W13_e packed, h [T*k][m8].
 * bf16: tcgen05 tensor cores, f32 accumulate, h rounded to bf16; for T <= 16
 * (decode-shaped batches) a weight-streaming kernel on mma.sync instead.
 * f32: CUDA-core FMA in f32 (no TF32).  Row tables stay on the device. */
int moe_expert_up(const moe_params_t *p, const void *x_perm, const int32_t *offsets,
                  const void *W13_e, void *h, void *ws, size_t ws_bytes, void *stream);

/* a3 reading the activations in place ["LLaMA-MoE v2", code sample, class Expert]:
 * h[r] = silu(x[row_token[r]] W1_e^T) * (x[row_token[r]] W3_e^T) for the kept rows
 * r of expert e.  x [T][d] (unpermuted), row_token from moe_dispatch(_rows); the
 * tensor-core kernel gathers four rows of x per TMA instruction.  bf16 only
 * (MOE_ERR_DTYPE otherwise).  Bit-identical to moe_expert_up on x_perm; it saves
 * the T*k*d x_perm buffer and its copy, but the one-row TMA gathers make the GEMM
 * about 2.8x slower on B200 (1593 vs 561 us at T=16384, d=4096, 8x1376, top-2),
 * so moe_forward does not use it. */
int moe_expert_up_gather(const moe_params_t *p, const void *x, const int32_t *row_token,
                         const int32_t *offsets, const void *W13_e, void *h, void *ws,
                         size_t ws_bytes, void *stream);

/* a4. Second half: out[r] = h[r] W2_e^T.  h [T*k][m8], W2_e packed, out [T*k][d].
 * bf16 with T <= 16: the weight-streaming kernel, as for moe_expert_up. */
int moe_expert_down(const moe_params_t *p, const void *h, const int32_t *offsets,
                    const void *W2_e, void *out, void *ws, size_t ws_bytes, void *stream);

/* a3 then a4. */
int moe_expert_ffn(const moe_params_t *p, const void *x_perm, const int32_t *offsets,
                   const void *W13_e, const void *W2_e, void *h, void *out, void *ws,
                   size_t ws_bytes, void *stream);

/* a5. Combine ["Llama 3 Meets MoE", section 3; "LLaMA-MoE v2", rescale]:
 *   y[t] = s * sum_{j<k, slot_row[t][j] >= 0} topk_w[t][j] * out[slot_row[t][j]],
 * summed in slot order in f32; s = E/k if p->rescale else 1.  A token whose
 * slots were all dropped gets y = 0.  out [T*k][d], y [T][d] (dtype). */
int moe_combine(const moe_params_t *p, const void *out, const int32_t *slot_row,
                const float *topk_w, void *y, void *stream);

/* a6. Gate statistics ["LLaMA-MoE v2", section "门控机制设计"]:
 *   f[e] = counts[e] / (T k),  P[e] = probs_sum[e] / T,
 *   loss[0] = lambda * sum_e f[e] P[e]   (all f32 device outputs; T = 0 gives 0). */
int moe_gate_stats(const moe_params_t *p, const int32_t *counts, const float *probs_sum,
                   float *f, float *P, float *loss, void *stream);

/* Every buffer moe_forward touches (device pointers, caller-owned). */
typedef struct {
    /* inputs */
    const void *x;          /* [T][d] */
    const void *Wg;         /* [d][E] */
    const void *Wnoise;     /* [d][E] or NULL */
    const float *noise;     /* [T][E] or NULL */
    const float *bias;      /* [E] or NULL */
    const void *W13_e;      /* packed */
    const void *W2_e;       /* packed */
    /* outputs */
    void *y;                /* [T][d] */
    float *loss;            /* [1] L_balance */
    int32_t *counts;        /* [E] gate load (pre-drop) */
    float *importance;      /* [E] gate importance */
    float *f;               /* [E] */
    float *P;               /* [E] */
    /* intermediates (kept for inspection) */
    int32_t *topk_idx;      /* [T][k] */
    float *topk_w;          /* [T][k] */
    float *probs_sum;       /* [E] */
    void *x_perm;           /* [T*k][d] */
    int32_t *row_token;     /* [T*k] */
    int32_t *slot_row;      /* [T][k] */
    int32_t *kept;          /* [E] */
    int32_t *offsets;       /* [E+1] */
    void *h;                /* [T*k][m8] */
    void *out;              /* [T*k][d] */
    /* optional input: Wg / Wnoise packed by moe_router_pack, or NULL (packed per call) */
    const void *router_packed;
} moe_buffers_t;

/* a1 -> a2 -> a3 -> a4 -> a5 -> a6 on one stream, no host synchronisation.
 * Every output equals what the step calls (moe_route, moe_dispatch, moe_expert_up,
 * moe_expert_down, moe_combine, moe_gate_stats) give on the same inputs, bit for bit.
 * How it launches depends on the batch: bf16 batches of at most 16 tokens run the
 * whole layer as one cooperative launch; batches of at most 64 tokens whose router is
 * the split-K one run a1, a2 and a6 as one cooperative launch of 32 CTAs before the
 * expert GEMMs and a5; larger batches run the steps' kernels.  A device wait past the
 * limit (moe_set_wait_limit_ns) is reported as MOE_ERR_DEVICE_TIMEOUT in the status
 * word, as in every call. */
int moe_forward(const moe_params_t *p, const moe_buffers_t *b, void *ws, size_t ws_bytes,
                void *stream);

/* ---- residual MoE: shared neurons plus disjoint experts ------------------
 * "LLaMA-MoE v2", section "共享神经元划分" (Shared Neuron Partitioning): a set S
 * of the dense FFN's intermediate neurons is shared by all experts and the
 * remaining neurons are split into E equal disjoint experts; the hub page "从大炼
 * 到巧炼" lists the residual MoE module that holds it.  The pages give no output
 * formula; the layer computed here is the plain reading of a residual block that
 * every token passes through next to the routed experts:
 *     y_t = FFN_S(x_t) + s * sum_j G_tj E_{idx_tj}(x_t)
 * with FFN_S the SwiGLU FFN restricted to the neurons of S (not scaled by s,
 * applied to dropped tokens too) and E_e the experts over the other neurons.
 * Choosing S (importance scores from gradients) is out of scope: the caller
 * supplies it. */

/* a0 for the residual MoE.  shared_idx [m_s] (device int32): the neurons of S;
 * perm_rest [d_ff - m_s] (device int32): the other neurons in expert order
 * (expert e gets perm_rest[e m, (e+1) m), m = (d_ff - m_s) / E).  Outputs the
 * packed experts W13_e / W2_e (E experts of width m) and the packed shared
 * block W13_s / W2_s (one "expert" of width m_s), layouts as above.  Entries
 * outside [0, d_ff) write zero neurons and set MOE_ERR_DEVICE_BADINDEX in ws.
 * Errors: MOE_ERR_SHAPE unless 1 <= m_s < d_ff and E divides d_ff - m_s. */
int moe_partition_residual(const void *W1, const void *W3, const void *W2, int32_t d,
                           int32_t d_ff, int32_t E, const int32_t *shared_idx, int32_t m_s,
                           const int32_t *perm_rest, int32_t dtype, void *W13_e, void *W2_e,
                           void *W13_s, void *W2_s, void *ws, void *stream);

/* a5 with the residual term: y[t] = s * sum_j topk_w[t][j] out[slot_row[t][j]]
 * + resid[t] (the scaled sum in slot order in f32, then resid added, rounded
 * once).  resid [T][d] in dtype. */
int moe_combine_residual(const moe_params_t *p, const void *out, const int32_t *slot_row,
                         const float *topk_w, const void *resid, void *y, void *stream);

/* The residual MoE layer: a1, a2, a3, a4 for the routed experts (p->m = their
 * width), then the shared block FFN_S over all T tokens as a one-expert grouped
 * GEMM (h_s [T][m_s8], out_s [T][d], caller-owned; out_s = FFN_S(x)), then
 * moe_combine_residual and a6.  The workspace must be sized for p. */
int moe_forward_residual(const moe_params_t *p, const moe_buffers_t *b, const void *W13_s,
                         const void *W2_s, int32_t m_s, void *h_s, void *out_s, void *ws,
                         size_t ws_bytes, void *stream);

/* ---- clustering partition (an alternative source of a0's perm) ------------
 * ["LLaMA-MoE v2", section "专家构建方法", IndependentClustering: the neurons are
 * grouped by k-means over their weight vectors and each cluster becomes one
 * expert; the index set is split into E subsets of equal size m = d_ff / E.]
 * Balanced k-means over the rows of F [d_ff][d] (dtype; the caller passes W1,
 * the gate projection):
 *   start:      C[e] = F[init_idx[e]] (E distinct neuron indices, device int32);
 *   iteration:  D[i][e] = sum over c of (F[i][c] - C[e][c])^2;  in rounds, every
 *               unplaced neuron proposes to its nearest cluster that is not full
 *               (ties to the lower cluster index) and a cluster with room r keeps
 *               its r proposals of smallest (D, neuron index), until all d_ff
 *               neurons are placed (each cluster then holds m);  C[e] = mean of
 *               the features of its members.
 * All arithmetic is f64, one rounding per operation, sums in ascending column
 * and neuron order: the result is that of the sequential definition, bit for bit.
 * Outputs (device, caller-allocated): assign [d_ff] int32 (cluster of each neuron
 * in the last assignment), centers [E][d] f64 (the means of that assignment),
 * perm [d_ff] int32 (cluster 0's neurons in ascending order, then cluster 1's,
 * ...; pass it to moe_partition_experts in DISJOINT mode).
 * ws: moe_cluster_workspace_size bytes, zeroed once with moe_workspace_init.
 * An init index out of range or repeated sets MOE_ERR_DEVICE_BADINDEX in the
 * status word of ws (read it with moe_get_device_status) and gives a zero center.
 * Errors: MOE_ERR_INVALID_ARG (NULL pointer, E outside 1..64, n_iter < 1),
 * MOE_ERR_SHAPE (d % 8, d_ff % E), MOE_ERR_DTYPE, MOE_ERR_ALIGN (F, centers and ws
 * 16-byte, index arrays 4-byte), MOE_ERR_WORKSPACE, MOE_ERR_CUDA.
 * Launches 1 + n_iter * (2E + 3) kernels on `stream`. */
size_t moe_cluster_workspace_size(int32_t d, int32_t d_ff, int32_t E);
int moe_cluster_partition(const void *F, int32_t d, int32_t d_ff, int32_t E, int32_t dtype,
                          int32_t n_iter, const int32_t *init_idx, int32_t *assign,
                          double *centers, int32_t *perm, void *ws, size_t ws_bytes,
                          void *stream);

/* The distance step of the clustering alone: D [d_ff][E] f64 (device) receives
 * sum over c of (F[i][c] - centers[e][c])^2 for F [d_ff][d] (dtype) and centers
 * [E][d] f64, with the arithmetic of moe_cluster_partition (one launch).
 * Errors: MOE_ERR_INVALID_ARG, MOE_ERR_SHAPE (d % 8), MOE_ERR_DTYPE,
 * MOE_ERR_ALIGN (F and centers 16-byte, D 8-byte), MOE_ERR_CUDA. */
int moe_cluster_distances(const void *F, int32_t d, int32_t d_ff, int32_t E, int32_t dtype,
                          const double *centers, double *D, void *stream);

/* ---- backward of the layer (bf16 layers, T >= 1) ---------------------------
 * Gradients of l(y) + c * L_balance for a scalar loss l, given dy = dl/dy and c
 * (dLb below); the chain rule of each forward step ("Llama 3 Meets MoE",
 * section 3: the noisy Top-k router and the combine; "LLaMA-MoE v2": the SwiGLU
 * expert of the code sample, L_balance = lambda sum f_i P_i in "门控机制设计"):
 *   combine  d_out[r] = s G_tj dy_t,  dG_tj = s <dy_t, out_r>  (dropped slot: 0)
 *   expert   dh = W2_e^T d_out, du = dh silu(g), dg = dh u silu'(g),
 *            dx_perm = W1_e^T dg + W3_e^T du, dW2_e = sum d_out h^T,
 *            dW1_e = sum dg x^T, dW3_e = sum du x^T (over the expert's rows)
 *   router   Mixtral: dH[idx_j] = G_j (dG_j - sum_l G_l dG_l);
 *            ST: dH_e = p_e (g_e - sum_l p_l g_l), g the dG of the selected experts;
 *            balance: dH_e += p_e (b_e - sum_l p_l b_l), b_e = c lambda f_e / T;
 *            dL = dH, dN = dH eps sigmoid(N);  dW_g = x^T dL, dW_noise = x^T dN,
 *            db = sum_t dL
 *   input    dx_t = sum_j dx_perm[slot_row[t][j]] + W_g dL_t + W_noise dN_t
 * The top-k choice, the dispatch and the counts f carry no gradient.  The forward
 * intermediates (moe_buffers_t of the same batch) are inputs.  bf16 gradients
 * are rounded once from f32 sums; router weight gradients are f32.  g and u are
 * recomputed (x_perm W13_e^T), not stored by the forward.
 * The workspace (moe_backward_workspace_size bytes, zeroed once with
 * moe_workspace_init) holds dGU [T*k][2 m16] (the gate and up gradients of every
 * row) and the router-gradient partials (0.20 GB at T=16384, d=4096, 8 x 1376,
 * k=2); the weight-gradient GEMMs read the activations in place. */
typedef struct {
    const void *dy;    /* [T][d] dl/dy */
    void *dx;          /* [T][d] out: dl/dx (complete: experts and router) */
    float *dWg;        /* [d][E] out */
    float *dWnoise;    /* [d][E] out, NULL iff the layer has no noise term */
    float *dbias;      /* [E] out, NULL iff the layer has no bias */
    void *dW13_e;      /* out, packed like W13_e */
    void *dW2_e;       /* out, packed like W2_e */
    void *d_out;       /* [T*k][d] intermediate: dl/d out */
    float *dG;         /* [T][k] intermediate: dl/d topk_w */
    void *dh;          /* [T*k][m8] intermediate: dl/dh */
    void *dx_perm;     /* [T*k][d] intermediate: the experts' part of dl/dx, per row */
} moe_bwd_buffers_t;

size_t moe_backward_workspace_size(const moe_params_t *p);

/* Combine backward: d_out [T*k][d] (rows of kept slots) and dG [T][k] f32. */
int moe_combine_backward(const moe_params_t *p, const void *dy, const void *out,
                         const int32_t *slot_row, const float *topk_w, void *d_out, float *dG,
                         void *stream);

/* Expert GEMM 2 backward: dh [T*k][m8] and dW2_e (packed).  Transposes W2_e and
 * the activations into the workspace for the tensor-core GEMMs. */
int moe_expert_down_backward(const moe_params_t *p, const void *d_out, const void *h,
                             const int32_t *offsets, const void *W2_e, void *dh, void *dW2_e,
                             void *ws, size_t ws_bytes, void *stream);

/* Expert GEMM 1 + SwiGLU backward: recomputes g, u, forms dg, du, then
 * dx_perm [T*k][d] and dW13_e (packed). */
int moe_expert_up_backward(const moe_params_t *p, const void *x_perm, const void *dh,
                           const int32_t *offsets, const void *W13_e, void *dx_perm,
                           void *dW13_e, void *ws, size_t ws_bytes, void *stream);

/* Router backward and the input gradient: dx [T][d] (overwritten with the full
 * gradient: expert rows through slot_row plus the router term), dWg, dWnoise,
 * dbias (f32).  Wnoise, noise and dWnoise are given together or all NULL; bias
 * and dbias likewise.  counts [E] are the routed counts of the forward. */
int moe_route_backward(const moe_params_t *p, const void *x, const void *Wg, const void *Wnoise,
                       const float *noise, const float *bias, const int32_t *topk_idx,
                       const float *topk_w, const float *dG, const int32_t *counts, float dLb,
                       const void *dx_perm, const int32_t *slot_row, void *dx, float *dWg,
                       float *dWnoise, float *dbias, void *ws, size_t ws_bytes, void *stream);

/* The whole backward: combine, GEMM 2, GEMM 1 + SwiGLU, router and input, on one
 * stream.  b holds the forward's inputs and intermediates of the same batch. */
int moe_backward(const moe_params_t *p, const moe_buffers_t *b, const moe_bwd_buffers_t *g,
                 float dLb, void *ws, size_t ws_bytes, void *stream);

/* Backward of the residual MoE layer y = FFN_S(x) + s sum_j G_j E_j(x) (see
 * moe_forward_residual): the routed part as moe_backward, and the shared block
 * FFN_S, whose output gradient is dy itself, as the backward of a one-expert layer
 * over all T tokens.  b and g as for moe_backward (b->x, b->out etc. of the routed
 * part of the same forward); h_s [T][m_s8] is the shared block's forward
 * activation; outputs dh_s [T][m_s8], dx_s [T][d] (the shared block's part of dx;
 * g->dx receives the whole input gradient), dW13_s / dW2_s (packed like W13_s /
 * W2_s).  ws: moe_backward_residual_workspace_size(p, m_s) bytes. */
size_t moe_backward_residual_workspace_size(const moe_params_t *p, int32_t m_s);
int moe_backward_residual(const moe_params_t *p, const moe_buffers_t *b,
                          const moe_bwd_buffers_t *g, const void *W13_s, const void *W2_s,
                          int32_t m_s, const void *h_s, void *dh_s, void *dx_s, void *dW13_s,
                          void *dW2_s, float dLb, void *ws, size_t ws_bytes, void *stream);

/* ---- expert parallelism --------------------------------------------------
 * "Llama 3 Meets MoE", section "训练框架" (5-D hybrid parallelism: Expert
 * Parallelism places the experts of the MoE layer on different devices; the
 * training configuration uses 8-way expert parallelism).  N ranks, rank r holds
 * T_r tokens and the experts [r E/N, (r+1) E/N) (packed weights of those E/N
 * experts only).  One layer step on rank r:
 *   1. moe_route and moe_dispatch on its own tokens with capacity < 0 (dropless);
 *   2. all ranks gather every rank's counts [E] into counts_all [N][E] and sum
 *      probs_sum and importance (collectives of the caller, e.g. NCCL);
 *   3. moe_ep_plan (host) on counts_all; moe_ep_mask_slots marks the dropped
 *      assignments in slot_row;
 *   4. run send_cnt[e] rows from x_perm row send_row[e] go to rank e / (E/N);
 *      run i = p (E/N) + l from rank p lands at xin row recv_row[i] (recv_cnt[i]
 *      rows); the runs between one pair of ranks pair up in expert order;
 *   5. moe_expert_ffn on xin with E/N experts, k = 1, T = in_offsets[E/N] rows,
 *      offsets in_offsets (copied to the device);
 *   6. the same runs travel back (out rows from recv_row to send_row);
 *   7. moe_combine with the masked slot_row; moe_ep_gate_stats. */
enum { MOE_EP_CAPACITY_GLOBAL = 0, MOE_EP_CAPACITY_LOCAL = 1 };

/* The exchange plan of rank `rank`.  Host-only; every rank computes the same
 * keep_all from the same counts_all.
 *   counts_all [N][E] (host int32): routed (pre-drop) rows of rank p for expert e.
 *   capacity: rows an expert keeps (< 0: no limit).  scope GLOBAL: an expert's
 *     assignments are ranked over the ranks' batches concatenated in rank order
 *     (the layer then equals the one-device layer on that batch); LOCAL: each
 *     rank's batch has its own capacity.  Inside a rank, lower tokens first
 *     ("Llama 3 Meets MoE", section 3 "容量因子").
 * Outputs (host int32, caller-allocated):
 *   keep_all [N][E]  rows of rank p kept for expert e;
 *   send_row [E], send_cnt [E]  this rank's run for expert e: dispatch-output
 *     rows [send_row[e], send_row[e] + send_cnt[e]) (send_row is the prefix sum
 *     of this rank's dropless counts);
 *   recv_row [E], recv_cnt [E]  entry p (E/N) + l: the run of rank p for local
 *     expert l lands at rows [recv_row, recv_row + recv_cnt) of xin;
 *   in_offsets [E/N + 1]  expert-major offsets of xin (ranks ascending inside an
 *     expert); in_offsets[E/N] = rows received.
 * Errors: MOE_ERR_INVALID_ARG (NULL, rank outside [0,N), a negative count, bad
 * scope), MOE_ERR_SHAPE (E outside 1..64, N not dividing E, row totals above
 * 2^30). */
int moe_ep_plan(const int32_t *counts_all, int32_t N, int32_t E, int32_t rank,
                int32_t capacity, int32_t scope, int32_t *keep_all, int32_t *send_row,
                int32_t *send_cnt, int32_t *recv_row, int32_t *recv_cnt, int32_t *in_offsets);

/* Marks the assignments the capacity drops: slot_row[t][j] = -1 where
 * slot_row[t][j] - offsets[topk_idx[t][j]] >= keep[topk_idx[t][j]].  p: this
 * rank's layer (T = its tokens); topk_idx, offsets, slot_row from a dropless
 * moe_dispatch (device); keep [E] host int32 (row `rank` of keep_all).  Entries
 * already -1 or with an index outside [0,E) stay untouched. */
int moe_ep_mask_slots(const moe_params_t *p, const int32_t *topk_idx, const int32_t *offsets,
                      const int32_t *keep, int32_t *slot_row, void *stream);

/* a6 over all ranks: counts[e] = sum_p counts_all[p][e] (device [N][E] -> [E]),
 * then f, P and loss as moe_gate_stats with p->T = the tokens of all ranks and
 * probs_sum the sum over ranks. */
int moe_ep_gate_stats(const moe_params_t *p, const int32_t *counts_all, int32_t N,
                      const float *probs_sum, int32_t *counts, float *f, float *P, float *loss,
                      void *stream);

/* Reads the device status word of `ws` (synchronises `stream`): *status is 0 or
 * one of MOE_ERR_DEVICE_*; clear != 0 resets it to 0 afterwards, together with
 * the workspace's internal launch counters. */
int moe_get_device_status(void *ws, int32_t *status, int32_t clear, void *stream);

/* Time limit, in nanoseconds, of every bounded wait inside the kernels that
 * launch after this call (default 2e9).  0 makes every such wait give up at its
 * first check, which exercises the timeout path; tests use it.  Host-only. */
void moe_set_wait_limit_ns(uint64_t ns);

/* Tile order of the expert GEMMs on 2-SM pairs (4096 rows or more), a tuning knob
 * with no effect on results: the CTA pairs that run at the same time take the
 * output tiles of a band of `rows` rows of an expert (rounded up to 256) across all
 * output columns before the next band, so the band's activations stay in L2 while
 * the weight tiles stream past, and each weight tile is read by the band's pairs at
 * about the same time.  Default 2048; 0 makes the band an expert's whole row range.
 * Launches after the call use it.  Host-only. */
void moe_set_gemm_band_rows(int32_t rows);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
