/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle for the forward pass of a sparse
 * Mixture-of-Experts SwiGLU FFN layer (noisy Top-K routing, capacity dispatch,
 * gate-weighted combine, gate statistics).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file: only the tests, the package smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or constant with the
 * CUDA library; the only thing both sides consume is the seeded input data.
 *
 * Every floating-point input is widened exactly to double (bf16 -> f32 -> f64 is
 * exact) and all arithmetic is done in double.  There is no blocking, fusion or
 * reordering beyond what the formulas state: each function is the definition
 * written out as index loops, so it can be checked against the pages by eye.
 *
 * Sources (web pages; cited by title and section):
 *  [UPCYCLE]  "Llama 3 Meets MoE: Efficient Upcycling" (paper review), section 3
 *             "核心公式": MoE output y = sum_i G(x)_i E_i(x); noisy Top-k routing
 *             G = Softmax(KeepTopK(H, k)), H_i = (x W_g)_i + StandardNormal() *
 *             Softplus((x W_noise)_i); KeepTopK; expert capacity =
 *             tokens per batch / N * CF with overflow tokens excluded; section 5
 *             "路由器算法消融实验": Mixtral type (KeepTopK then Softmax) vs ST type
 *             (Softmax then KeepTopK); section 2 "解决方案概述": experts made by
 *             copying the dense FFN.
 *  [V2]       "LLaMA-MoE v2: 基于后训练混合专家模型的稀疏性探索与技术突破",
 *             section "专家构建方法" (independent neuron partition: split the
 *             intermediate-neuron index set U into M equal disjoint subsets),
 *             section "门控机制设计" (noisy gate, L_balance = lambda sum f_i P_i),
 *             section "重新缩放机制与负载均衡" (y = N/k sum G_i E_i), and the code
 *             sample in "代码实现示例" (SwiGLU expert down(silu(gate(x)) * up(x))).
 *  [HUB]      "从大炼到巧炼：LLaMA-MoE 如何用 MoE 架构让 LLM 变快变省", section
 *             "持续预训练" (Gate Load and Gate Importance are monitored).
 *
 * Readings where the pages are silent or ambiguous (each is also listed in the
 * design notes of the repository):
 *  - the partition permutation is supplied by the caller;
 *  - the noise draw StandardNormal() is a supplied [T,E] tensor;
 *  - the per-expert bias (when given) is added to the clean logits;
 *  - Top-k ties go to the lower expert index; slots are ordered by descending H;
 *  - capacity drops are per (token, expert) assignment, lower token index wins;
 *  - a dropped assignment contributes nothing (the residual outside the layer
 *    carries x); the remaining weights are not renormalised;
 *  - f_i = routed count_i / (T k), P_i = mean over tokens of the full softmax of
 *    the routing logits H (pre-drop);
 *  - gate importance_i = sum over tokens of the final gate weight of expert i;
 *  - softplus is the plain function log(1 + e^z).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* element types of the inputs the oracle reads (its own constants) */
#define ORC_F32 0
#define ORC_BF16 1

#define ORC_MIXTRAL 0
#define ORC_ST 1

#define ORC_DISJOINT 0
#define ORC_COPY 1

#define ORC_EINVAL (-1)

/* Exact widening of one stored element to double. */
static double orc_load(const void *p, int dt, size_t i)
{
    if (dt == ORC_F32)
        return (double)((const float *)p)[i];
    uint32_t u = ((uint32_t)((const uint16_t *)p)[i]) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static size_t orc_esize(int dt) { return dt == ORC_F32 ? 4 : 2; }

int oracle_version(void) { return 1; }

int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Sets the number of host threads later parallel loops use (n >= 1); the per-row
 * arithmetic, and so every result, does not depend on it.  Used to time the oracle
 * on one core. */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    omp_set_num_threads(n < 1 ? 1 : n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------------- */
/* a0. Expert construction [V2 "专家构建方法"; UPCYCLE section 2].
 * DISJOINT: expert e owns intermediate neurons perm[e*m .. (e+1)*m), m = d_ff/E;
 *   W1_e = W1[idx_e, :], W3_e = W3[idx_e, :], W2_e = W2[:, idx_e].
 * COPY: every expert is the whole FFN (m = d_ff).
 * W1, W3 are [d_ff][d] (out x in), W2 is [d][d_ff].  Outputs, in the input's
 * element type: W1e, W3e [E][m][d], W2e [E][d][m].  A pure element gather. */
int oracle_partition(const void *W1, const void *W3, const void *W2, int dt,
                     int d, int d_ff, int E, int mode, const int32_t *perm,
                     void *W1e, void *W3e, void *W2e)
{
    if (d <= 0 || d_ff <= 0 || E <= 0)
        return ORC_EINVAL;
    if (mode == ORC_DISJOINT && (d_ff % E != 0 || perm == NULL))
        return ORC_EINVAL;
    const size_t es = orc_esize(dt);
    const int m = (mode == ORC_DISJOINT) ? d_ff / E : d_ff;
    for (int e = 0; e < E; ++e) {
        for (int i = 0; i < m; ++i) {
            int src = (mode == ORC_DISJOINT) ? perm[(size_t)e * m + i] : i;
            if (src < 0 || src >= d_ff)
                return ORC_EINVAL;
            for (int c = 0; c < d; ++c) {
                size_t s = (size_t)src * d + c;
                size_t o = ((size_t)e * m + i) * d + c;
                memcpy((char *)W1e + o * es, (const char *)W1 + s * es, es);
                memcpy((char *)W3e + o * es, (const char *)W3 + s * es, es);
            }
            for (int r = 0; r < d; ++r) {
                size_t s = (size_t)r * d_ff + src;
                size_t o = ((size_t)e * d + r) * m + i;
                memcpy((char *)W2e + o * es, (const char *)W2 + s * es, es);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Softplus(z) = log(1 + e^z), written in the overflow-free form
 * max(z, 0) + log1p(exp(-|z|)), which is the same function. */
double oracle_softplus(double z) { return (z > 0 ? z : 0.0) + log1p(exp(-fabs(z))); }

/* SiLU (Swish) of the SwiGLU expert [V2 code sample, Expert.act_fn]: z * sigmoid(z). */
double oracle_silu(double z) { return z / (1.0 + exp(-z)); }

/* Ordering used by KeepTopK: larger value first, then lower expert index. */
typedef struct {
    double v;
    int e;
} orc_key;

static int orc_key_cmp(const void *a, const void *b)
{
    const orc_key *x = (const orc_key *)a, *y = (const orc_key *)b;
    if (x->v > y->v)
        return -1;
    if (x->v < y->v)
        return 1;
    return (x->e < y->e) ? -1 : (x->e > y->e);
}

/* KeepTopK [UPCYCLE section 3]: the indices of the k largest entries of h[0..E),
 * found by a full sort of (value desc, index asc).  idx[j] is the j-th largest.
 * Returns ORC_EINVAL if any entry is NaN. */
int oracle_topk(int E, int k, const double *h, int32_t *idx)
{
    if (E <= 0 || k <= 0 || k > E)
        return ORC_EINVAL;
    orc_key *keys = (orc_key *)malloc(sizeof(orc_key) * (size_t)E);
    if (!keys)
        return ORC_EINVAL;
    for (int e = 0; e < E; ++e) {
        if (isnan(h[e])) {
            free(keys);
            return ORC_EINVAL;
        }
        keys[e].v = h[e];
        keys[e].e = e;
    }
    qsort(keys, (size_t)E, sizeof(orc_key), orc_key_cmp);
    for (int j = 0; j < k; ++j)
        idx[j] = keys[j].e;
    free(keys);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* a1. Router [UPCYCLE section 3 and section 5; V2 "门控机制设计"].
 *   L_t = x_t . W_g (+ b)            (W_g stored [d][E])
 *   H_t = L_t + eps_t * Softplus(x_t . W_noise)   if W_noise is given
 *   idx_t = KeepTopK(H_t, k)
 *   Mixtral: G_tj = exp(H_t,idx_j) / sum_{j'<k} exp(H_t,idx_j')
 *   ST:      G_tj = exp(H_t,idx_j) / sum_{e<E} exp(H_t,e)
 * Also (all optional, may be NULL):
 *   H_out [T][E]            the routing logits H,
 *   probs_sum [E]           sum over tokens of softmax(H_t) over all E,
 *   clean_probs_sum [E]     sum over tokens of softmax(L_t) (page-2 sketch variant),
 *   importance [E]          sum over tokens of the gate weight given to expert e.
 * x, W_g, W_noise share element type dt; eps [T][E] and b [E] are f32. */
int oracle_router(int T, int d, int E, int k, int router_type,
                  const void *x, int dt, const void *Wg, const void *Wnoise,
                  const float *eps, const float *bias,
                  double *H_out, int32_t *idx, double *G,
                  double *probs_sum, double *clean_probs_sum, double *importance)
{
    if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E)
        return ORC_EINVAL;
    if (Wnoise != NULL && eps == NULL)
        return ORC_EINVAL;
    int bad = 0;
    double *P = (double *)calloc((size_t)T * E + 1, sizeof(double));
    double *PC = (double *)calloc((size_t)T * E + 1, sizeof(double));
    if (!P || !PC) {
        free(P);
        free(PC);
        return ORC_EINVAL;
    }
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int t = 0; t < T; ++t) {
        double *L = (double *)malloc(sizeof(double) * (size_t)E * 2);
        double *H = L + E;
        for (int e = 0; e < E; ++e) {
            double acc = 0.0, accn = 0.0;
            for (int c = 0; c < d; ++c) {
                double xv = orc_load(x, dt, (size_t)t * d + c);
                acc += xv * orc_load(Wg, dt, (size_t)c * E + e);
                if (Wnoise)
                    accn += xv * orc_load(Wnoise, dt, (size_t)c * E + e);
            }
            if (bias)
                acc += (double)bias[e];
            L[e] = acc;
            H[e] = Wnoise ? acc + (double)eps[(size_t)t * E + e] * oracle_softplus(accn) : acc;
        }
        if (H_out)
            for (int e = 0; e < E; ++e)
                H_out[(size_t)t * E + e] = H[e];
        int32_t *it = idx + (size_t)t * k;
        if (oracle_topk(E, k, H, it) != 0) {
            bad = 1;
            for (int j = 0; j < k; ++j) {
                it[j] = -1;
                G[(size_t)t * k + j] = 0.0;
            }
            free(L);
            continue;
        }
        /* full softmax of H (used by ST weights and by P) */
        double hmax = H[it[0]];
        double zall = 0.0;
        for (int e = 0; e < E; ++e)
            zall += exp(H[e] - hmax);
        for (int e = 0; e < E; ++e)
            P[(size_t)t * E + e] = exp(H[e] - hmax) / zall;
        /* softmax of the clean logits L (page-2 sketch's P) */
        double lmax = L[0];
        for (int e = 1; e < E; ++e)
            if (L[e] > lmax)
                lmax = L[e];
        double zl = 0.0;
        for (int e = 0; e < E; ++e)
            zl += exp(L[e] - lmax);
        for (int e = 0; e < E; ++e)
            PC[(size_t)t * E + e] = exp(L[e] - lmax) / zl;
        if (router_type == ORC_MIXTRAL) {
            double zsel = 0.0;
            for (int j = 0; j < k; ++j)
                zsel += exp(H[it[j]] - hmax);
            for (int j = 0; j < k; ++j)
                G[(size_t)t * k + j] = exp(H[it[j]] - hmax) / zsel;
        } else {
            for (int j = 0; j < k; ++j)
                G[(size_t)t * k + j] = P[(size_t)t * E + it[j]];
        }
        free(L);
    }
    /* token-ordered sums */
    for (int e = 0; e < E; ++e) {
        double s = 0.0, sc = 0.0, si = 0.0;
        for (int t = 0; t < T; ++t) {
            s += P[(size_t)t * E + e];
            sc += PC[(size_t)t * E + e];
            for (int j = 0; j < k; ++j)
                if (idx[(size_t)t * k + j] == e)
                    si += G[(size_t)t * k + j];
        }
        if (probs_sum)
            probs_sum[e] = s;
        if (clean_probs_sum)
            clean_probs_sum[e] = sc;
        if (importance)
            importance[e] = si;
    }
    free(P);
    free(PC);
    return bad ? ORC_EINVAL : 0;
}

/* ------------------------------------------------------------------------- */
/* Expert capacity [UPCYCLE section 3 "容量因子"]: tokens per batch / N * CF,
 * read with tokens = T (not T*k) and rounded up to a whole token.
 * cf < 0 means no limit (returns -1). */
int oracle_capacity(int T, int E, double cf)
{
    if (cf < 0)
        return -1;
    return (int)ceil((double)T / (double)E * cf);
}

/* a2. Dispatch with capacity [UPCYCLE section 3 "容量因子"].
 * Assignments (t, j) are visited in token order (t outer, slot j inner).  Each
 * expert keeps a running count; an assignment whose rank within its expert is
 * >= C is dropped (C < 0: no limit), so the lower token index wins.
 *   counts[e]   routed (pre-drop) assignments of expert e
 *   kept[e]     min(counts[e], C)
 *   offsets[e]  exclusive prefix sum of kept (offsets[E] = R)
 *   row_token[r] token of kept row r; rows are grouped by expert, token-ascending
 *   slot_row[t*k+j] row of assignment (t, j), or -1 if dropped
 * Entries of idx outside [0, E) are treated as dropped.  Returns R. */
int oracle_dispatch(int T, int E, int k, const int32_t *idx, int C,
                    int32_t *counts, int32_t *kept, int32_t *offsets,
                    int32_t *row_token, int32_t *slot_row)
{
    if (T < 0 || E <= 0 || k <= 0)
        return ORC_EINVAL;
    int32_t *rank = (int32_t *)malloc(sizeof(int32_t) * ((size_t)T * k + 1));
    if (!rank)
        return ORC_EINVAL;
    for (int e = 0; e < E; ++e)
        counts[e] = 0;
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = idx[(size_t)t * k + j];
            if (e < 0 || e >= E) {
                rank[(size_t)t * k + j] = -1;
                continue;
            }
            rank[(size_t)t * k + j] = counts[e]++;
        }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) {
        kept[e] = (C < 0 || counts[e] < C) ? counts[e] : C;
        offsets[e + 1] = offsets[e] + kept[e];
    }
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            size_t a = (size_t)t * k + j;
            int e = idx[a];
            int r = rank[a];
            if (r < 0 || r >= kept[e]) {
                slot_row[a] = -1;
                continue;
            }
            int row = offsets[e] + r;
            slot_row[a] = row;
            row_token[row] = t;
        }
    free(rank);
    return offsets[E];
}

/* ------------------------------------------------------------------------- */
/* a3 + a4. One SwiGLU expert applied to n input rows [V2 code sample, Expert]:
 *   out_r = W2_e ( silu(W1_e x_r) * (W3_e x_r) ),  e = expert_of_row[r]
 * Expert weights in the standard layout W1e, W3e [E][m][d], W2e [E][d][m]
 * (element type dt, as produced by oracle_partition).  x_rows [n][d] has type
 * xdt.  out [n][d] double.  If h is not NULL it receives the [n][m] activations. */
int oracle_expert_ffn(int d, int m, int E, const void *W1e, const void *W3e,
                      const void *W2e, int dt, const void *x_rows, int xdt,
                      const int32_t *expert_of_row, int n, double *out, double *h)
{
    if (d <= 0 || m <= 0 || E <= 0 || n < 0)
        return ORC_EINVAL;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int r = 0; r < n; ++r) {
        int e = expert_of_row[r];
        if (e < 0 || e >= E) {
            bad = 1;
            continue;
        }
        double *xr = (double *)malloc(sizeof(double) * ((size_t)d + m));
        double *hr = xr + d;
        for (int c = 0; c < d; ++c)
            xr[c] = orc_load(x_rows, xdt, (size_t)r * d + c);
        for (int i = 0; i < m; ++i) {
            double g = 0.0, u = 0.0;
            size_t base = ((size_t)e * m + i) * d;
            for (int c = 0; c < d; ++c) {
                g += orc_load(W1e, dt, base + c) * xr[c];
                u += orc_load(W3e, dt, base + c) * xr[c];
            }
            hr[i] = oracle_silu(g) * u;
            if (h)
                h[(size_t)r * m + i] = hr[i];
        }
        for (int o = 0; o < d; ++o) {
            double acc = 0.0;
            size_t base = ((size_t)e * d + o) * m;
            for (int i = 0; i < m; ++i)
                acc += orc_load(W2e, dt, base + i) * hr[i];
            out[(size_t)r * d + o] = acc;
        }
        free(xr);
    }
    return bad ? ORC_EINVAL : 0;
}

/* The dense SwiGLU FFN the experts were cut from: y = W2 (silu(W1 x) * (W3 x)),
 * W1, W3 [d_ff][d], W2 [d][d_ff].  x [n][d] (type xdt), y [n][d] double. */
int oracle_dense_ffn(int d, int d_ff, const void *W1, const void *W3, const void *W2,
                     int dt, const void *x, int xdt, int n, double *y)
{
    if (d <= 0 || d_ff <= 0 || n < 0)
        return ORC_EINVAL;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n; ++r) {
        double *xr = (double *)malloc(sizeof(double) * ((size_t)d + d_ff));
        double *hr = xr + d;
        for (int c = 0; c < d; ++c)
            xr[c] = orc_load(x, xdt, (size_t)r * d + c);
        for (int i = 0; i < d_ff; ++i) {
            double g = 0.0, u = 0.0;
            for (int c = 0; c < d; ++c) {
                g += orc_load(W1, dt, (size_t)i * d + c) * xr[c];
                u += orc_load(W3, dt, (size_t)i * d + c) * xr[c];
            }
            hr[i] = oracle_silu(g) * u;
        }
        for (int o = 0; o < d; ++o) {
            double acc = 0.0;
            for (int i = 0; i < d_ff; ++i)
                acc += orc_load(W2, dt, (size_t)o * d_ff + i) * hr[i];
            y[(size_t)r * d + o] = acc;
        }
        free(xr);
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* a5. Gate-weighted combine [UPCYCLE section 3, y = sum_i G(x)_i E_i(x); V2
 * "重新缩放机制", y = N/k sum_i G(x)_i E_i(x)]:
 *   y_t = scale * sum_{j<k, slot kept} G_tj * out_{slot_row[t,j]}
 * out_rows [R][d] double, G [T][k] double, y [T][d] double.  A token whose
 * slots are all dropped gets y_t = 0. */
int oracle_combine(int T, int d, int k, const double *out_rows, const int32_t *slot_row,
                   const double *G, double scale, double *y)
{
    if (T < 0 || d <= 0 || k <= 0)
        return ORC_EINVAL;
    for (int t = 0; t < T; ++t)
        for (int o = 0; o < d; ++o) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) {
                int r = slot_row[(size_t)t * k + j];
                if (r >= 0)
                    acc += G[(size_t)t * k + j] * out_rows[(size_t)r * d + o];
            }
            y[(size_t)t * d + o] = scale * acc;
        }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* a6. Gate statistics [V2 "门控机制设计", L_balance = lambda sum_i f_i P_i;
 * HUB "持续预训练": Gate Load, Gate Importance].
 *   f_e = counts_e / (T k),  P_e = probs_sum_e / T,  L = lambda sum_e f_e P_e.
 * T = 0 gives f = P = 0 and L = 0. */
int oracle_gate_stats(int T, int E, int k, const int32_t *counts, const double *probs_sum,
                      double lambda, double *f, double *P, double *L)
{
    if (T < 0 || E <= 0 || k <= 0)
        return ORC_EINVAL;
    double s = 0.0;
    for (int e = 0; e < E; ++e) {
        f[e] = T > 0 ? (double)counts[e] / ((double)T * k) : 0.0;
        P[e] = T > 0 ? probs_sum[e] / (double)T : 0.0;
        s += f[e] * P[e];
    }
    *L = lambda * s;
    return 0;
}

/* The load-balance loss as the V2 code sample computes it (information only):
 * frequency = per-expert sum of gate weights normalised to sum 1 (with the
 * sample's 1e-6 guard), P = mean softmax of the clean logits, times E. */
int oracle_balance_sketch(int T, int E, int k, const int32_t *idx, const double *G,
                          const double *clean_probs_sum, double *L)
{
    if (T <= 0 || E <= 0 || k <= 0)
        return ORC_EINVAL;
    double *w = (double *)calloc((size_t)E, sizeof(double));
    double tot = 0.0, s = 0.0;
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = idx[(size_t)t * k + j];
            if (e >= 0 && e < E)
                w[e] += G[(size_t)t * k + j];
        }
    for (int e = 0; e < E; ++e)
        tot += w[e];
    for (int e = 0; e < E; ++e)
        s += (w[e] / (tot + 1e-6)) * (clean_probs_sum[e] / (double)T);
    *L = s * (double)E;
    free(w);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* f4. Clustering partition [V2 "专家构建方法", IndependentClustering: k-means
 * over the neurons' weight vectors, the neurons of one cluster form one expert;
 * the subsets are of equal size m = d_ff / E].
 *
 * Readings (the page names k-means and equal sizes, nothing more):
 *  - the feature of neuron i is row i of F [d_ff][d] (the caller passes W1);
 *  - the E initial centers are the features of E distinct caller-chosen neurons;
 *  - one iteration = assignment step, then center step;
 *  - distance D[i][e] = sum over c of (F[i][c] - C[e][c])^2, summed in
 *    ascending c, each difference, square and sum rounded (no fused multiply-add);
 *  - the assignment step keeps every cluster at m neurons: in rounds, every
 *    unassigned neuron proposes to its nearest cluster that is not full (ties
 *    to the lower cluster index); a cluster with room r accepts its r proposals
 *    of smallest (D, neuron index) and its acceptances are final; repeat until
 *    every neuron is placed (at most E rounds: a round either places every
 *    proposer or fills a cluster);
 *  - the center step sets C[e] to the mean of its m members' features, summed in
 *    ascending neuron index, then divided by m.
 * Outputs after n_iter iterations: assign[i] (cluster of neuron i in the last
 * assignment), centers [E][d] (after the last center step, so the means of
 * that assignment), perm [d_ff] (cluster 0's neurons ascending, then cluster
 * 1's, ...: the permutation a0 takes). */
/* Squared Euclidean distance of every feature row to every center, summed in
 * ascending column order: D[i][e] = sum_c (F[i][c] - C[e][c])^2. */
int oracle_sqdist(const void *F, int dt, int d, int d_ff, int E, const double *C, double *D)
{
    if (d <= 0 || d_ff <= 0 || E <= 0)
        return ORC_EINVAL;
#pragma omp parallel for schedule(static)
    for (int i = 0; i < d_ff; ++i)
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int c = 0; c < d; ++c) {
                double diff = orc_load(F, dt, (size_t)i * d + c) - C[(size_t)e * d + c];
                double sq = diff * diff;
                s = s + sq;
            }
            D[(size_t)i * E + e] = s;
        }
    return 0;
}

static const double *orc_sort_keys;

static int orc_cmp_key(const void *a, const void *b)
{
    int i = *(const int32_t *)a, j = *(const int32_t *)b;
    double di = orc_sort_keys[i], dj = orc_sort_keys[j];
    if (di < dj)
        return -1;
    if (di > dj)
        return 1;
    return (i > j) - (i < j);
}

int oracle_cluster(const void *F, int dt, int d, int d_ff, int E, int n_iter,
                   const int32_t *init, int32_t *assign, double *centers, int32_t *perm)
{
    if (d <= 0 || d_ff <= 0 || E <= 0 || n_iter < 1 || d_ff % E != 0)
        return ORC_EINVAL;
    const int m = d_ff / E;
    for (int e = 0; e < E; ++e) {
        if (init[e] < 0 || init[e] >= d_ff)
            return ORC_EINVAL;
        for (int f = 0; f < e; ++f)
            if (init[f] == init[e])
                return ORC_EINVAL;
    }
    double *D = (double *)malloc((size_t)d_ff * E * sizeof(double));
    double *key = (double *)malloc((size_t)d_ff * sizeof(double));
    int32_t *target = (int32_t *)malloc((size_t)d_ff * sizeof(int32_t));
    int32_t *cand = (int32_t *)malloc((size_t)d_ff * sizeof(int32_t));
    int *fill = (int *)malloc((size_t)E * sizeof(int));
    if (!D || !key || !target || !cand || !fill) {
        free(D), free(key), free(target), free(cand), free(fill);
        return ORC_EINVAL;
    }
    for (int e = 0; e < E; ++e)
        for (int c = 0; c < d; ++c)
            centers[(size_t)e * d + c] = orc_load(F, dt, (size_t)init[e] * d + c);

    for (int it = 0; it < n_iter; ++it) {
        oracle_sqdist(F, dt, d, d_ff, E, centers, D);
        /* balanced assignment in rounds */
        for (int i = 0; i < d_ff; ++i)
            assign[i] = -1;
        for (int e = 0; e < E; ++e)
            fill[e] = 0;
        int left = d_ff;
        while (left > 0) {
            for (int i = 0; i < d_ff; ++i) {
                target[i] = -1;
                if (assign[i] >= 0)
                    continue;
                for (int e = 0; e < E; ++e)
                    if (fill[e] < m && (target[i] < 0 || D[(size_t)i * E + e] < D[(size_t)i * E + target[i]]))
                        target[i] = e;
            }
            for (int e = 0; e < E; ++e) {
                int n = 0;
                for (int i = 0; i < d_ff; ++i)
                    if (target[i] == e) {
                        cand[n++] = i;
                        key[i] = D[(size_t)i * E + e];
                    }
                orc_sort_keys = key;
                qsort(cand, (size_t)n, sizeof(int32_t), orc_cmp_key);
                int room = m - fill[e];
                for (int r = 0; r < n && r < room; ++r) {
                    assign[cand[r]] = e;
                    fill[e] += 1;
                    left -= 1;
                }
            }
        }
        /* centers: mean of the members, ascending neuron index */
        for (int e = 0; e < E; ++e)
            for (int c = 0; c < d; ++c) {
                double s = 0.0;
                for (int i = 0; i < d_ff; ++i)
                    if (assign[i] == e)
                        s = s + orc_load(F, dt, (size_t)i * d + c);
                centers[(size_t)e * d + c] = s / (double)m;
            }
    }
    int pos = 0;
    for (int e = 0; e < E; ++e)
        for (int i = 0; i < d_ff; ++i)
            if (assign[i] == e)
                perm[pos++] = i;
    free(D), free(key), free(target), free(cand), free(fill);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* f1. Backward of the layer.  The loss is l(y) + c * L_balance; the caller gives
 * dy = dl/dy [T][d] and c.  Every function below is the chain rule of one forward
 * step written out in f64 loops, in the forward's notation:
 *   combine   y_t = s sum_j G_tj out_{r(t,j)}
 *   expert    g = W1_e x, u = W3_e x, h = silu(g) * u, out = W2_e h
 *   router    L = x W_g + b, N = x W_noise, H = L + eps * softplus(N),
 *             G = softmax over the k selected H (Mixtral) or softmax(H)_idx (ST),
 *             P_e = mean_t softmax(H_t)_e, L_balance = lambda sum_e f_e P_e
 * The top-k choice, the dispatch and f_e (counts) are piecewise constant and
 * carry no gradient; a dropped slot gets dG = 0. */

/* Combine backward: for every kept slot (t, j) with row r = slot_row[t][j]:
 *   d_out[r] = s * G_tj * dy_t,   dG_tj = s * <dy_t, out_r>;   dropped: dG_tj = 0.
 * out_rows / d_out [R][d], dy [T][d], G / dG [T][k]. */
int oracle_combine_backward(int T, int d, int k, const double *out_rows, const int32_t *slot_row,
                            const double *G, double scale, const double *dy, double *d_out,
                            double *dG)
{
    if (T < 0 || d <= 0 || k <= 0)
        return ORC_EINVAL;
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            size_t a = (size_t)t * k + j;
            int r = slot_row[a];
            if (r < 0) {
                dG[a] = 0.0;
                continue;
            }
            double dot = 0.0;
            for (int o = 0; o < d; ++o) {
                dot += dy[(size_t)t * d + o] * out_rows[(size_t)r * d + o];
                d_out[(size_t)r * d + o] = scale * G[a] * dy[(size_t)t * d + o];
            }
            dG[a] = scale * dot;
        }
    return 0;
}

/* Derivative of silu: sigma(z) (1 + z (1 - sigma(z))). */
static double orc_dsilu(double z)
{
    double s = 1.0 / (1.0 + exp(-z));
    return s * (1.0 + z * (1.0 - s));
}

/* Expert backward for n rows (row r belongs to expert expert_of_row[r]):
 *   dh = W2_e^T d_out,  du = dh * silu(g),  dg = dh * u * silu'(g),
 *   dx_r = W1_e^T dg + W3_e^T du,
 *   dW2_e += d_out h^T,  dW1_e += dg x^T,  dW3_e += du x^T  (rows summed in ascending r).
 * Layouts as oracle_expert_ffn: W1e, W3e, dW1e, dW3e [E][m][d]; W2e, dW2e [E][d][m];
 * x_rows [n][d] (type xdt); d_out, dx_rows [n][d]; optional dh, dg, du [n][m]. */
int oracle_expert_ffn_backward(int d, int m, int E, const void *W1e, const void *W3e,
                               const void *W2e, int dt, const void *x_rows, int xdt,
                               const int32_t *expert_of_row, int n, const double *d_out,
                               double *dx_rows, double *dW1e, double *dW3e, double *dW2e,
                               double *dh_out, double *dg_out, double *du_out)
{
    if (d <= 0 || m <= 0 || E <= 0 || n < 0)
        return ORC_EINVAL;
    for (int r = 0; r < n; ++r)
        if (expert_of_row[r] < 0 || expert_of_row[r] >= E)
            return ORC_EINVAL;
    double *X = (double *)malloc(sizeof(double) * ((size_t)n * d + 1));
    double *Hh = (double *)malloc(sizeof(double) * ((size_t)n * m + 1));
    double *Dg = (double *)malloc(sizeof(double) * ((size_t)n * m + 1));
    double *Du = (double *)malloc(sizeof(double) * ((size_t)n * m + 1));
    if (!X || !Hh || !Dg || !Du) {
        free(X), free(Hh), free(Dg), free(Du);
        return ORC_EINVAL;
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n; ++r) {
        int e = expert_of_row[r];
        double *xr = X + (size_t)r * d;
        for (int c = 0; c < d; ++c)
            xr[c] = orc_load(x_rows, xdt, (size_t)r * d + c);
        for (int i = 0; i < m; ++i) {
            double g = 0.0, u = 0.0, dh = 0.0;
            size_t base = ((size_t)e * m + i) * d;
            for (int c = 0; c < d; ++c) {
                g += orc_load(W1e, dt, base + c) * xr[c];
                u += orc_load(W3e, dt, base + c) * xr[c];
            }
            for (int o = 0; o < d; ++o)
                dh += orc_load(W2e, dt, ((size_t)e * d + o) * m + i) * d_out[(size_t)r * d + o];
            Hh[(size_t)r * m + i] = oracle_silu(g) * u;
            Du[(size_t)r * m + i] = dh * oracle_silu(g);
            Dg[(size_t)r * m + i] = dh * u * orc_dsilu(g);
            if (dh_out)
                dh_out[(size_t)r * m + i] = dh;
        }
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int i = 0; i < m; ++i) {
                size_t w = ((size_t)e * m + i) * d + c;
                acc += orc_load(W1e, dt, w) * Dg[(size_t)r * m + i] +
                       orc_load(W3e, dt, w) * Du[(size_t)r * m + i];
            }
            dx_rows[(size_t)r * d + c] = acc;
        }
    }
    /* weight gradients: each entry sums the rows of its expert in ascending order */
    int32_t *rows_of = (int32_t *)malloc(sizeof(int32_t) * ((size_t)n + 1));
    int32_t *start = (int32_t *)calloc((size_t)E + 1, sizeof(int32_t));
    if (!rows_of || !start) {
        free(X), free(Hh), free(Dg), free(Du), free(rows_of), free(start);
        return ORC_EINVAL;
    }
    for (int e = 0, pos = 0; e < E; ++e) {
        start[e] = pos;
        for (int r = 0; r < n; ++r)
            if (expert_of_row[r] == e)
                rows_of[pos++] = r;
        start[e + 1] = pos;
    }
#pragma omp parallel for schedule(static) collapse(2)
    for (int e = 0; e < E; ++e)
        for (int i = 0; i < m; ++i) {
            for (int c = 0; c < d; ++c) {
                double a1 = 0.0, a3 = 0.0;
                for (int q = start[e]; q < start[e + 1]; ++q) {
                    int r = rows_of[q];
                    a1 += Dg[(size_t)r * m + i] * X[(size_t)r * d + c];
                    a3 += Du[(size_t)r * m + i] * X[(size_t)r * d + c];
                }
                dW1e[((size_t)e * m + i) * d + c] = a1;
                dW3e[((size_t)e * m + i) * d + c] = a3;
            }
            for (int o = 0; o < d; ++o) {
                double a2 = 0.0;
                for (int q = start[e]; q < start[e + 1]; ++q) {
                    int r = rows_of[q];
                    a2 += d_out[(size_t)r * d + o] * Hh[(size_t)r * m + i];
                }
                dW2e[((size_t)e * d + o) * m + i] = a2;
            }
        }
    free(rows_of), free(start);
    if (dg_out)
        memcpy(dg_out, Dg, sizeof(double) * (size_t)n * m);
    if (du_out)
        memcpy(du_out, Du, sizeof(double) * (size_t)n * m);
    free(X), free(Hh), free(Dg), free(Du);
    return 0;
}

/* Router backward.  Recomputes L, N, H and p = softmax(H) per token (as
 * oracle_router), then with dG [T][k] (from the combine backward), the forward's
 * idx / G [T][k], counts [E] (routed, pre-drop) and c = dLb:
 *   Mixtral: S = sum_j G_j dG_j,  dH[idx_j] += G_j (dG_j - S)
 *   ST:      g_e = dG_j if e = idx_j else 0,  S = sum_e p_e g_e,  dH_e += p_e (g_e - S)
 *   balance: b_e = c lambda f_e / T,  B = sum_e p_e b_e,  dH_e += p_e (b_e - B)
 *   dL = dH,  dN = dH * eps * sigmoid(N)
 *   dx_t += W_g dL_t + W_noise dN_t,  dW_g = x^T dL,  dW_noise = x^T dN,  db = sum_t dL_t
 * dx [T][d] is ADDED to; dWg, dWnoise [d][E], dbias [E] are written (NULL when the
 * input is absent); dH_out [T][E] and dN_out [T][E] optional. */
int oracle_router_backward_norm(int T, int T_norm, int d, int E, int k, int router_type,
                                const void *x, int dt, const void *Wg, const void *Wnoise,
                                const float *eps, const float *bias, const int32_t *idx,
                                const double *G, const double *dG, const int32_t *counts,
                                double lambda, double dLb, double *dx, double *dWg,
                                double *dWnoise, double *dbias, double *dH_out, double *dN_out);

int oracle_router_backward(int T, int d, int E, int k, int router_type, const void *x, int dt,
                           const void *Wg, const void *Wnoise, const float *eps, const float *bias,
                           const int32_t *idx, const double *G, const double *dG,
                           const int32_t *counts, double lambda, double dLb, double *dx,
                           double *dWg, double *dWnoise, double *dbias, double *dH_out,
                           double *dN_out)
{
    return oracle_router_backward_norm(T, T, d, E, k, router_type, x, dt, Wg, Wnoise, eps, bias,
                                       idx, G, dG, counts, lambda, dLb, dx, dWg, dWnoise, dbias,
                                       dH_out, dN_out);
}

/* The same for a subset of the batch's tokens: the T rows given are some of the
 * T_norm tokens of the batch, whose counts f_e = counts_e / (T_norm k) and 1/T_norm
 * the balance term uses.  (The weight-gradient outputs then cover only these rows.) */
int oracle_router_backward_norm(int T, int T_norm, int d, int E, int k, int router_type,
                                const void *x, int dt, const void *Wg, const void *Wnoise,
                                const float *eps, const float *bias, const int32_t *idx,
                                const double *G, const double *dG, const int32_t *counts,
                                double lambda, double dLb, double *dx, double *dWg,
                                double *dWnoise, double *dbias, double *dH_out, double *dN_out)
{
    if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E)
        return ORC_EINVAL;
    if (Wnoise != NULL && eps == NULL)
        return ORC_EINVAL;
    double *DL = (double *)calloc((size_t)T * E + 1, sizeof(double));
    double *DN = (double *)calloc((size_t)T * E + 1, sizeof(double));
    if (!DL || !DN) {
        free(DL), free(DN);
        return ORC_EINVAL;
    }
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        double *L = (double *)malloc(sizeof(double) * (size_t)E * 5);
        double *N = L + E, *H = N + E, *p = H + E, *dH = p + E;
        for (int e = 0; e < E; ++e) {
            double acc = 0.0, accn = 0.0;
            for (int c = 0; c < d; ++c) {
                double xv = orc_load(x, dt, (size_t)t * d + c);
                acc += xv * orc_load(Wg, dt, (size_t)c * E + e);
                if (Wnoise)
                    accn += xv * orc_load(Wnoise, dt, (size_t)c * E + e);
            }
            if (bias)
                acc += (double)bias[e];
            L[e] = acc;
            N[e] = accn;
            H[e] = Wnoise ? acc + (double)eps[(size_t)t * E + e] * oracle_softplus(accn) : acc;
        }
        double hmax = H[0];
        for (int e = 1; e < E; ++e)
            if (H[e] > hmax)
                hmax = H[e];
        double z = 0.0;
        for (int e = 0; e < E; ++e)
            z += exp(H[e] - hmax);
        for (int e = 0; e < E; ++e) {
            p[e] = exp(H[e] - hmax) / z;
            dH[e] = 0.0;
        }
        const int32_t *it = idx + (size_t)t * k;
        const double *Gt = G + (size_t)t * k, *dGt = dG + (size_t)t * k;
        if (router_type == ORC_MIXTRAL) {
            double S = 0.0;
            for (int j = 0; j < k; ++j)
                S += Gt[j] * dGt[j];
            for (int j = 0; j < k; ++j)
                if (it[j] >= 0 && it[j] < E)
                    dH[it[j]] += Gt[j] * (dGt[j] - S);
        } else {
            double S = 0.0;
            for (int j = 0; j < k; ++j)
                if (it[j] >= 0 && it[j] < E)
                    S += p[it[j]] * dGt[j];
            for (int e = 0; e < E; ++e) {
                double ge = 0.0;
                for (int j = 0; j < k; ++j)
                    if (it[j] == e)
                        ge += dGt[j];
                dH[e] += p[e] * (ge - S);
            }
        }
        if (lambda != 0.0 && dLb != 0.0 && T_norm > 0) {
            double B = 0.0;
            for (int e = 0; e < E; ++e)
                B += p[e] * (dLb * lambda * ((double)counts[e] / ((double)T_norm * k)) /
                             (double)T_norm);
            for (int e = 0; e < E; ++e) {
                double be = dLb * lambda * ((double)counts[e] / ((double)T_norm * k)) /
                            (double)T_norm;
                dH[e] += p[e] * (be - B);
            }
        }
        for (int e = 0; e < E; ++e) {
            DL[(size_t)t * E + e] = dH[e];
            if (Wnoise) {
                double sg = 1.0 / (1.0 + exp(-N[e]));
                DN[(size_t)t * E + e] = dH[e] * (double)eps[(size_t)t * E + e] * sg;
            }
            if (dH_out)
                dH_out[(size_t)t * E + e] = dH[e];
            if (dN_out)
                dN_out[(size_t)t * E + e] = DN[(size_t)t * E + e];
        }
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int e = 0; e < E; ++e) {
                acc += orc_load(Wg, dt, (size_t)c * E + e) * DL[(size_t)t * E + e];
                if (Wnoise)
                    acc += orc_load(Wnoise, dt, (size_t)c * E + e) * DN[(size_t)t * E + e];
            }
            dx[(size_t)t * d + c] += acc;
        }
        free(L);
    }
#pragma omp parallel for schedule(static)
    for (int c = 0; c < d; ++c)
        for (int e = 0; e < E; ++e) {
            double a = 0.0, an = 0.0;
            for (int t = 0; t < T; ++t) {
                double xv = orc_load(x, dt, (size_t)t * d + c);
                a += xv * DL[(size_t)t * E + e];
                an += xv * DN[(size_t)t * E + e];
            }
            dWg[(size_t)c * E + e] = a;
            if (dWnoise)
                dWnoise[(size_t)c * E + e] = an;
        }
    if (dbias)
        for (int e = 0; e < E; ++e) {
            double a = 0.0;
            for (int t = 0; t < T; ++t)
                a += DL[(size_t)t * E + e];
            dbias[e] = a;
        }
    free(DL), free(DN);
    return 0;
}

/* One neuron's weight gradients over the n rows of one expert (a sample of what
 * oracle_expert_ffn_backward computes for every neuron):
 *   dW1[c] = sum_r dg_r x_r[c],  dW3[c] = sum_r du_r x_r[c],  dW2[o] = sum_r d_out_r[o] h_r
 * with g = W1_i . x_r, u = W3_i . x_r, h = silu(g) u, dh = sum_o W2[o][i] d_out_r[o],
 * du = dh silu(g), dg = dh u silu'(g), rows in ascending order.  W1i, W3i [d] and
 * the column W2[:, i] given as W2e [d][m] with the neuron index i (element type dt);
 * x_rows [n][d] (type xdt); d_out [n][d] f64. */
int oracle_neuron_wgrad(int d, int m, int i, const void *W1i, const void *W3i, const void *W2e,
                        int dt, const void *x_rows, int xdt, int n, const double *d_out,
                        double *dW1, double *dW3, double *dW2)
{
    if (d <= 0 || m <= 0 || i < 0 || i >= m || n < 0)
        return ORC_EINVAL;
    for (int c = 0; c < d; ++c)
        dW1[c] = dW3[c] = dW2[c] = 0.0;
    for (int r = 0; r < n; ++r) {
        double g = 0.0, u = 0.0, dh = 0.0;
        for (int c = 0; c < d; ++c) {
            double xv = orc_load(x_rows, xdt, (size_t)r * d + c);
            g += orc_load(W1i, dt, (size_t)c) * xv;
            u += orc_load(W3i, dt, (size_t)c) * xv;
        }
        for (int o = 0; o < d; ++o)
            dh += orc_load(W2e, dt, (size_t)o * m + i) * d_out[(size_t)r * d + o];
        double h = oracle_silu(g) * u;
        double du = dh * oracle_silu(g);
        double dg = dh * u * orc_dsilu(g);
        for (int c = 0; c < d; ++c) {
            double xv = orc_load(x_rows, xdt, (size_t)r * d + c);
            dW1[c] = dW1[c] + dg * xv;
            dW3[c] = dW3[c] + du * xv;
            dW2[c] = dW2[c] + d_out[(size_t)r * d + c] * h;
        }
    }
    return 0;
}
