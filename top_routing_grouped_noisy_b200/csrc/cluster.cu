// cluster.cu -- clustering partition of the FFN neurons ("LLaMA-MoE v2",
// section "专家构建方法", IndependentClustering: k-means over the neurons' weight
// vectors, the neurons of one cluster form one expert, E subsets of equal size
// m = d_ff / E).  The result is the neuron permutation that a0
// (moe_partition_experts, DISJOINT) takes.
//
// One iteration:
//   distances  D[i][e] = sum_c (F[i][c] - C[e][c])^2
//   assignment in rounds: every unplaced neuron proposes to its nearest cluster
//              that is not full (ties to the lower cluster index); a cluster with
//              room r keeps its r proposals of smallest (D, neuron index); kept
//              neurons stay; at most E rounds (a round places every proposer or
//              fills a cluster)
//   permutation: cluster 0's neurons ascending, then cluster 1's, ...
//   centers    C[e] = mean of the members' features, summed in ascending index
// All arithmetic is f64 with one rounding per operation (the _rn intrinsics keep
// the compiler from contracting into fused multiply-adds) and every sum runs in
// ascending column / neuron order, so distances, decisions and centers equal
// those of the plain sequential definition bit for bit.
//
// Off the per-batch path: run once per weight set, like a0.
#include <cstdio>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kDistRows = 32;   // neurons per CTA of the distance kernel (one per lane)
constexpr int kDistCols = 64;   // feature columns staged per step

struct ClusterLayout {
    size_t D, keys, list, cnt, fill, total;
};

size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

ClusterLayout cluster_layout(int d_ff, int E)
{
    ClusterLayout L;
    size_t o = kWsHeader;
    L.D = o;
    o = up256(o + (size_t)d_ff * E * sizeof(double));
    L.keys = o;
    o = up256(o + (size_t)E * d_ff * sizeof(double));
    L.list = o;
    o = up256(o + (size_t)E * d_ff * sizeof(int32_t));
    L.cnt = o;  // cnt [E rounds][E] then fill [E+1][E], contiguous
    L.fill = o + (size_t)E * E * sizeof(int32_t);
    o = up256(L.fill + (size_t)(E + 1) * E * sizeof(int32_t));
    L.total = o;
    return L;
}

}  // namespace

// Initial centers: the features of the E caller-chosen neurons.  An index out of
// range or repeated sets MOE_ERR_DEVICE_BADINDEX and gives a zero center.
template <typename E_T>
__global__ void __launch_bounds__(256) cluster_init_kernel(const E_T *__restrict__ F, int d,
                                                           int d_ff, int E,
                                                           const int32_t *__restrict__ init,
                                                           double *__restrict__ centers,
                                                           int32_t *status)
{
    pdl_wait();
    pdl_trigger();
    const int e = blockIdx.x;
    const int src = init[e];
    bool good = src >= 0 && src < d_ff;
    for (int f = 0; f < e; ++f)
        good = good && init[f] != src;
    if (!good && blockIdx.y == 0 && threadIdx.x == 0)
        set_status(status, MOE_ERR_DEVICE_BADINDEX);
    const int c = blockIdx.y * blockDim.x + threadIdx.x;
    if (c < d)
        centers[(size_t)e * d + c] = good ? (double)to_f32(F[(size_t)src * d + c]) : 0.0;
}

// Distances of 32 neurons (lane = neuron) to every center.  Each lane carries
// two clusters (a pair), warp w the pairs w, w+NW, ... (NJ pairs), so every
// feature value read from shared memory feeds two independent sums.  Inside the
// clustering the kernel also starts the iteration's assignment (assign and
// counters non-null): every neuron unplaced, round counters zero.
//
// Columns are staged 64 at a time as f64: the feature tile Fs [32][64] (row
// stride 66 doubles; a warp writes one row per store, lanes on consecutive
// column pairs, and a lane later reads its own row in 16-byte pairs, both
// without bank conflicts) and the center tile Cs [E][64] (16-byte broadcasts).
// The global loads of tile t+1 are issued into registers before the sums of
// tile t run.  The last tile is zero-padded in both: a padded column adds
// (0 - 0)^2 = +0 to a non-negative sum, which leaves it unchanged, so the inner
// loop always runs 64 columns.
constexpr int kFsStride = kDistCols + 2;

template <typename E_T, int NW, int NJ>
__global__ void __launch_bounds__(NW * 32) cluster_dist_kernel(
    const E_T *__restrict__ F, int d, int d_ff, int E, const double *__restrict__ centers,
    double *__restrict__ D, int32_t *__restrict__ assign, int32_t *__restrict__ counters)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(16) double cl_smem[];
    double *Fs = cl_smem;                           // [32][kFsStride]
    double *Cs = cl_smem + kDistRows * kFsStride;   // [E][kDistCols]
    constexpr int RPW = kDistRows / NW;             // feature rows staged per warp
    constexpr int CPT = 2 * NJ;  // center column pairs per thread: E <= 2 * NW * NJ
    using FReg = typename std::conditional<sizeof(E_T) == 2, uint32_t, float2>::type;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int i0 = blockIdx.x * kDistRows;
    const int cpt = (E + NW - 1) / NW;

    if (counters != nullptr && blockIdx.x == 0)
        for (int j = tid; j < E * E + (E + 1) * E; j += NW * 32)
            counters[j] = 0;
    if (assign != nullptr && warp == 0 && i0 + lane < d_ff)
        assign[i0 + lane] = -1;

    FReg freg[RPW];
    double2 creg[CPT];
    auto fetch = [&](int c0) {
        const int col = c0 + 2 * lane;  // d is even: a column pair is all in or all out
#pragma unroll
        for (int k = 0; k < RPW; ++k) {
            const int r = warp + NW * k;
            if constexpr (sizeof(E_T) == 2)
                freg[k] = 0u;
            else
                freg[k] = make_float2(0.f, 0.f);
            if (i0 + r < d_ff && col < d) {
                const E_T *src = F + (size_t)(i0 + r) * d + col;
                if constexpr (sizeof(E_T) == 2)
                    freg[k] = __ldg(reinterpret_cast<const unsigned int *>(src));
                else
                    freg[k] = __ldg(reinterpret_cast<const float2 *>(src));
            }
        }
#pragma unroll
        for (int k = 0; k < CPT; ++k) {
            const int v = tid + NW * 32 * k;  // v / 32 = cluster, lane = column pair
            creg[k] = make_double2(0.0, 0.0);
            if (k < cpt && v / 32 < E && col < d)
                creg[k] = *reinterpret_cast<const double2 *>(centers + (size_t)(v / 32) * d + col);
        }
    };
    auto stash = [&]() {
#pragma unroll
        for (int k = 0; k < RPW; ++k) {
            double2 f2;
            if constexpr (sizeof(E_T) == 2)
                f2 = make_double2((double)__uint_as_float(freg[k] << 16),
                                  (double)__uint_as_float(freg[k] & 0xffff0000u));
            else
                f2 = make_double2((double)freg[k].x, (double)freg[k].y);
            *reinterpret_cast<double2 *>(Fs + (warp + NW * k) * kFsStride + 2 * lane) = f2;
        }
#pragma unroll
        for (int k = 0; k < CPT; ++k) {
            const int v = tid + NW * 32 * k;
            if (k < cpt && v / 32 < E)
                *reinterpret_cast<double2 *>(Cs + (v / 32) * kDistCols + 2 * lane) = creg[k];
        }
    };

    double acc[NJ][2];
#pragma unroll
    for (int j = 0; j < NJ; ++j)
        acc[j][0] = acc[j][1] = 0.0;

    fetch(0);
    for (int c0 = 0; c0 < d; c0 += kDistCols) {
        __syncthreads();  // the previous tile is consumed
        stash();
        __syncthreads();
        if (c0 + kDistCols < d)
            fetch(c0 + kDistCols);
        const double2 *fr = reinterpret_cast<const double2 *>(Fs + lane * kFsStride);
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            const int e0 = 2 * (warp + NW * j);
            if (e0 < E) {
                const bool two = e0 + 1 < E;
                const double2 *c0r = reinterpret_cast<const double2 *>(Cs + e0 * kDistCols);
                const double2 *c1r =
                    reinterpret_cast<const double2 *>(Cs + (two ? e0 + 1 : e0) * kDistCols);
                double a0 = acc[j][0], a1 = acc[j][1];
#pragma unroll
                for (int h = 0; h < kDistCols / 2; ++h) {
                    const double2 f2 = fr[h], p = c0r[h], q = c1r[h];
                    double t = __dsub_rn(f2.x, p.x);
                    a0 = __dadd_rn(a0, __dmul_rn(t, t));
                    t = __dsub_rn(f2.x, q.x);
                    a1 = __dadd_rn(a1, __dmul_rn(t, t));
                    t = __dsub_rn(f2.y, p.y);
                    a0 = __dadd_rn(a0, __dmul_rn(t, t));
                    t = __dsub_rn(f2.y, q.y);
                    a1 = __dadd_rn(a1, __dmul_rn(t, t));
                }
                acc[j][0] = a0;
                acc[j][1] = a1;
            }
        }
    }
    const int i = i0 + lane;
    if (i < d_ff) {
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            const int e0 = 2 * (warp + NW * j);
            if (e0 < E)
                D[(size_t)i * E + e0] = acc[j][0];
            if (e0 + 1 < E)
                D[(size_t)i * E + e0 + 1] = acc[j][1];
        }
    }
}

// Round r, proposals: each unplaced neuron appends itself to the list of its
// nearest non-full cluster.  The list order is arbitrary; acceptance ranks by
// (distance, index), so it does not matter.
__global__ void __launch_bounds__(256) cluster_propose_kernel(
    const double *__restrict__ D, int d_ff, int E, int m, int r, const int32_t *__restrict__ assign,
    int32_t *__restrict__ cnt, const int32_t *__restrict__ fill, int32_t *__restrict__ list,
    double *__restrict__ keys, int32_t *status)
{
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t s_fill[MOE_MAX_EXPERTS];
    if (threadIdx.x < E)
        s_fill[threadIdx.x] = fill[r * E + threadIdx.x];
    __syncthreads();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= d_ff || assign[i] >= 0)
        return;
    int best = -1;
    double bd = 0.0;
    for (int e = 0; e < E; ++e) {
        if (s_fill[e] >= m)
            continue;
        const double v = D[(size_t)i * E + e];
        if (best < 0 || v < bd) {
            best = e;
            bd = v;
        }
    }
    if (best < 0) {  // every cluster full with this neuron unplaced: not reachable
        set_status(status, MOE_ERR_DEVICE_BADINDEX);
        return;
    }
    const int pos = atomicAdd(&cnt[r * E + best], 1);
    if (pos < d_ff) {
        list[(size_t)best * d_ff + pos] = i;
        keys[(size_t)best * d_ff + pos] = bd;
    }
}

// Round r, acceptance: cluster blockIdx.y keeps the proposals whose rank by
// (distance, index) is below its room.  CTA x ranks proposals 32x .. 32x+31
// (lane = proposal); its 8 warps split the cluster's list into 8 ranges, count
// the smaller keys in their range (warp-uniform loads, broadcast to the lanes),
// and the 8 partial counts are added in shared memory.
constexpr int kAcceptWarps = 8;

__global__ void __launch_bounds__(kAcceptWarps * 32) cluster_accept_kernel(
    int d_ff, int E, int m, int r, const int32_t *__restrict__ cnt, int32_t *__restrict__ fill,
    const int32_t *__restrict__ list, const double *__restrict__ keys,
    int32_t *__restrict__ assign)
{
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t part[kAcceptWarps][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e = blockIdx.y;
    const int n = min(cnt[r * E + e], d_ff);
    const int f = fill[r * E + e];
    const int room = m - f;
    if (blockIdx.x == 0 && threadIdx.x == 0)
        fill[(r + 1) * E + e] = f + min(n, room);
    const int p0 = blockIdx.x * 32;
    if (p0 >= n)
        return;
    const int p = p0 + lane;
    const bool have = p < n;
    const double *ke = keys + (size_t)e * d_ff;
    const int32_t *le = list + (size_t)e * d_ff;
    const double ki = have ? ke[p] : 0.0;
    const int ii = have ? le[p] : 0;
    if (n <= room) {  // every proposal fits
        if (have && warp == 0)
            assign[ii] = e;
        return;
    }
    const int q0 = (int)((int64_t)n * warp / kAcceptWarps);
    const int q1 = (int)((int64_t)n * (warp + 1) / kAcceptWarps);
    int rank = 0;
#pragma unroll 8
    for (int q = q0; q < q1; ++q) {
        const double kj = __ldg(ke + q);
        const int j = __ldg(le + q);
        rank += (kj < ki || (kj == ki && j < ii)) ? 1 : 0;
    }
    part[warp][lane] = rank;
    __syncthreads();
    if (warp == 0) {
        int tot = 0;
#pragma unroll
        for (int w = 0; w < kAcceptWarps; ++w)
            tot += part[w][lane];
        if (have && tot < room)
            assign[ii] = e;
    }
}

// Permutation: perm[e*m + j] = the j-th smallest neuron index of cluster e.
// One CTA walks the neurons in chunks of 1024; per chunk a ballot per cluster
// gives each neuron its rank among the chunk's members of its cluster.
__global__ void __launch_bounds__(1024) cluster_perm_kernel(const int32_t *__restrict__ assign,
                                                            int d_ff, int E, int m,
                                                            int32_t *__restrict__ perm,
                                                            int32_t *status)
{
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t base[MOE_MAX_EXPERTS];
    __shared__ int32_t wc[32][MOE_MAX_EXPERTS];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    if (tid < E)
        base[tid] = 0;
    __syncthreads();
    constexpr int G = 8;  // chunks whose assignment is loaded at once
    int av[G];
    for (int i0 = 0; i0 < d_ff; i0 += blockDim.x) {
        const int ci = (i0 / blockDim.x) % G;
        if (ci == 0) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const int ig = i0 + g * blockDim.x + tid;
                av[g] = ig < d_ff ? assign[ig] : -1;
            }
        }
        const int i = i0 + tid;
        int a = -1;
#pragma unroll
        for (int g = 0; g < G; ++g)
            if (g == ci)
                a = av[g];
        if (i < d_ff && (a < 0 || a >= E)) {
            set_status(status, MOE_ERR_DEVICE_BADINDEX);
            a = -1;
        }
        int mine = 0;
        for (int e = 0; e < E; ++e) {
            const uint32_t mask = __ballot_sync(0xffffffffu, a == e);
            if (lane == 0)
                wc[warp][e] = __popc(mask);
            if (a == e)
                mine = __popc(mask & lt);
        }
        __syncthreads();
        // exclusive scan over the 32 warps, one warp per cluster: lane l holds
        // warp l's count
        for (int e = warp; e < E; e += 32) {
            const int cnt = wc[lane][e];
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o)
                    incl += t;
            }
            const int b0 = base[e];
            wc[lane][e] = b0 + incl - cnt;
            __syncwarp();
            if (lane == 31)
                base[e] = b0 + incl;
        }
        __syncthreads();
        if (a >= 0) {
            const int pos = wc[warp][a] + mine;
            if (pos < m)
                perm[(size_t)a * m + pos] = i;
            else
                set_status(status, MOE_ERR_DEVICE_BADINDEX);
        }
        __syncthreads();
    }
    if (tid < E && base[tid] != m)
        set_status(status, MOE_ERR_DEVICE_BADINDEX);
}

// Centers: CTA (cluster e, 64 columns), thread per column; the members' rows
// are summed in ascending neuron index.  The member indices are staged in
// shared memory (2048 at a time) and the rows stream through a 4-stage ring of
// 8 KB batches filled with cp.async, so three batches of gathered 128- or
// 256-byte row segments are in flight while one is summed.  A member index out
// of range (only after a failed assignment, which the status word reports)
// reads as a zero row, adding +0.
constexpr int kCenterCols = 64;
constexpr int kCenterBatchBytes = 8 * 1024;
constexpr int kCenterStages = 4;
constexpr int kCenterIdxChunk = 2048;

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem)
{
    const uint32_t sa = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit()
{
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N> __device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <typename E_T>
__global__ void __launch_bounds__(kCenterCols) cluster_center_kernel(
    const E_T *__restrict__ F, int d, int d_ff, int m, const int32_t *__restrict__ perm,
    double *__restrict__ centers)
{
    pdl_wait();
    pdl_trigger();
    constexpr int VN = 16 / sizeof(E_T);
    constexpr int VPR = kCenterCols / VN;                                  // vectors per row
    constexpr int RB = kCenterBatchBytes / (kCenterCols * (int)sizeof(E_T));  // rows per batch
    constexpr int VPT = RB * VPR / kCenterCols;                            // vectors per thread
    __shared__ __align__(16) E_T rows[kCenterStages][RB][kCenterCols];
    __shared__ int32_t s_idx[kCenterIdxChunk];
    const int e = blockIdx.x;
    const int c0 = blockIdx.y * kCenterCols;
    const int tid = threadIdx.x;
    double acc = 0.0;

    for (int pc = 0; pc < m; pc += kCenterIdxChunk) {
        const int cn = min(kCenterIdxChunk, m - pc);
        __syncthreads();  // the previous chunk's batches are summed
        for (int q = tid; q < cn; q += kCenterCols) {
            const int v = perm[(size_t)e * m + pc + q];
            s_idx[q] = (v >= 0 && v < d_ff) ? v : -1;
        }
        __syncthreads();
        const int nb = (cn + RB - 1) / RB;
        auto issue = [&](int b) {
            if (b < nb) {
                E_T(*slot)[kCenterCols] = rows[b % kCenterStages];
#pragma unroll
                for (int j = 0; j < VPT; ++j) {
                    const int v = tid + kCenterCols * j;
                    const int r = v / VPR, q = v % VPR;
                    const int p = b * RB + r;
                    const int col = c0 + q * VN;  // d % 8 == 0: a vector is all in or out
                    const int src = p < cn ? s_idx[p] : -1;
                    if (src >= 0 && col < d)
                        cp_async16(&slot[r][q * VN], F + (size_t)src * d + col);
                    else
                        *reinterpret_cast<uint4 *>(&slot[r][q * VN]) = make_uint4(0, 0, 0, 0);
                }
            }
            cp_async_commit();  // an empty group past the end keeps the count uniform
        };
#pragma unroll
        for (int b = 0; b < kCenterStages - 1; ++b)
            issue(b);
        for (int b = 0; b < nb; ++b) {
            issue(b + kCenterStages - 1);
            cp_async_wait<kCenterStages - 1>();  // this thread's copies of batch b landed
            __syncthreads();                     // everyone's
            const E_T(*slot)[kCenterCols] = rows[b % kCenterStages];
            const int rn = min(RB, cn - b * RB);
            if (rn == RB) {
#pragma unroll 16
                for (int r = 0; r < RB; ++r)
                    acc = __dadd_rn(acc, (double)to_f32(slot[r][tid]));
            } else {
                for (int r = 0; r < rn; ++r)
                    acc = __dadd_rn(acc, (double)to_f32(slot[r][tid]));
            }
            __syncthreads();  // the slot is free for the batch issued next
        }
        cp_async_wait<0>();
    }
    if (c0 + tid < d)
        centers[(size_t)e * d + c0 + tid] = __ddiv_rn(acc, (double)m);
}

namespace {

template <typename E_T, int NW, int NJ>
cudaError_t launch_dist_t(const void *F, int d, int d_ff, int E, const double *centers, double *D,
                          int32_t *assign, int32_t *counters, cudaStream_t s)
{
    const size_t smem = ((size_t)E * kDistCols + (size_t)kDistRows * kFsStride) * sizeof(double);
    auto kern = cluster_dist_kernel<E_T, NW, NJ>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess)
            return e;
    }
    const int grid = (d_ff + kDistRows - 1) / kDistRows;
    count_launch();
    return launch_pdl(kern, dim3(grid), dim3(NW * 32), smem, s, static_cast<const E_T *>(F), d,
                      d_ff, E, centers, D, assign, counters);
}

template <typename E_T>
cudaError_t launch_dist(const void *F, int d, int d_ff, int E, const double *centers, double *D,
                        int32_t *assign, int32_t *counters, cudaStream_t s)
{
    // NW warps, NJ cluster pairs per lane: NW * NJ >= ceil(E / 2)
    if (E <= 8)
        return launch_dist_t<E_T, 4, 1>(F, d, d_ff, E, centers, D, assign, counters, s);
    if (E <= 16)
        return launch_dist_t<E_T, 8, 1>(F, d, d_ff, E, centers, D, assign, counters, s);
    if (E <= 32)
        return launch_dist_t<E_T, 8, 2>(F, d, d_ff, E, centers, D, assign, counters, s);
    return launch_dist_t<E_T, 8, 4>(F, d, d_ff, E, centers, D, assign, counters, s);
}

template <typename E_T>
cudaError_t run_cluster(const void *F, int d, int d_ff, int E, int n_iter, const int32_t *init,
                        int32_t *assign, double *centers, int32_t *perm, char *ws,
                        cudaStream_t s)
{
    const ClusterLayout L = cluster_layout(d_ff, E);
    int32_t *status = reinterpret_cast<int32_t *>(ws);
    double *D = reinterpret_cast<double *>(ws + L.D);
    double *keys = reinterpret_cast<double *>(ws + L.keys);
    int32_t *list = reinterpret_cast<int32_t *>(ws + L.list);
    int32_t *cnt = reinterpret_cast<int32_t *>(ws + L.cnt);
    int32_t *fill = reinterpret_cast<int32_t *>(ws + L.fill);
    const int m = d_ff / E;
    const E_T *Ft = static_cast<const E_T *>(F);

    count_launch();
    cudaError_t e = launch_pdl(cluster_init_kernel<E_T>, dim3(E, (d + 255) / 256), dim3(256), 0,
                               s, Ft, d, d_ff, E, init, centers, status);
    for (int it = 0; it < n_iter && e == cudaSuccess; ++it) {
        e = launch_dist<E_T>(F, d, d_ff, E, centers, D, assign, cnt, s);
        for (int r = 0; r < E && e == cudaSuccess; ++r) {
            count_launch(2);
            e = launch_pdl(cluster_propose_kernel, dim3((d_ff + 255) / 256), dim3(256), 0, s,
                           (const double *)D, d_ff, E, m, r, (const int32_t *)assign, cnt,
                           (const int32_t *)fill, list, keys, status);
            if (e == cudaSuccess)
                e = launch_pdl(cluster_accept_kernel, dim3((d_ff + 31) / 32, E),
                               dim3(kAcceptWarps * 32), 0,
                               s, d_ff, E, m, r, (const int32_t *)cnt, fill,
                               (const int32_t *)list, (const double *)keys, assign);
        }
        if (e == cudaSuccess) {
            count_launch(2);
            e = launch_pdl(cluster_perm_kernel, dim3(1), dim3(1024), 0, s,
                           (const int32_t *)assign, d_ff, E, m, perm, status);
        }
        if (e == cudaSuccess)
            e = launch_pdl(cluster_center_kernel<E_T>, dim3(E, (d + kCenterCols - 1) / kCenterCols),
                           dim3(kCenterCols), 0, s,
                           Ft, d, d_ff, m, (const int32_t *)perm, centers);
    }
    return e;
}

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" size_t moe_cluster_workspace_size(int32_t d, int32_t d_ff, int32_t E)
{
    if (d < 8 || d_ff < 1 || E < 1 || E > MOE_MAX_EXPERTS || d_ff % E != 0 || d_ff > (1 << 22))
        return 0;
    return cluster_layout(d_ff, E).total;
}

extern "C" int moe_cluster_distances(const void *F, int32_t d, int32_t d_ff, int32_t E,
                                     int32_t dtype, const double *centers, double *D,
                                     void *stream)
{
    const char *fn = "moe_cluster_distances";
    char msg[256];
    if (!F || !centers || !D) {
        snprintf(msg, sizeof msg, "%s: a pointer argument is NULL", fn);
        return report_error(MOE_ERR_INVALID_ARG, msg);
    }
    if ((reinterpret_cast<uintptr_t>(F) & 15u) || (reinterpret_cast<uintptr_t>(centers) & 15u) ||
        (reinterpret_cast<uintptr_t>(D) & 7u)) {
        snprintf(msg, sizeof msg, "%s: F and centers need 16-byte, D 8-byte alignment", fn);
        return report_error(MOE_ERR_ALIGN, msg);
    }
    if (dtype != MOE_BF16 && dtype != MOE_F32) {
        snprintf(msg, sizeof msg, "%s: dtype=%d", fn, dtype);
        return report_error(MOE_ERR_DTYPE, msg);
    }
    if (E < 1 || E > MOE_MAX_EXPERTS) {
        snprintf(msg, sizeof msg, "%s: E=%d outside 1..%d", fn, E, MOE_MAX_EXPERTS);
        return report_error(MOE_ERR_INVALID_ARG, msg);
    }
    if (d < 8 || d % 8 != 0 || d_ff < 1 || d_ff > (1 << 22)) {
        snprintf(msg, sizeof msg, "%s: d=%d (multiple of 8), d_ff=%d", fn, d, d_ff);
        return report_error(MOE_ERR_SHAPE, msg);
    }
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = dtype == MOE_BF16
                        ? launch_dist<bf16>(F, d, d_ff, E, centers, D, nullptr, nullptr, s)
                        : launch_dist<float>(F, d, d_ff, E, centers, D, nullptr, nullptr, s);
    if (e == cudaSuccess)
        e = cudaGetLastError();
    if (e != cudaSuccess)
        return report_cuda(e, fn);
    return report_ok();
}

extern "C" int moe_cluster_partition(const void *F, int32_t d, int32_t d_ff, int32_t E,
                                     int32_t dtype, int32_t n_iter, const int32_t *init_idx,
                                     int32_t *assign, double *centers, int32_t *perm, void *ws,
                                     size_t ws_bytes, void *stream)
{
    const char *fn = "moe_cluster_partition";
    char msg[256];
    if (!F || !init_idx || !assign || !centers || !perm || !ws) {
        snprintf(msg, sizeof msg, "%s: a pointer argument is NULL", fn);
        return report_error(MOE_ERR_INVALID_ARG, msg);
    }
    if ((reinterpret_cast<uintptr_t>(F) & 15u) || (reinterpret_cast<uintptr_t>(ws) & 15u) ||
        (reinterpret_cast<uintptr_t>(centers) & 15u) || (reinterpret_cast<uintptr_t>(assign) & 3u) ||
        (reinterpret_cast<uintptr_t>(perm) & 3u) || (reinterpret_cast<uintptr_t>(init_idx) & 3u)) {
        snprintf(msg, sizeof msg, "%s: F, centers and ws need 16-byte, index arrays 4-byte"
                 " alignment", fn);
        return report_error(MOE_ERR_ALIGN, msg);
    }
    if (dtype != MOE_BF16 && dtype != MOE_F32) {
        snprintf(msg, sizeof msg, "%s: dtype=%d", fn, dtype);
        return report_error(MOE_ERR_DTYPE, msg);
    }
    if (E < 1 || E > MOE_MAX_EXPERTS || n_iter < 1) {
        snprintf(msg, sizeof msg, "%s: E=%d (1..%d), n_iter=%d (>= 1)", fn, E, MOE_MAX_EXPERTS,
                 n_iter);
        return report_error(MOE_ERR_INVALID_ARG, msg);
    }
    if (d < 8 || d % 8 != 0 || d_ff < 1 || d_ff > (1 << 22) || d_ff % E != 0) {
        snprintf(msg, sizeof msg, "%s: d=%d (multiple of 8), d_ff=%d (multiple of E=%d)", fn, d,
                 d_ff, E);
        return report_error(MOE_ERR_SHAPE, msg);
    }
    const size_t need = cluster_layout(d_ff, E).total;
    if (ws_bytes < need) {
        snprintf(msg, sizeof msg, "%s: workspace %zu bytes, need %zu", fn, ws_bytes, need);
        return report_error(MOE_ERR_WORKSPACE, msg);
    }
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = dtype == MOE_BF16
                        ? run_cluster<bf16>(F, d, d_ff, E, n_iter, init_idx, assign, centers,
                                            perm, static_cast<char *>(ws), s)
                        : run_cluster<float>(F, d, d_ff, E, n_iter, init_idx, assign, centers,
                                             perm, static_cast<char *>(ws), s);
    if (e == cudaSuccess)
        e = cudaGetLastError();
    if (e != cudaSuccess)
        return report_cuda(e, fn);
    return report_ok();
}
