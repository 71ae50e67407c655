// bwd_tc.cu -- the grouped GEMMs of the layer's backward pass on the tcgen05
// tensor cores ("LLaMA-MoE v2", code sample "代码实现示例", class Expert, read
// backwards: the gradients of out = W2 (silu(W1 x) * W3 x)).
//
// One persistent kernel, two tile orders:
//   row-grouped (dgrad): C[rows of expert e][N] = A[rows][K] B_e[N][K]^T, the rows
//     of expert e being [offsets[e], offsets[e+1]) -- the forward's tile order:
//       dh      = d_out  W2_e        (A = d_out,  B = W2_e^T  [m16][d])
//       dGU     = SwiGLU backward of x_perm W13_e^T   (fused epilogue, below)
//       dx_perm = dGU    W13_e       (A = dGU,    B = W13_e^T [d][2 m16])
//   K-grouped (wgrad): C_e[M][N] = A[M][K_e] B[N][K_e]^T, the reduction running over
//     the rows of expert e, which the transposes below lay out as the column range
//     [koff[e], koff[e+1]) of A and B, koff[e] = sum over e' < e of the rows of e'
//     rounded up to 64 (zero columns pad each range):
//       dW2_e  = d_out_e^T h_e       (A = d_out^T [d][K], B = h^T [m16][K])
//       dW13_e = dGU_e^T x_e         (A = dGU^T [2 m16][K], B = x_perm^T [d][K])
//     An expert with no rows gets a zero gradient.
// Both operands are K-major bf16 loaded by TMA (128-byte swizzle, 128x64 and
// 256x64 boxes, 4-stage ring); every K coordinate is a multiple of 64, so every
// TMA x coordinate is 128-byte aligned.  f32 accumulators in TMEM, double
// buffered; outputs rounded to bf16 once.
//
// SwiGLU backward epilogue: the accumulator tile is [g | u] of the packed W13
// layout (per 32 columns: the gate values of 16 neurons, then their up values);
// with dh read from global memory:
//   du = dh * silu(g),  dg = dh * u * sigma(g) (1 + g (1 - sigma(g)))
// written in the same packed order (dGU [rows][2 m16]), so dGU times W13_e^T is
// the input gradient.
//
// Warp roles and bounded waits as in the forward kernel: warp 0 TMA, warp 1 MMA,
// warps 2-9 epilogue; a wait past its limit records MOE_ERR_DEVICE_TIMEOUT,
// every role stops, copies and MMAs are drained and TMEM is freed.  No TMA load
// uses cluster multicast.
#include <mutex>

#include "tc_common.cuh"

namespace moe {
namespace bwd {

using tc::bulk_commit;
using tc::bulk_wait_all;
using tc::bulk_wait_read_1;
using tc::fence_proxy_async_smem;
using tc::mbar_arrive;
using tc::mbar_drain;
using tc::mbar_expect_tx;
using tc::mbar_init;
using tc::mbar_wait;
using tc::sdesc;
using tc::smem_u32;
using tc::st_shared_v4;
using tc::tc_fence_after;
using tc::tc_fence_before;
using tc::tma_load_2d;
using tc::tma_load_3d;
using tc::tma_store_2d;
using tc::tmem_ld32_async;
using tc::tmem_wait_ld;
using tc::umma_commit;
using tc::umma_f16;

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int ACC = 2;
constexpr int TMEM_COLS = ACC * BN;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TILE_BYTES = STAGES * STAGE_BYTES;
constexpr int NUM_THREADS = 320;
constexpr int EPI_WARPS = 8;
constexpr int kStageSlotBytes = 32 * 64;
constexpr int kEpiStageBytes = EPI_WARPS * 2 * kStageSlotBytes;

enum { EPI_STORE = 0, EPI_SWIGLU_BWD = 1 };

struct Aux {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[ACC];
    uint64_t tempty[ACC];
    uint64_t drain;
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t off[MOE_MAX_EXPERTS + 1];   // row offsets (row-grouped) / K offsets (K-grouped)
    int32_t tstart[MOE_MAX_EXPERTS + 1];
};
constexpr int SMEM_BYTES = 1024 + TILE_BYTES + kEpiStageBytes + (int)sizeof(Aux);

// kind::f16: D f32, A and B bf16, both K-major, N = BN, M = BM.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);
// the same with B MN-major (bit 16): the dgrad GEMMs read the expert weights as they
// are packed, N contiguous, instead of a transposed copy
constexpr uint32_t kIdescBt = kIdesc | (1u << 16);
// MN-major B in shared memory: 64-wide N chunks of BK K rows (128 bytes each)
constexpr uint32_t kMnChunkBytes = BK * 128;
// descriptor advance for 16 more K rows of an MN-major tile (2048 bytes, 16-byte units)
constexpr int kMnKStep = 2048 >> 4;

// Output staging as in the forward kernel: two 2 KB slots per epilogue warp, each a
// [32 rows][64 bytes] box in the 64-byte swizzle the output map expects.
struct EpiStore {
    const CUtensorMap *map;
    uint32_t slots;
    int slot;
};

__device__ __forceinline__ void stage_box(EpiStore &st, const uint32_t (&pk)[16], int col, int row0)
{
    const int lane = threadIdx.x & 31;
    if (lane == 0)
        bulk_wait_read_1();
    __syncwarp();
    const uint32_t base = st.slots + (uint32_t)(st.slot * kStageSlotBytes) + (uint32_t)(lane * 64);
#pragma unroll
    for (int j = 0; j < 4; ++j)
        st_shared_v4(base + (uint32_t)(((j ^ ((lane >> 1) & 3)) << 4)), pk[4 * j], pk[4 * j + 1],
                     pk[4 * j + 2], pk[4 * j + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(st.map, st.slots + (uint32_t)(st.slot * kStageSlotBytes), col, row0);
        bulk_commit();
    }
    st.slot ^= 1;
}

// 32 output columns of this lane's row: a full box goes through staging, a
// partial one is written per lane (n_valid is a multiple of 8).
__device__ __forceinline__ void emit32(EpiStore &st, const float (&f)[32], int col, int row0,
                                       int row, bool rv, bool full_rows, bf16 *__restrict__ out,
                                       int ld_out, int n_valid)
{
    if (full_rows && col + 32 <= n_valid) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(f[2 * i], f[2 * i + 1]);
        stage_box(st, pk, col, row0);
    } else if (rv) {
        bf16 *dst = out + (int64_t)row * ld_out + col;
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (col + q * 8 < n_valid)
                st_v4(dst + q * 8, f32x8_to_bf16(f + q * 8));
    }
}

// Epilogue of one warp's 32-row slab; chunks of 32 accumulator columns
// [c_first, c_first + n_chunks) of the tile at output column n0.  zero: the tile
// had no K blocks (an expert without rows in the K-grouped order).
template <int EPI>
__device__ __forceinline__ void epilogue_slab(uint32_t taddr, int c_first, int n_chunks, int row0,
                                              int row_end, int n0, bool zero,
                                              bf16 *__restrict__ out, int ld_out, int n_valid,
                                              const bf16 *__restrict__ dh, int ld_dh,
                                              EpiStore &st)
{
    const int lane = threadIdx.x & 31;
    const int row = row0 + lane;
    const bool rv = row < row_end;
    const bool full_rows = row0 + 32 <= row_end;
#pragma unroll 1
    for (int c = c_first; c < c_first + n_chunks; c += 2) {
        uint32_t v[2][32];
        if (zero) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                v[0][i] = v[1][i] = 0u;
        } else {
            tmem_ld32_async(taddr + (uint32_t)(c * 32), v[0]);
            tmem_ld32_async(taddr + (uint32_t)((c + 1) * 32), v[1]);
            tmem_wait_ld();
        }
        if constexpr (EPI == EPI_SWIGLU_BWD) {
            // neurons nb .. nb+31: 16 per chunk; dh columns past ld_dh are zero
            const int nb = n0 / 2 + c * 16;
            float dhv[32];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint4 u4 = make_uint4(0, 0, 0, 0);
                if (rv && nb + 8 * q < ld_dh)
                    u4 = *reinterpret_cast<const uint4 *>(dh + (int64_t)row * ld_dh + nb + 8 * q);
                bf16x8_to_f32(u4, dhv + 8 * q);
            }
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                float o[32];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float g = __uint_as_float(v[q2][i]);
                    const float u = __uint_as_float(v[q2][16 + i]);
                    const float s = 1.0f / (1.0f + __expf(-g));
                    const float dhi = dhv[q2 * 16 + i];
                    o[i] = dhi * u * s * (1.0f + g * (1.0f - s));  // dg
                    o[16 + i] = dhi * g * s;                       // du = dh * silu(g)
                }
                emit32(st, o, n0 + (c + q2) * 32, row0, row, rv, full_rows, out, ld_out, n_valid);
            }
        } else {
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                float o[32];
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    o[i] = __uint_as_float(v[q2][i]);
                emit32(st, o, n0 + (c + q2) * 32, row0, row, rv, full_rows, out, ld_out, n_valid);
            }
        }
    }
}

struct Tile {
    int e, a_row, row0, row_end, n0, k0, nkb;
};

// KG = false: tiles of expert e are its row tiles x N tiles (forward order).
// KG = true:  every expert has ceil(M / BM) x N tiles; K range from aux->off.
template <bool KG>
__device__ __forceinline__ Tile decode_tile(const Aux *aux, int tile, int n_tiles, int M,
                                            int num_kb)
{
    Tile t;
    int e = 0;
    while (tile >= aux->tstart[e + 1])
        ++e;
    const int local = tile - aux->tstart[e];
    t.e = e;
    if constexpr (KG) {
        const int mtiles = (M + BM - 1) / BM;
        const int mt = local % mtiles, nt = local / mtiles;
        t.a_row = mt * BM;
        t.row0 = e * M + mt * BM;
        t.row_end = e * M + M;
        t.n0 = nt * BN;
        t.k0 = aux->off[e];
        t.nkb = (aux->off[e + 1] - aux->off[e]) / BK;
    } else {
        const int rows = aux->off[e + 1] - aux->off[e];
        const int mtiles = (rows + BM - 1) / BM;
        const int mt = local % mtiles, nt = local / mtiles;
        t.a_row = aux->off[e] + mt * BM;
        t.row0 = t.a_row;
        t.row_end = aux->off[e + 1];
        t.n0 = nt * BN;
        t.k0 = 0;
        t.nkb = num_kb;
    }
    return t;
}

template <int EPI, bool KG, bool BT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmO, const int32_t *__restrict__ offsets,
                    int E, int N, int K, int M, bf16 *__restrict__ out, int ld_out, int n_valid,
                    const bf16 *__restrict__ dh, int ld_dh, int32_t *status, uint64_t wait_ns)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Aux *aux = reinterpret_cast<Aux *>(smem + TILE_BYTES + kEpiStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int32_t *abort_flag = &aux->abort_flag;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&aux->full[s]), 1);
            mbar_init(smem_u32(&aux->empty[s]), 1);
        }
        for (int a = 0; a < ACC; ++a) {
            mbar_init(smem_u32(&aux->tfull[a]), 1);
            mbar_init(smem_u32(&aux->tempty[a]), EPI_WARPS);
        }
        mbar_init(smem_u32(&aux->drain), 1);
        aux->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmO)) : "memory");
    }
    const int n_tiles = (N + BN - 1) / BN;
    if (warp == 2 && lane == 0) {
        // row offsets; in the K-grouped order their rounded-up prefix sums
        int acc = 0, kacc = 0;
        for (int e = 0; e < E; ++e) {
            const int rows = offsets[e + 1] - offsets[e];
            aux->tstart[e] = acc;
            if constexpr (KG) {
                aux->off[e] = kacc;
                kacc += (rows + BK - 1) / BK * BK;
                acc += (M + BM - 1) / BM * n_tiles;
            } else {
                aux->off[e] = offsets[e];
                acc += (rows + BM - 1) / BM * n_tiles;
            }
        }
        aux->off[E] = KG ? kacc : offsets[E];
        aux->tstart[E] = acc;
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&aux->tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = aux->tmem_base;
    const int total = aux->tstart[E];
    const int num_kb = (K + BK - 1) / BK;
    const uint32_t smem_base = smem_u32(smem);

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------- TMA producer
            int stage = 0;
            uint32_t phase = 0;
            int64_t fills = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                if (*abort_flag)
                    break;
                const Tile t = decode_tile<KG>(aux, tile, n_tiles, M, num_kb);
                for (int kb = 0; kb < t.nkb; ++kb) {
                    if (!mbar_wait(smem_u32(&aux->empty[stage]), phase ^ 1u, wait_ns, abort_flag,
                                   status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&aux->full[stage]);
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    mbar_expect_tx(fb, STAGE_BYTES);
                    const int kc = t.k0 + kb * BK;
                    tma_load_2d(&tmA, fb, sa, kc, t.a_row);
                    if constexpr (BT) {  // MN-major B: 64-wide N chunks of BK K rows
#pragma unroll
                        for (int j = 0; j < BN / 64; ++j)
                            tma_load_3d(&tmB, fb, sa + A_BYTES + j * kMnChunkBytes, t.n0 + 64 * j,
                                        kc, t.e);
                    } else if constexpr (KG) {
                        tma_load_2d(&tmB, fb, sa + A_BYTES, kc, t.n0);
                    } else {
                        tma_load_3d(&tmB, fb, sa + A_BYTES, kc, t.n0, t.e);
                    }
                    ++fills;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int s = 0; s < STAGES; ++s) {
                const int64_t n = fills / STAGES + (s < fills % STAGES ? 1 : 0);
                if (n > 0)
                    mbar_drain(smem_u32(&aux->full[s]), (uint32_t)((n - 1) & 1));
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------- MMA issuer
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const Tile t = decode_tile<KG>(aux, tile, n_tiles, M, num_kb);
                if (!mbar_wait(smem_u32(&aux->tempty[acc]), acc_phase ^ 1u, wait_ns, abort_flag,
                               status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < t.nkb; ++kb) {
                    if (!mbar_wait(smem_u32(&aux->full[stage]), phase, wait_ns, abort_flag,
                                   status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    const uint64_t da = sdesc(sa);
                    const uint64_t db = BT ? tc::sdesc_mn(sa + A_BYTES, kMnChunkBytes)
                                           : sdesc(sa + A_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma_f16(d_tmem, da + (uint64_t)(2 * k),
                                 db + (uint64_t)(BT ? kMnKStep * k : 2 * k),
                                 BT ? kIdescBt : kIdesc, (kb | k) != 0);
                    umma_commit(smem_u32(&aux->empty[stage]));
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                umma_commit(smem_u32(&aux->tfull[acc]));  // also with no MMA (zero tile)
                if (++acc == ACC) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            umma_commit(smem_u32(&aux->drain));
            mbar_drain(smem_u32(&aux->drain), 0);
        }
    } else {
        // -------------------------------------------------------------- epilogue
        const int wq = warp & 3;
        const int lane_base = wq * 32;
        const int c_first = ((warp - 2) / 4) * (BN / 64);
        EpiStore st{&tmO, smem_base + TILE_BYTES + (uint32_t)((warp - 2) * 2 * kStageSlotBytes), 0};
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const Tile t = decode_tile<KG>(aux, tile, n_tiles, M, num_kb);
            if (!mbar_wait(smem_u32(&aux->tfull[acc]), acc_phase, wait_ns, abort_flag, status))
                break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)lane_base << 16) + (uint32_t)(acc * BN);
            epilogue_slab<EPI>(taddr, c_first, BN / 64, t.row0 + lane_base, t.row_end, t.n0,
                               t.nkb == 0, out, ld_out, n_valid, dh, ld_dh, st);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&aux->tempty[acc]));
            if (++acc == ACC) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (lane == 0)
            bulk_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(TMEM_COLS)
                     : "memory");
    }
}

// ------------------------------------------------------------------------ 2-SM variant
// The same GEMMs with cta_group::2 (the forward's pair kernel, with the two tile
// orders and the epilogues above): a cluster of two CTAs owns a 256-row output
// tile; CTA r loads rows [128r, 128r+128) of the A tile and rows [128r, 128r+128) of
// the B tile, the leader issues M=256 MMAs reading A from each CTA and B from both,
// and every CTA drains its own 128 accumulator rows.  Barriers as in the forward
// pair kernel (full: leader counts both CTAs' bytes; empty/tfull: multicast
// commits; tempty: both CTAs' epilogue warps arrive on the leader).  Loads carry no
// multicast qualifier.
namespace pair {

constexpr int BM = 128;   // rows per CTA
constexpr int BNH = 128;  // B rows per CTA
constexpr int STAGES = 6;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BNH * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TILE_BYTES = STAGES * STAGE_BYTES;
constexpr uint64_t kAbortSettleNs = 200000ull;

struct Aux {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[ACC];
    uint64_t tempty[ACC];
    uint64_t drain;
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t off[MOE_MAX_EXPERTS + 1];
    int32_t tstart[MOE_MAX_EXPERTS + 1];
};
constexpr int SMEM_BYTES = 1024 + TILE_BYTES + kEpiStageBytes + (int)sizeof(Aux);

// kind::f16, D f32, A/B bf16 K-major, N = 256, M = 256 (the pair)
constexpr uint32_t kIdesc2 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                             ((uint32_t)(256 >> 4) << 24);

__device__ __forceinline__ uint32_t cta_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}
__device__ __forceinline__ uint32_t map_rank(uint32_t saddr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}
__device__ __forceinline__ int32_t ld_cluster_s32(uint32_t cluster_addr)
{
    int32_t v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
    return v;
}
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap *map, uint32_t bar_cluster,
                                                 uint32_t dst, int c0, int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(const CUtensorMap *map, uint32_t bar_cluster,
                                                 uint32_t dst, int c0, int c1, int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
__device__ __forceinline__ void umma_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void umma_commit_both(uint32_t bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(bar),
        "h"((uint16_t)3)
        : "memory");
}
__device__ __forceinline__ void umma_commit_own(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

// Pair tiles: row-grouped, 256 rows of an expert per tile; K-grouped, 256 of the M
// rows of every expert per tile.  row0 / a_row: the pair's first row (rank 0).
template <bool KG>
__device__ __forceinline__ Tile decode_tile(const Aux *aux, int tile, int n_tiles, int M,
                                            int num_kb)
{
    Tile t;
    int e = 0;
    while (tile >= aux->tstart[e + 1])
        ++e;
    const int local = tile - aux->tstart[e];
    t.e = e;
    if constexpr (KG) {
        const int mtiles = (M + 2 * BM - 1) / (2 * BM);
        const int mt = local % mtiles, nt = local / mtiles;
        t.a_row = mt * 2 * BM;
        t.row0 = e * M + mt * 2 * BM;
        t.row_end = e * M + M;
        t.n0 = nt * BN;
        t.k0 = aux->off[e];
        t.nkb = (aux->off[e + 1] - aux->off[e]) / BK;
    } else {
        const int rows = aux->off[e + 1] - aux->off[e];
        const int mtiles = (rows + 2 * BM - 1) / (2 * BM);
        const int mt = local % mtiles, nt = local / mtiles;
        t.a_row = aux->off[e] + mt * 2 * BM;
        t.row0 = t.a_row;
        t.row_end = aux->off[e + 1];
        t.n0 = nt * BN;
        t.k0 = 0;
        t.nkb = num_kb;
    }
    return t;
}

template <int EPI, bool KG, bool BT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_gemm_2sm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmO,
                        const int32_t *__restrict__ offsets, int E, int N, int K, int M,
                        bf16 *__restrict__ out, int ld_out, int n_valid,
                        const bf16 *__restrict__ dh, int ld_dh, int32_t *status, uint64_t wait_ns)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Aux *aux = reinterpret_cast<Aux *>(smem + TILE_BYTES + kEpiStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int32_t *abort_flag = &aux->abort_flag;
    const uint32_t rank = cta_rank();
    const bool leader = rank == 0;
    const int cluster_id = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&aux->full[s]), 1);
            mbar_init(smem_u32(&aux->empty[s]), 1);
        }
        for (int a = 0; a < ACC; ++a) {
            mbar_init(smem_u32(&aux->tfull[a]), 1);
            mbar_init(smem_u32(&aux->tempty[a]), 2 * EPI_WARPS);
        }
        mbar_init(smem_u32(&aux->drain), 1);
        aux->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmO)) : "memory");
    }
    const int n_tiles = (N + BN - 1) / BN;
    if (warp == 2 && lane == 0) {
        int acc = 0, kacc = 0;
        for (int e = 0; e < E; ++e) {
            const int rows = offsets[e + 1] - offsets[e];
            aux->tstart[e] = acc;
            if constexpr (KG) {
                aux->off[e] = kacc;
                kacc += (rows + BK - 1) / BK * BK;
                acc += (M + 2 * BM - 1) / (2 * BM) * n_tiles;
            } else {
                aux->off[e] = offsets[e];
                acc += (rows + 2 * BM - 1) / (2 * BM) * n_tiles;
            }
        }
        aux->off[E] = KG ? kacc : offsets[E];
        aux->tstart[E] = acc;
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&aux->tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers exist before either signals the other's
    tc_fence_after();
    const uint32_t tmem_base = aux->tmem_base;
    const int total = aux->tstart[E];
    const int num_kb = (K + BK - 1) / BK;
    const uint32_t smem_base = smem_u32(smem);

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------- TMA producer (both)
            int stage = 0;
            uint32_t phase = 0;
            int64_t fills = 0;
            bool ok = true;
            for (int tile = cluster_id; tile < total && ok; tile += nclusters) {
                if (*abort_flag)
                    break;
                const Tile t = decode_tile<KG>(aux, tile, n_tiles, M, num_kb);
                for (int kb = 0; kb < t.nkb; ++kb) {
                    if (!mbar_wait(smem_u32(&aux->empty[stage]), phase ^ 1u, wait_ns, abort_flag,
                                   status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&aux->full[stage]);
                    if (leader)
                        mbar_expect_tx(fb, 2 * STAGE_BYTES);
                    const uint32_t fb0 = map_rank(fb, 0);
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    const int kc = t.k0 + kb * BK;
                    tma_load_2d_pair(&tmA, fb0, sa, kc, t.a_row + (int)rank * BM);
                    if constexpr (BT) {  // MN-major B: this CTA's 64-wide N chunks
#pragma unroll
                        for (int j = 0; j < BNH / 64; ++j)
                            tma_load_3d_pair(&tmB, fb0, sa + A_BYTES + j * kMnChunkBytes,
                                             t.n0 + (int)rank * BNH + 64 * j, kc, t.e);
                    } else if constexpr (KG) {
                        tma_load_2d_pair(&tmB, fb0, sa + A_BYTES, kc, t.n0 + (int)rank * BNH);
                    } else {
                        tma_load_3d_pair(&tmB, fb0, sa + A_BYTES, kc, t.n0 + (int)rank * BNH,
                                         t.e);
                    }
                    ++fills;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (leader) {  // the leader's full barriers count both CTAs' bytes
                for (int s = 0; s < STAGES; ++s) {
                    const int64_t n = fills / STAGES + (s < fills % STAGES ? 1 : 0);
                    if (n > 0)
                        mbar_drain(smem_u32(&aux->full[s]), (uint32_t)((n - 1) & 1));
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------------------- MMA issuer (leader)
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = cluster_id; tile < total && ok; tile += nclusters) {
                const Tile t = decode_tile<KG>(aux, tile, n_tiles, M, num_kb);
                if (!mbar_wait(smem_u32(&aux->tempty[acc]), acc_phase ^ 1u, wait_ns, abort_flag,
                               status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < t.nkb; ++kb) {
                    if (!mbar_wait(smem_u32(&aux->full[stage]), phase, wait_ns, abort_flag,
                                   status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    const uint64_t da = sdesc(sa);
                    const uint64_t db = BT ? tc::sdesc_mn(sa + A_BYTES, kMnChunkBytes)
                                           : sdesc(sa + A_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma_pair(d_tmem, da + (uint64_t)(2 * k),
                                  db + (uint64_t)(BT ? kMnKStep * k : 2 * k),
                                  BT ? kIdesc2 | (1u << 16) : kIdesc2, (kb | k) != 0);
                    umma_commit_both(smem_u32(&aux->empty[stage]));
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                umma_commit_both(smem_u32(&aux->tfull[acc]));  // also with no MMA (zero tile)
                if (++acc == ACC) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            umma_commit_own(smem_u32(&aux->drain));
            mbar_drain(smem_u32(&aux->drain), 0);
        }
    } else {
        // ------------------------------------------------------------ epilogue (both)
        const int wq = warp & 3;
        const int lane_base = wq * 32;
        const int c_first = ((warp - 2) / 4) * (BN / 64);
        const uint32_t tempty0 = map_rank(smem_u32(&aux->tempty[0]), 0);
        const uint32_t tempty1 = map_rank(smem_u32(&aux->tempty[1]), 0);
        EpiStore st{&tmO, smem_base + TILE_BYTES + (uint32_t)((warp - 2) * 2 * kStageSlotBytes), 0};
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = cluster_id; tile < total; tile += nclusters) {
            const Tile t = decode_tile<KG>(aux, tile, n_tiles, M, num_kb);
            if (!mbar_wait(smem_u32(&aux->tfull[acc]), acc_phase, wait_ns, abort_flag, status))
                break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)lane_base << 16) + (uint32_t)(acc * BN);
            epilogue_slab<EPI>(taddr, c_first, BN / 64, t.row0 + (int)rank * BM + lane_base,
                               t.row_end, t.n0, t.nkb == 0, out, ld_out, n_valid, dh, ld_dh, st);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(acc == 0 ? tempty0 : tempty1);
            if (++acc == ACC) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (lane == 0)
            bulk_wait_all();
    }
    tc_fence_before();
    cluster_sync();
    if (threadIdx.x == 0) {
        const int peer_abort = ld_cluster_s32(map_rank(smem_u32(&aux->abort_flag), rank ^ 1u));
        if (*abort_flag || peer_abort) {
            const uint64_t t0 = globaltimer_ns();
            while (globaltimer_ns() - t0 < kAbortSettleNs) {
            }
        }
    }
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(TMEM_COLS)
                     : "memory");
    }
}

}  // namespace pair

// ------------------------------------------------------------------------ transposes
// Both transposes move 8 x 8 bf16 blocks through registers: a thread loads 8 rows
// of 8 columns (8 x 16 bytes), transposes them with byte permutes and stores 8
// rows of 8 columns.  Lane l of a warp takes row group l % 8 and column group
// l / 8 (+ 4 per warp), so a warp reads 8 rows x 64 bytes and writes 4 rows x
// 128 bytes per instruction; a CTA (8 warps) covers 64 rows x 256 columns.

// out[c] = column c of the 8 x 8 block whose rows are in[0..7].
__device__ __forceinline__ void transpose8x8(const uint4 (&in)[8], uint4 (&out)[8])
{
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint32_t sel = (c & 1) ? 0x7632u : 0x5410u;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t *a = reinterpret_cast<const uint32_t *>(&in[2 * q]);
            const uint32_t *b = reinterpret_cast<const uint32_t *>(&in[2 * q + 1]);
            w[q] = __byte_perm(a[c >> 1], b[c >> 1], sel);
        }
        out[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Zeroes the elements of v at columns >= limit, v holding columns col .. col+7.
__device__ __forceinline__ uint4 mask_cols(uint4 v, int col, int limit)
{
    if (col + 8 <= limit)
        return v;
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if (col + i >= limit)
            w[i >> 1] &= (i & 1) ? 0x0000ffffu : 0xffff0000u;
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Row-segment transpose for the K-grouped GEMMs: src [rows][ld_src] (columns
// [0, c_valid) meaningful, ld_src >= c_valid rounded up to 8), rows grouped by
// expert through offsets; dst [c_pad][ld_dst] with dst[c][koff[e] + j] =
// src[offsets[e] + j][c] for j < rows_e, zero for j in [rows_e, round_up(rows_e, 64))
// and for c in [c_valid, c_pad).  CTA = 64 padded columns of dst (64 consecutive
// rows of one expert) x 256 rows of dst.
__global__ void __launch_bounds__(256) transpose_rows_kernel(
    const bf16 *__restrict__ src, int ld_src, const int32_t *__restrict__ offsets, int E,
    int c_valid, int c_pad, bf16 *__restrict__ dst, int ld_dst)
{
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t s_koff[MOE_MAX_EXPERTS + 1];
    if (threadIdx.x == 0) {
        int k = 0;
        for (int e = 0; e < E; ++e) {
            s_koff[e] = k;
            k += (offsets[e + 1] - offsets[e] + 63) / 64 * 64;
        }
        s_koff[E] = k;
    }
    __syncthreads();
    const int kc0 = blockIdx.x * 64;   // padded column of dst
    const int c0 = blockIdx.y * 256;   // first dst row (src column)
    if (kc0 >= s_koff[E])
        return;
    int e = 0;
    while (kc0 >= s_koff[e + 1])
        ++e;
    const int rows = offsets[e + 1] - offsets[e];
    const int j0 = kc0 - s_koff[e];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int rg = lane & 7, cq = (lane >> 3) + 4 * warp;
    const int col = c0 + 8 * cq;
    if (col >= c_pad)
        return;
    uint4 in[8], out[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int j = j0 + 8 * rg + i;
        in[i] = make_uint4(0, 0, 0, 0);
        if (j < rows && col < c_valid)
            in[i] = mask_cols(*reinterpret_cast<const uint4 *>(
                                  src + (int64_t)(offsets[e] + j) * ld_src + col),
                              col, c_valid);
    }
    transpose8x8(in, out);
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if (col + i < c_pad)
            *reinterpret_cast<uint4 *>(dst + (int64_t)(col + i) * ld_dst + kc0 + 8 * rg) = out[i];
}

// ------------------------------------------------------------------------ host side

struct DevInfo {
    int sms = 0;
    int pair_clusters = 0;
    bool attr[8] = {false, false, false, false, false, false, false, false};
};
static std::mutex g_mu;
static DevInfo g_dev[64];

template <typename Kern>
static cudaError_t set_attr(Kern kern, bool &done, int bytes = SMEM_BYTES)
{
    if (done)
        return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         bytes);
    if (e == cudaSuccess)
        done = true;
    return e;
}

static cudaError_t prepare(DevInfo **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    DevInfo &di = g_dev[dev];
    if (di.sms == 0 &&
        (e = cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    if ((e = set_attr(bwd_gemm_kernel<EPI_STORE, false, true>, di.attr[0])) != cudaSuccess ||
        (e = set_attr(bwd_gemm_kernel<EPI_SWIGLU_BWD, false, false>, di.attr[1])) !=
            cudaSuccess ||
        (e = set_attr(bwd_gemm_kernel<EPI_STORE, true, false>, di.attr[2])) != cudaSuccess ||
        (e = set_attr(pair::bwd_gemm_2sm_kernel<EPI_STORE, false, true>, di.attr[3],
                      pair::SMEM_BYTES)) != cudaSuccess ||
        (e = set_attr(pair::bwd_gemm_2sm_kernel<EPI_SWIGLU_BWD, false, false>, di.attr[4],
                      pair::SMEM_BYTES)) != cudaSuccess ||
        (e = set_attr(pair::bwd_gemm_2sm_kernel<EPI_STORE, true, false>, di.attr[5],
                      pair::SMEM_BYTES)) != cudaSuccess)
        return e;
    if (di.pair_clusters == 0) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * (di.sms / 2));
        cfg.blockDim = dim3(NUM_THREADS);
        cfg.dynamicSmemBytes = pair::SMEM_BYTES;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, pair::bwd_gemm_2sm_kernel<EPI_STORE, false, true>,
                                           &cfg);
        if (e != cudaSuccess)
            return e;
        di.pair_clusters = n > 0 ? n : 1;
    }
    *out = &di;
    return cudaSuccess;
}

// Rows (T*k) from which the 2-SM kernels are used, as in the forward.
constexpr int64_t kPairMinRows = 4096;

// One backward GEMM.  A [a_rows][a_ld] (K extent a_k); B: row-grouped [E][b_rows][b_ld],
// K-grouped [b_rows][b_ld] (K extent b_k); with BT (MN-major B) [E][b_k][b_ld] with N
// extent b_rows; out [out_rows][ld_out], n_valid columns.
template <int EPI, bool KG, bool BT>
static cudaError_t launch(const void *A, uint64_t a_k, uint64_t a_ld, uint64_t a_rows,
                          const void *B, uint64_t b_k, uint64_t b_ld, uint64_t b_rows,
                          const int32_t *offsets, int E, int M, bf16 *out, int ld_out,
                          uint64_t out_rows, int n_valid, const bf16 *dh, int ld_dh,
                          int32_t *status, cudaStream_t s, bool use_pair)
{
    DevInfo *di = nullptr;
    cudaError_t e = prepare(&di);
    if (e != cudaSuccess)
        return e;
    CUtensorMap ta, tb, to;
    const uint64_t da[2] = {a_k, a_rows}, sa[1] = {a_ld * 2};
    const uint32_t ba[2] = {BK, BM};
    const uint32_t b_box = use_pair ? (uint32_t)pair::BNH : (uint32_t)BN;
    if ((e = tc::make_map(&ta, A, 2, da, sa, ba)) != cudaSuccess)
        return e;
    if constexpr (BT) {
        // N innermost: boxes of 64 N x BK K rows, N and K past their extents read as zero
        const uint64_t db[3] = {b_rows, b_k, (uint64_t)E};
        const uint64_t sb[2] = {b_ld * 2, b_k * b_ld * 2};
        const uint32_t bb[3] = {64, BK, 1};
        if ((e = tc::make_map(&tb, B, 3, db, sb, bb)) != cudaSuccess)
            return e;
    } else if constexpr (KG) {
        const uint64_t db[2] = {b_k, b_rows}, sb[1] = {b_ld * 2};
        const uint32_t bb[2] = {BK, b_box};
        if ((e = tc::make_map(&tb, B, 2, db, sb, bb)) != cudaSuccess)
            return e;
    } else {
        const uint64_t db[3] = {b_k, b_rows, (uint64_t)E};
        const uint64_t sb[2] = {b_ld * 2, b_rows * b_ld * 2};
        const uint32_t bb[3] = {BK, b_box, 1};
        if ((e = tc::make_map(&tb, B, 3, db, sb, bb)) != cudaSuccess)
            return e;
    }
    const uint64_t dout[2] = {(uint64_t)n_valid, out_rows}, sout[1] = {(uint64_t)ld_out * 2};
    const uint32_t bout[2] = {32, 32};
    if ((e = tc::make_map(&to, out, 2, dout, sout, bout, CU_TENSOR_MAP_SWIZZLE_64B)) !=
        cudaSuccess)
        return e;
    count_launch();
    if (!use_pair)
        return launch_pdl(bwd_gemm_kernel<EPI, KG, BT>, dim3(di->sms), dim3(NUM_THREADS), SMEM_BYTES,
                          s, ta, tb, to, offsets, E, (int)b_rows, (int)a_k, M, out, ld_out,
                          n_valid, dh, ld_dh, status, wait_limit_ns());
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(2 * di->pair_clusters);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = pair::SMEM_BYTES;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, pair::bwd_gemm_2sm_kernel<EPI, KG, BT>, ta, tb, to, offsets, E,
                              (int)b_rows, (int)a_k, M, out, ld_out, n_valid, dh, ld_dh, status,
                              wait_limit_ns());
}

}  // namespace bwd

using namespace bwd;

// dh [rows][m8] = d_out [rows][d] x W2_e [d][m8] (B MN-major: the packed W2 as it is)
cudaError_t launch_bwd_dh(const moe_params_t *p, const void *d_out, const int32_t *offsets,
                          const void *W2_e, void *dh, int32_t *status, cudaStream_t s)
{
    const uint64_t d = p->d, m8 = round_up(p->m, 8);
    const uint64_t rows = (uint64_t)p->T * p->k;
    return launch<EPI_STORE, false, true>(d_out, d, d, rows, W2_e, d, m8, m8, offsets, p->E, 0,
                                          (bf16 *)dh, (int)m8, rows, (int)m8, nullptr, 0, status,
                                          s, (int64_t)rows >= kPairMinRows);
}

// dGU [rows][2 m16] = SwiGLU backward of (x_perm x W13_e^T) with dh [rows][m8]
cudaError_t launch_bwd_dgu(const moe_params_t *p, const void *x_perm, const int32_t *offsets,
                           const void *W13, const void *dh, void *dgu, int32_t *status,
                           cudaStream_t s)
{
    const uint64_t d = p->d, m8 = round_up(p->m, 8), m16 = round_up(p->m, 16);
    const uint64_t rows = (uint64_t)p->T * p->k;
    return launch<EPI_SWIGLU_BWD, false, false>(x_perm, d, d, rows, W13, d, d, 2 * m16, offsets, p->E,
                                         0, (bf16 *)dgu, (int)(2 * m16), rows, (int)(2 * m16),
                                         (const bf16 *)dh, (int)m8, status, s,
                                         (int64_t)rows >= kPairMinRows);
}

// dx_perm [rows][d] = dGU [rows][2 m16] x W13_e [2 m16][d] (B MN-major: the packed W13)
cudaError_t launch_bwd_dx(const moe_params_t *p, const void *dgu, const int32_t *offsets,
                          const void *W13_e, void *dx_perm, int32_t *status, cudaStream_t s)
{
    const uint64_t d = p->d, m16 = round_up(p->m, 16);
    const uint64_t rows = (uint64_t)p->T * p->k;
    return launch<EPI_STORE, false, true>(dgu, 2 * m16, 2 * m16, rows, W13_e, 2 * m16, d, d,
                                          offsets, p->E, 0, (bf16 *)dx_perm, (int)d, rows, (int)d,
                                          nullptr, 0, status, s, (int64_t)rows >= kPairMinRows);
}

// dW [E][M][n_valid]: A^T [M][kmax] and B^T [b_rows][kmax] in the padded K order
cudaError_t launch_bwd_wgrad(const moe_params_t *p, const void *AT, int M, const void *BT,
                             int b_rows, uint64_t kmax, const int32_t *offsets, void *dW,
                             int ld_dw, int n_valid, int32_t *status, cudaStream_t s)
{
    return launch<EPI_STORE, true, false>(AT, kmax, kmax, (uint64_t)M, BT, kmax, kmax, (uint64_t)b_rows,
                                   offsets, p->E, M, (bf16 *)dW, ld_dw, (uint64_t)p->E * M,
                                   n_valid, nullptr, 0, status, s,
                                   (int64_t)p->T * p->k >= kPairMinRows);
}

cudaError_t launch_transpose_rows(const void *src, int ld_src, const int32_t *offsets, int E,
                                  int c_valid, int c_pad, void *dst, int ld_dst, int64_t kmax,
                                  cudaStream_t s)
{
    count_launch();
    return launch_pdl(transpose_rows_kernel, dim3((unsigned)(kmax / 64), (c_pad + 255) / 256),
                      dim3(256), 0, s, (const bf16 *)src, ld_src, offsets, E, c_valid, c_pad,
                      (bf16 *)dst, ld_dst);
}


}  // namespace moe
