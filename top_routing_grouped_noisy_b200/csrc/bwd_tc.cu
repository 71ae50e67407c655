// bwd_tc.cu -- the grouped GEMMs of the layer's backward pass on the tcgen05
// tensor cores ("LLaMA-MoE v2", code sample "代码实现示例", class Expert, read
// backwards: the gradients of out = W2 (silu(W1 x) * W3 x)).
//
// One persistent kernel, two tile orders:
//   row-grouped (dgrad): C[rows of expert e][N] = A[rows][K] B_e, the rows of expert
//     e being [offsets[e], offsets[e+1]) -- the forward's tile order:
//       dh      = d_out  W2_e        (B = the packed W2_e [d][m8], read MN-major)
//       dGU     = SwiGLU backward of x_perm W13_e^T   (B K-major; fused epilogue, below)
//       dx_perm = dGU    W13_e       (B = the packed W13_e [2 m16][d], read MN-major)
//   K-grouped (wgrad): C_e[M][N] = A_e^T B_e, the reduction running over the rows
//     [offsets[e], offsets[e+1]) of expert e of two row-major activations, both read
//     MN-major (64-wide column chunks of 64 rows):
//       dW2_e  = d_out_e^T h_e       (A = d_out [rows][d], B = h [rows][m8])
//       dW13_e = dGU_e^T x_e         (A = dGU [rows][2 m16], B = x_perm [rows][d])
//     The last K block of an expert also holds the first rows of the next expert:
//     the MMA warp zeroes those K rows of both operands in shared memory before its
//     MMAs.  An expert with no rows gets a zero gradient.
// Operands bf16, loaded by TMA (128-byte swizzle, 4-stage ring); every TMA x
// coordinate is a multiple of 64 elements (128-byte aligned).  f32 accumulators in
// TMEM, double buffered; outputs rounded to bf16 once.
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
    uint64_t tbar[STAGES];  // K-grouped: the copies of an expert's last K block landed
    uint64_t zbar[STAGES];  // K-grouped: the K rows past the expert zeroed
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
// both operands MN-major (bits 15 and 16): the K-grouped wgrad
constexpr uint32_t kIdescMn = kIdesc | (1u << 15) | (1u << 16);
// MN-major operand in shared memory: 64-wide M or N chunks of BK K rows (128 bytes each)
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
                    const float s = __fdividef(1.0f, 1.0f + __expf(-g));  // as the forward
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
    int kv;  // K-grouped: rows of the expert in its last K block (1..BK)
};

// Zeroes K rows [r0, BK) of n MN-major chunks from chunk address base (each K row
// 128 bytes, so the swizzle does not matter); lanes 1..31 of the calling warp.
__device__ __forceinline__ void zero_k_rows(uint32_t base, int n, int r0)
{
    const int lane = threadIdx.x & 31;
    const int per = (BK - r0) * 8;  // 16-byte units per chunk
    for (int i = lane - 1; i < n * per; i += 31) {
        const int c = i / per, rem = i - c * per;
        st_shared_v4(base + (uint32_t)(c * kMnChunkBytes + (r0 + (rem >> 3)) * 128 + (rem & 7) * 16),
                     0u, 0u, 0u, 0u);
    }
}

template <bool KG>
__device__ __forceinline__ Tile decode_tile(const Aux *aux, int tile, int n_tiles, int M,
                                            int num_kb, int order)
{
    Tile t;
    int e = 0;
    while (tile >= aux->tstart[e + 1])
        ++e;
    const int local = tile - aux->tstart[e];
    t.e = e;
    if constexpr (KG) {
        const int mtiles = (M + BM - 1) / BM;
        // order bit 0 clear: m-tiles fastest (concurrent tiles share a B chunk, A_e is
        // reused across n); set: n-tiles fastest (B_e reused across m): the smaller
        // operand stays in L2.  Bits 1 and 2: A and B come as one 3-D box per stage.
        const int mt = (order & 1) ? local / n_tiles : local % mtiles;
        const int nt = (order & 1) ? local % n_tiles : local / mtiles;
        t.a_row = mt * BM;
        t.row0 = e * M + mt * BM;
        t.row_end = e * M + M;
        t.n0 = nt * BN;
        t.k0 = aux->off[e];
        const int rows = aux->off[e + 1] - aux->off[e];
        t.nkb = (rows + BK - 1) / BK;
        t.kv = rows - (t.nkb - 1) * BK;
    } else {
        // bands of `order` m-tiles (0: the whole expert), m-tiles fastest inside a band:
        // concurrent tiles share the band's A rows while it sweeps N
        const int rows = aux->off[e + 1] - aux->off[e];
        const int mtiles = (rows + BM - 1) / BM;
        const int G = (order > 0 && order < mtiles) ? order : mtiles;
        const int bi = local / (G * n_tiles), rem = local - bi * G * n_tiles;
        const int gr = min(G, mtiles - bi * G);
        const int mt = bi * G + rem % gr, nt = rem / gr;
        t.a_row = aux->off[e] + mt * BM;
        t.row0 = t.a_row;
        t.row_end = aux->off[e + 1];
        t.n0 = nt * BN;
        t.k0 = 0;
        t.nkb = num_kb;
        t.kv = BK;
    }
    return t;
}

template <int EPI, bool KG, bool BT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmO, const int32_t *__restrict__ offsets,
                    int E, int N, int K, int M, bf16 *__restrict__ out, int ld_out, int n_valid,
                    const bf16 *__restrict__ dh, int ld_dh, int32_t *status, uint64_t wait_ns,
                    int order)
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
            mbar_init(smem_u32(&aux->tbar[s]), 1);
            mbar_init(smem_u32(&aux->zbar[s]), 1);
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
        // row offsets: the row tiles of the dgrad order, the K ranges of the wgrad order
        int acc = 0;
        for (int e = 0; e < E; ++e) {
            const int rows = offsets[e + 1] - offsets[e];
            aux->tstart[e] = acc;
            aux->off[e] = offsets[e];
            acc += KG ? (M + BM - 1) / BM * n_tiles : (rows + BM - 1) / BM * n_tiles;
        }
        aux->off[E] = offsets[E];
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
            int tfills[STAGES] = {};
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                if (*abort_flag)
                    break;
                const Tile t = decode_tile<KG>(aux, tile, n_tiles, M, num_kb, order);
                for (int kb = 0; kb < t.nkb; ++kb) {
                    if (!mbar_wait(smem_u32(&aux->empty[stage]), phase ^ 1u, wait_ns, abort_flag,
                                   status)) {
                        ok = false;
                        break;
                    }
                    uint32_t fb = smem_u32(&aux->full[stage]);
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    const int kc = t.k0 + kb * BK;
                    if constexpr (KG) {  // both MN-major: 64-wide chunks of BK rows from row kc
                        if (kb == t.nkb - 1 && t.kv < BK) {
                            // an expert's last block: its copies complete on tbar, for lanes
                            // 1-31 to zero the rows past the expert; full completes now
                            mbar_arrive(fb);
                            fb = smem_u32(&aux->tbar[stage]);
                            ++tfills[stage];
                        }
                        mbar_expect_tx(fb, STAGE_BYTES);
                        if (order & 2)  // one 3-D box: the tile's 64-wide chunks of BK rows
                            tma_load_3d(&tmA, fb, sa, 0, kc, t.a_row / 64);
                        else
#pragma unroll
                            for (int j = 0; j < BM / 64; ++j)
                                tma_load_2d(&tmA, fb, sa + j * kMnChunkBytes, t.a_row + 64 * j,
                                            kc);
                        if (order & 4)
                            tma_load_3d(&tmB, fb, sa + A_BYTES, 0, kc, t.n0 / 64);
                        else
#pragma unroll
                            for (int j = 0; j < BN / 64; ++j)
                                tma_load_2d(&tmB, fb, sa + A_BYTES + j * kMnChunkBytes,
                                            t.n0 + 64 * j, kc);
                    } else if constexpr (BT) {  // MN-major B: 64-wide N chunks of BK K rows
                        mbar_expect_tx(fb, STAGE_BYTES);
                        tma_load_2d(&tmA, fb, sa, kc, t.a_row);
#pragma unroll
                        for (int j = 0; j < BN / 64; ++j)
                            tma_load_3d(&tmB, fb, sa + A_BYTES + j * kMnChunkBytes, t.n0 + 64 * j,
                                        kc, t.e);
                    } else {
                        mbar_expect_tx(fb, STAGE_BYTES);
                        tma_load_2d(&tmA, fb, sa, kc, t.a_row);
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
                if (tfills[s] > 0)
                    mbar_drain(smem_u32(&aux->tbar[s]), (uint32_t)((tfills[s] - 1) & 1));
            }
        } else if constexpr (KG) {
            // ------------------------------------------- lanes 1-31: tail zeroing
            // Once an expert's last K block has landed, zero its K rows past the
            // expert in both operands (they hold the next expert's rows) and arrive
            // on zbar, which the MMA issuer waits for.  Lane 1 waits; the other lanes
            // follow its verdict, so the 31 lanes stay converged.
            int stage = 0;
            uint32_t tpar = 0;
            for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
                const Tile t = decode_tile<KG>(aux, tile, n_tiles, M, num_kb, order);
                if (t.nkb > 0 && t.kv < BK) {
                    const int ts = (stage + t.nkb - 1) % STAGES;
                    bool ok = true;
                    if (lane == 1)
                        ok = mbar_wait(smem_u32(&aux->tbar[ts]), (tpar >> ts) & 1u, wait_ns,
                                       abort_flag, status);
                    if (!__shfl_sync(0xfffffffeu, ok ? 1 : 0, 1))
                        break;
                    tpar ^= 1u << ts;
                    const uint32_t sa = smem_base + ts * STAGE_BYTES;
                    zero_k_rows(sa, BM / 64, t.kv);
                    zero_k_rows(sa + A_BYTES, BN / 64, t.kv);
                    fence_proxy_async_smem();
                    __syncwarp(0xfffffffeu);
                    if (lane == 1)
                        mbar_arrive(smem_u32(&aux->zbar[ts]));
                }
                stage = (stage + t.nkb) % STAGES;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------- MMA issuer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t tpar = 0;  // K-grouped: phase parity of each stage's zbar
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const Tile t = decode_tile<KG>(aux, tile, n_tiles, M, num_kb, order);
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
                    if (KG && kb == t.nkb - 1 && t.kv < BK) {  // the K rows past the expert zeroed
                        if (!mbar_wait(smem_u32(&aux->zbar[stage]), (tpar >> stage) & 1u, wait_ns,
                                       abort_flag, status)) {
                            ok = false;
                            break;
                        }
                        tpar ^= 1u << stage;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    const uint64_t da = KG ? tc::sdesc_mn(sa, kMnChunkBytes) : sdesc(sa);
                    const uint64_t db = (KG || BT) ? tc::sdesc_mn(sa + A_BYTES, kMnChunkBytes)
                                                   : sdesc(sa + A_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma_f16(d_tmem, da + (uint64_t)(KG ? kMnKStep * k : 2 * k),
                                 db + (uint64_t)((KG || BT) ? kMnKStep * k : 2 * k),
                                 KG ? kIdescMn : (BT ? kIdescBt : kIdesc), (kb | k) != 0);
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
            const Tile t = decode_tile<KG>(aux, tile, n_tiles, M, num_kb, order);
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
    uint64_t tbar[STAGES];  // K-grouped: the copies of an expert's last K block landed
    uint64_t zbar[STAGES];  // K-grouped: the K rows past the expert zeroed
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
                                            int num_kb, int order)
{
    Tile t;
    int e = 0;
    while (tile >= aux->tstart[e + 1])
        ++e;
    const int local = tile - aux->tstart[e];
    t.e = e;
    if constexpr (KG) {
        const int mtiles = (M + 2 * BM - 1) / (2 * BM);
        const int mt = (order & 1) ? local / n_tiles : local % mtiles;
        const int nt = (order & 1) ? local % n_tiles : local / mtiles;
        t.a_row = mt * 2 * BM;
        t.row0 = e * M + mt * 2 * BM;
        t.row_end = e * M + M;
        t.n0 = nt * BN;
        t.k0 = aux->off[e];
        const int rows = aux->off[e + 1] - aux->off[e];
        t.nkb = (rows + BK - 1) / BK;
        t.kv = rows - (t.nkb - 1) * BK;
    } else {
        const int rows = aux->off[e + 1] - aux->off[e];
        const int mtiles = (rows + 2 * BM - 1) / (2 * BM);
        const int G = (order > 0 && order < mtiles) ? order : mtiles;
        const int bi = local / (G * n_tiles), rem = local - bi * G * n_tiles;
        const int gr = min(G, mtiles - bi * G);
        const int mt = bi * G + rem % gr, nt = rem / gr;
        t.a_row = aux->off[e] + mt * 2 * BM;
        t.row0 = t.a_row;
        t.row_end = aux->off[e + 1];
        t.n0 = nt * BN;
        t.k0 = 0;
        t.nkb = num_kb;
        t.kv = BK;
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
                        const bf16 *__restrict__ dh, int ld_dh, int32_t *status, uint64_t wait_ns,
                    int order)
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
            mbar_init(smem_u32(&aux->tbar[s]), 1);
            mbar_init(smem_u32(&aux->zbar[s]), 2);  // one arrival from each CTA
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
        int acc = 0;
        for (int e = 0; e < E; ++e) {
            const int rows = offsets[e + 1] - offsets[e];
            aux->tstart[e] = acc;
            aux->off[e] = offsets[e];
            acc += KG ? (M + 2 * BM - 1) / (2 * BM) * n_tiles
                      : (rows + 2 * BM - 1) / (2 * BM) * n_tiles;
        }
        aux->off[E] = offsets[E];
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
            int tfills[STAGES] = {};
            bool ok = true;
            for (int tile = cluster_id; tile < total && ok; tile += nclusters) {
                if (*abort_flag)
                    break;
                const Tile t = decode_tile<KG>(aux, tile, n_tiles, M, num_kb, order);
                for (int kb = 0; kb < t.nkb; ++kb) {
                    if (!mbar_wait(smem_u32(&aux->empty[stage]), phase ^ 1u, wait_ns, abort_flag,
                                   status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&aux->full[stage]);
                    const uint32_t fb0 = map_rank(fb, 0);
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    const int kc = t.k0 + kb * BK;
                    if (KG && kb == t.nkb - 1 && t.kv < BK) {
                        // an expert's last block: each CTA's copies complete on its own
                        // tbar, for its lanes 1-31 to zero the rows past the expert; the
                        // leader's full completes now
                        if (leader)
                            mbar_arrive(fb);
                        const uint32_t tb = smem_u32(&aux->tbar[stage]);
                        ++tfills[stage];
                        mbar_expect_tx(tb, STAGE_BYTES);
                        if (order & 2)
                            tma_load_3d(&tmA, tb, sa, 0, kc, (t.a_row + (int)rank * BM) / 64);
                        else
#pragma unroll
                            for (int j = 0; j < BM / 64; ++j)
                                tma_load_2d(&tmA, tb, sa + j * kMnChunkBytes,
                                            t.a_row + (int)rank * BM + 64 * j, kc);
                        if (order & 4)
                            tma_load_3d(&tmB, tb, sa + A_BYTES, 0, kc,
                                        (t.n0 + (int)rank * BNH) / 64);
                        else
#pragma unroll
                            for (int j = 0; j < BNH / 64; ++j)
                                tma_load_2d(&tmB, tb, sa + A_BYTES + j * kMnChunkBytes,
                                            t.n0 + (int)rank * BNH + 64 * j, kc);
                    } else if constexpr (KG) {  // both MN-major: this CTA's 64-wide chunks
                        if (leader)
                            mbar_expect_tx(fb, 2 * STAGE_BYTES);
                        if (order & 2)  // one 3-D box: this CTA's chunks of BK rows
                            tma_load_3d_pair(&tmA, fb0, sa, 0, kc, (t.a_row + (int)rank * BM) / 64);
                        else
#pragma unroll
                            for (int j = 0; j < BM / 64; ++j)
                                tma_load_2d_pair(&tmA, fb0, sa + j * kMnChunkBytes,
                                                 t.a_row + (int)rank * BM + 64 * j, kc);
                        if (order & 4)
                            tma_load_3d_pair(&tmB, fb0, sa + A_BYTES, 0, kc,
                                             (t.n0 + (int)rank * BNH) / 64);
                        else
#pragma unroll
                            for (int j = 0; j < BNH / 64; ++j)
                                tma_load_2d_pair(&tmB, fb0, sa + A_BYTES + j * kMnChunkBytes,
                                                 t.n0 + (int)rank * BNH + 64 * j, kc);
                    } else if constexpr (BT) {
                        if (leader)
                            mbar_expect_tx(fb, 2 * STAGE_BYTES);  // MN-major B: this CTA's 64-wide N chunks
                        tma_load_2d_pair(&tmA, fb0, sa, kc, t.a_row + (int)rank * BM);
#pragma unroll
                        for (int j = 0; j < BNH / 64; ++j)
                            tma_load_3d_pair(&tmB, fb0, sa + A_BYTES + j * kMnChunkBytes,
                                             t.n0 + (int)rank * BNH + 64 * j, kc, t.e);
                    } else {
                        if (leader)
                            mbar_expect_tx(fb, 2 * STAGE_BYTES);
                        tma_load_2d_pair(&tmA, fb0, sa, kc, t.a_row + (int)rank * BM);
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
            for (int s = 0; s < STAGES; ++s)
                if (tfills[s] > 0)
                    mbar_drain(smem_u32(&aux->tbar[s]), (uint32_t)((tfills[s] - 1) & 1));
        } else if constexpr (KG) {
            // ------------------------------------------- lanes 1-31: tail zeroing
            // As in the 1-SM kernel, in this CTA's tiles; the arrival goes to the
            // leader's zbar (count 2, one per CTA).
            int stage = 0;
            uint32_t tpar = 0;
            for (int tile = cluster_id; tile < total; tile += nclusters) {
                const Tile t = decode_tile<KG>(aux, tile, n_tiles, M, num_kb, order);
                if (t.nkb > 0 && t.kv < BK) {
                    const int ts = (stage + t.nkb - 1) % STAGES;
                    bool ok = true;
                    if (lane == 1)
                        ok = mbar_wait(smem_u32(&aux->tbar[ts]), (tpar >> ts) & 1u, wait_ns,
                                       abort_flag, status);
                    if (!__shfl_sync(0xfffffffeu, ok ? 1 : 0, 1))
                        break;
                    tpar ^= 1u << ts;
                    const uint32_t sa = smem_base + ts * STAGE_BYTES;
                    zero_k_rows(sa, BM / 64, t.kv);
                    zero_k_rows(sa + A_BYTES, BNH / 64, t.kv);
                    fence_proxy_async_smem();
                    __syncwarp(0xfffffffeu);
                    if (lane == 1)
                        mbar_arrive_cluster(map_rank(smem_u32(&aux->zbar[ts]), 0));
                }
                stage = (stage + t.nkb) % STAGES;
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------------------- MMA issuer (leader)
            int stage = 0;
            uint32_t phase = 0;
            uint32_t tpar = 0;  // K-grouped: phase parity of each stage's zbar
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = cluster_id; tile < total && ok; tile += nclusters) {
                const Tile t = decode_tile<KG>(aux, tile, n_tiles, M, num_kb, order);
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
                    if (KG && kb == t.nkb - 1 && t.kv < BK) {  // both CTAs' tails zeroed
                        if (!mbar_wait(smem_u32(&aux->zbar[stage]), (tpar >> stage) & 1u, wait_ns,
                                       abort_flag, status)) {
                            ok = false;
                            break;
                        }
                        tpar ^= 1u << stage;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    const uint64_t da = KG ? tc::sdesc_mn(sa, kMnChunkBytes) : sdesc(sa);
                    const uint64_t db = (KG || BT) ? tc::sdesc_mn(sa + A_BYTES, kMnChunkBytes)
                                                   : sdesc(sa + A_BYTES);
                    const uint32_t idesc = KG ? kIdesc2 | (1u << 15) | (1u << 16)
                                              : (BT ? kIdesc2 | (1u << 16) : kIdesc2);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma_pair(d_tmem, da + (uint64_t)(KG ? kMnKStep * k : 2 * k),
                                  db + (uint64_t)((KG || BT) ? kMnKStep * k : 2 * k), idesc,
                                  (kb | k) != 0);
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
            const Tile t = decode_tile<KG>(aux, tile, n_tiles, M, num_kb, order);
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

// One backward GEMM; out [out_rows][ld_out], n_valid columns.
//   row-grouped: A [a_rows][a_ld] (K extent a_k); B [E][b_rows][b_ld] (K extent b_k),
//     with BT (MN-major B) [E][b_k][b_ld] with N extent b_rows.
//   K-grouped: A [a_rows][a_ld] with M extent a_k, B [a_rows][b_ld] with N extent
//     b_rows (rows = the experts' rows, the K of the reduction; b_k unused).
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
    const uint32_t b_box = use_pair ? (uint32_t)pair::BNH : (uint32_t)BN;
    // K-grouped operands whose column count is a multiple of 64 load a stage's 64-wide
    // chunks with one 3-D box (columns within a chunk, rows, chunks)
    const bool a3d = KG && a_k % 64 == 0, b3d = KG && b_rows % 64 == 0;
    if (a3d) {
        const uint64_t da[3] = {64, a_rows, a_k / 64}, sa[2] = {a_ld * 2, 128};
        const uint32_t ba[3] = {64, BK, BM / 64};
        if ((e = tc::make_map(&ta, A, 3, da, sa, ba)) != cudaSuccess)
            return e;
    } else {
        const uint64_t da[2] = {a_k, a_rows}, sa[1] = {a_ld * 2};
        const uint32_t ba[2] = {KG ? 64u : (uint32_t)BK, KG ? (uint32_t)BK : (uint32_t)BM};
        if ((e = tc::make_map(&ta, A, 2, da, sa, ba)) != cudaSuccess)
            return e;
    }
    if constexpr (KG) {
        // MN-major boxes of 64 columns x BK rows; columns and rows past the extents
        // read as zero
        if (b3d) {
            const uint64_t db[3] = {64, a_rows, b_rows / 64}, sb[2] = {b_ld * 2, 128};
            const uint32_t bb[3] = {64, BK, b_box / 64};
            if ((e = tc::make_map(&tb, B, 3, db, sb, bb)) != cudaSuccess)
                return e;
        } else {
            const uint64_t db[2] = {b_rows, a_rows}, sb[1] = {b_ld * 2};
            const uint32_t bb[2] = {64, BK};
            if ((e = tc::make_map(&tb, B, 2, db, sb, bb)) != cudaSuccess)
                return e;
        }
    } else if constexpr (BT) {
        // N innermost: boxes of 64 N x BK K rows, N and K past their extents read as zero
        const uint64_t db[3] = {b_rows, b_k, (uint64_t)E};
        const uint64_t sb[2] = {b_ld * 2, b_k * b_ld * 2};
        const uint32_t bb[3] = {64, BK, 1};
        if ((e = tc::make_map(&tb, B, 3, db, sb, bb)) != cudaSuccess)
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
    // tile order: K-grouped, n-tiles fastest when B_e (N columns) is the smaller
    // operand; row-grouped, bands of m-tiles whose A rows take ~16 MB
    int order = 0;
    if constexpr (KG) {
        order = (b_rows < (uint64_t)M ? 1 : 0) | (a3d ? 2 : 0) | (b3d ? 4 : 0);
    } else {
        const uint64_t tile_a = (use_pair ? 2ull : 1ull) * BM * a_k * 2;
        const uint64_t g = (16ull << 20) / (tile_a > 0 ? tile_a : 1);
        order = g < 1 ? 1 : (int)(g > 1024 ? 1024 : g);
    }
    count_launch();
    if (!use_pair)
        return launch_pdl(bwd_gemm_kernel<EPI, KG, BT>, dim3(di->sms), dim3(NUM_THREADS), SMEM_BYTES,
                          s, ta, tb, to, offsets, E, (int)b_rows, (int)a_k, M, out, ld_out,
                          n_valid, dh, ld_dh, status, wait_limit_ns(), order);
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
                              wait_limit_ns(), order);
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

// dW [E][M][n_valid] (ld_dw): dW_e = A_e^T B_e over the rows of expert e, A [rows][a_ld]
// with M columns, B [rows][b_ld] with n_cols columns (N extent; columns up to the next
// multiple of 256 read as zero)
cudaError_t launch_bwd_wgrad(const moe_params_t *p, const void *A, int M, int a_ld, const void *B,
                             int n_cols, int b_ld, const int32_t *offsets, void *dW, int ld_dw,
                             int n_valid, int32_t *status, cudaStream_t s)
{
    const uint64_t rows = (uint64_t)p->T * p->k;
    return launch<EPI_STORE, true, false>(A, (uint64_t)M, (uint64_t)a_ld, rows, B, 0,
                                          (uint64_t)b_ld, (uint64_t)n_cols, offsets, p->E, M,
                                          (bf16 *)dW, ld_dw, (uint64_t)p->E * M, n_valid, nullptr,
                                          0, status, s, (int64_t)rows >= kPairMinRows);
}

}  // namespace moe
