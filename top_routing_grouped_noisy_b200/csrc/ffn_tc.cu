// ffn_tc.cu -- a3/a4 for bf16 layers: one persistent grouped GEMM kernel on the
// 5th-generation tensor cores (tcgen05.mma, accumulators in TMEM, operands
// staged by TMA), used twice:
//   a3: h   = silu(x_perm W1_e^T) * (x_perm W3_e^T)   (fused SwiGLU epilogue)
//   a4: out = h W2_e^T                                 (plain epilogue)
// ("LLaMA-MoE v2", code sample "代码实现示例", class Expert).
//
// Work: tiles of 128 rows x 256 columns over every expert e, the rows of expert e
// being [offsets[e], offsets[e+1]) of the row-permuted activations; the tile list
// is built on the device from the offsets, so no host round trip is needed.
// Both operands are K-major bf16; TMA copies 128x64 (A) and 256x64 (B) boxes with
// 128-byte swizzle into a 4-stage shared-memory ring; K tails, N tails and rows
// past the end of the buffer come back as zeros from TMA.  f32 accumulators live
// in TMEM, double-buffered (2 x 256 columns), so the epilogue of one tile
// overlaps the main loop of the next.
//
// Warp roles (320 threads, one CTA per SM, grid = #SMs):
//   warp 0     TMA producer (lane 0; every lane in the row-gathering variant)
//   warp 1     TMEM allocator and MMA issuer (one lane)
//   warps 2-9  epilogue: tcgen05.ld -> registers -> bf16 -> global; warp w reads
//              TMEM lanes 32*(w%4)..+31, i.e. tile rows, one row per thread, and
//              half of the 256 accumulator columns (warps 2-5 the first half).
// For a3 the packed W13 layout puts, in each 32-row group, 16 W1 rows and then the
// 16 W3 rows of the same 16 neurons, so each 32-column TMEM load holds the gate
// and up values of 16 neurons of the thread's row.
//
// Every mbarrier wait is bounded (%globaltimer): past the limit the kernel records
// MOE_ERR_DEVICE_TIMEOUT, every role stops, in-flight TMA copies and MMAs are
// drained (bounded again) and TMEM is freed before the CTA exits.  No TMA load here
// uses cluster multicast.
#include <atomic>
#include <mutex>

#include "tc_common.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;  // 64 bf16 = 128 bytes: one swizzle-128B row
constexpr int kABoxRows = 64;  // rows of one A box (two per 128-row tile)
constexpr int STAGES = 4;
constexpr int kMaxStages = 8;  // stages of the small-batch 160-wide tiles
constexpr int ACC = 2;
constexpr int TMEM_COLS = ACC * BN;  // 512
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TILE_BYTES = STAGES * STAGE_BYTES;
constexpr int NUM_THREADS = 320;  // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue
constexpr int EPI_WARPS = 8;

enum { EPI_SWIGLU = 0, EPI_STORE = 1 };

struct Aux {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t tfull[ACC];
    uint64_t tempty[ACC];
    uint64_t drain;
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t off[MOE_MAX_EXPERTS + 1];
    int32_t tstart[MOE_MAX_EXPERTS + 1];
};
constexpr int SMEM_BYTES = 1024 + TILE_BYTES + 8 * 2 * 32 * 64 + (int)sizeof(Aux);

// kind::f16 instruction descriptors (D f32, A and B bf16, both K-major, M = BM) are
// per tile width: Geo<BNT>::IDESC.

// Output staging: each epilogue warp owns two 2 KB shared-memory slots, each one
// [32 rows][64 bytes] box laid out with the 64-byte swizzle (16-byte chunk j of row
// r at r*64 + ((j ^ ((r >> 1) & 3)) * 16)), the layout the output tensor map's
// SWIZZLE_64B expects; the 32 lanes write their rows without bank conflicts.
constexpr int kStageSlotBytes = 32 * 64;
constexpr int kEpiStageBytes = 8 /* warps */ * 2 * kStageSlotBytes;

// Geometry of a 1-SM kernel instance with tiles BNT columns wide: 256, or 160 when
// the narrower tile puts every tile of a small batch on an SM of its own (a batch of
// at most 128 rows per expert has one row tile per expert, E x ceil(N / BNT) tiles).
// The accumulators keep the 256-column TMEM stride.  SMALL (every tile at most 64
// rows): a stage holds one 64-row A box and the B box -- the MMA's other 64 A rows are
// the first bytes of the B box, and only make accumulator rows nobody stores -- and
// the epilogue writes per lane without staging, so the ring gets the space: 8 stages
// of 160-wide tiles, 5 of 256-wide ones.
template <int BNT, bool SMALL = false>
struct Geo {
    static constexpr int A_REGION = SMALL ? kABoxRows * BK * 2 : A_BYTES;
    static constexpr int B_BYTES = BNT * BK * 2;
    static constexpr int STAGE_BYTES = A_REGION + B_BYTES;
    static constexpr int EPI_BYTES = SMALL ? 0 : kEpiStageBytes;
    static constexpr int FIXED_BYTES = 1024 + EPI_BYTES + (int)sizeof(Aux);
    static constexpr int FIT = (227 * 1024 - FIXED_BYTES) / STAGE_BYTES;
    static constexpr int NSTAGES =
        SMALL ? (FIT < kMaxStages ? FIT : kMaxStages) : (BNT == BN ? STAGES : 5);
    static constexpr int TILE_BYTES = NSTAGES * STAGE_BYTES;
    static constexpr int SMEM_BYTES = FIXED_BYTES + TILE_BYTES;
    static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) |
                                      ((uint32_t)(BNT >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
    static_assert(BNT % 32 == 0 && BNT <= BN && STAGE_BYTES % 1024 == 0, "tile width");
    static_assert(A_BYTES <= STAGE_BYTES, "the MMA's 128 A rows lie inside the stage");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    static_assert(SMEM_BYTES > 114 * 1024,
                  "one CTA per SM: the kernel allocates TMEM before its wait on the previous grid");
};
constexpr int kNarrowBN = 160;


struct EpiStore {
    const CUtensorMap *map;  // output [rows][cols], box {32 cols, 32 rows}, SWIZZLE_64B
    uint32_t slots;          // this warp's two slots (1024-byte aligned)
    int slot;                // slot to use next
};

// Writes 32 bf16 values (16 packed words) of this lane's row into the next slot and
// stores the warp's 32 x 32 box at (col, row0) with one bulk tensor store.
__device__ __forceinline__ void stage_box(EpiStore &st, const uint32_t (&pk)[16], int col, int row0)
{
    const int lane = threadIdx.x & 31;
    if (lane == 0)
        bulk_wait_read_1();  // the slot's previous store has finished reading it
    __syncwarp();
    const uint32_t base = st.slots + (uint32_t)(st.slot * kStageSlotBytes) + (uint32_t)(lane * 64);
#pragma unroll
    for (int j = 0; j < 4; ++j)
        st_shared_v4(base + (uint32_t)(((j ^ ((lane >> 1) & 3)) << 4)), pk[4 * j], pk[4 * j + 1],
                     pk[4 * j + 2], pk[4 * j + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d_evict_first(st.map, st.slots + (uint32_t)(st.slot * kStageSlotBytes), col,
                                 row0);
        bulk_commit();
    }
    st.slot ^= 1;
}

// Epilogue of the warp's 32-row slab (one row per lane), 32-column chunks
// [c_first, c_first + n_chunks) of the tile starting at output column n0.
//   SwiGLU: columns 32c..32c+15 are gate and 32c+16..32c+31 up of neurons
//           n0/2 + 16c + i; h = silu(gate) * up, rounded to bf16.
//   Store:  the 32 columns rounded to bf16.
// Boxes wholly inside the expert's rows and the valid columns go out through the
// staging slots as bulk tensor stores; the others are written per lane, masked.
template <int EPI, bool NOSTAGE = false>
__device__ __forceinline__ void epilogue_slab(uint32_t taddr, int c_first, int n_chunks,
                                              int row0, int row_end, int n0,
                                              bf16 *__restrict__ out, int ld_out, int n_valid,
                                              EpiStore &st)
{
    const int lane = threadIdx.x & 31;
    const int row = row0 + lane;
    const bool rv = row < row_end;
    const bool full_rows = !NOSTAGE && row0 + 32 <= row_end;  // NOSTAGE: no staging slots
#pragma unroll 1
    for (int c = c_first; c < c_first + n_chunks; c += 2) {
        uint32_t v[2][32];
        if (c + 1 == c_first + n_chunks) {
            // an odd last chunk (160-column tiles): 32 columns, stored per lane
            tmem_ld32_async(taddr + (uint32_t)(c * 32), v[0]);
            tmem_wait_ld();
            if constexpr (EPI == EPI_SWIGLU) {
                const int nb = n0 / 2 + c * 16;  // 16 neurons
                float hv[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float g = __uint_as_float(v[0][i]);
                    const float u = __uint_as_float(v[0][16 + i]);
                    hv[i] = __fdividef(g, 1.0f + __expf(-g)) * u;  // see below
                }
                if (rv && nb < n_valid) {
                    bf16 *dst = out + (int64_t)row * ld_out + nb;
                    if (nb + 16 <= n_valid) {
                        st_v4(dst, f32x8_to_bf16(hv));
                        st_v4(dst + 8, f32x8_to_bf16(hv + 8));
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i)  // unrolled: hv stays in registers
                            if (nb + i < n_valid)
                                dst[i] = __float2bfloat16_rn(hv[i]);
                    }
                }
            } else {
                const int col = n0 + c * 32;
                if (rv) {
                    bf16 *dst = out + (int64_t)row * ld_out + col;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (col + q * 8 < n_valid) {
                            float f[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                f[i] = __uint_as_float(v[0][q * 8 + i]);
                            st_v4(dst + q * 8, f32x8_to_bf16(f));
                        }
                    }
                }
            }
            break;
        }
        tmem_ld32_async(taddr + (uint32_t)(c * 32), v[0]);
        tmem_ld32_async(taddr + (uint32_t)((c + 1) * 32), v[1]);
        tmem_wait_ld();
        if constexpr (EPI == EPI_SWIGLU) {
            const int nb = n0 / 2 + c * 16;  // 32 neurons: 16 from each chunk
            float hv[32];
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2)
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float g = __uint_as_float(v[q2][i]);
                    const float u = __uint_as_float(v[q2][16 + i]);
                    // approximate division (2 ulp, 0 once 1 + e^-g > 2^126, silu's limit):
                    // the IEEE quotient's longer code took the small-batch epilogue
                    // from about 1 to 9 us; h is rounded to bf16 either way
                    hv[q2 * 16 + i] = __fdividef(g, 1.0f + __expf(-g)) * u;
                }
            if (full_rows && nb + 32 <= n_valid) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(hv[2 * i], hv[2 * i + 1]);
                stage_box(st, pk, nb, row0);
            } else if (rv && nb < n_valid) {
                bf16 *dst = out + (int64_t)row * ld_out + nb;
                if (nb + 32 <= n_valid) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        st_v4(dst + 8 * q, f32x8_to_bf16(hv + 8 * q));
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (nb + i < n_valid)
                            dst[i] = __float2bfloat16_rn(hv[i]);
                }
            }
        } else {
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                const int col = n0 + (c + q2) * 32;
                if (full_rows && col + 32 <= n_valid) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[i] = pack_bf16x2(__uint_as_float(v[q2][2 * i]),
                                            __uint_as_float(v[q2][2 * i + 1]));
                    stage_box(st, pk, col, row0);
                } else if (rv) {
                    bf16 *dst = out + (int64_t)row * ld_out + col;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (col + q * 8 < n_valid) {  // n_valid is a multiple of 8
                            float f[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                f[i] = __uint_as_float(v[q2][q * 8 + i]);
                            st_v4(dst + q * 8, f32x8_to_bf16(f));
                        }
                    }
                }
            }
        }
    }
}

struct Tile {
    int e, row0, row_end, n0;
};

template <int BNT>
__device__ __forceinline__ Tile decode_tile(const Aux *aux, int tile, int n_tiles)
{
    Tile t;
    int e = 0;
    while (tile >= aux->tstart[e + 1])
        ++e;
    const int local = tile - aux->tstart[e];
    const int rows = aux->off[e + 1] - aux->off[e];
    const int mtiles = (rows + BM - 1) / BM;
    const int mt = local % mtiles, nt = local / mtiles;
    (void)n_tiles;
    t.e = e;
    t.row0 = aux->off[e] + mt * BM;
    t.row_end = aux->off[e + 1];
    t.n0 = nt * BNT;
    return t;
}

// Without GATHER, tmA's box is 64 rows high: a tile with at most 64 rows (every tile of
// a batch of at most 64 tokens) loads one box per stage, others two.  The MMA always
// reads 128 rows; rows a tile does not load keep whatever the stage held and only make
// accumulator rows past the tile's last row, which the epilogue never stores.
// GATHER: tmA covers the unpermuted activations x [T][K] with a box one row high;
// the A rows of a tile are gathered through row_token (4 rows per TMA, one TMA
// per producer lane) instead of being read from a permuted copy.
template <int EPI, bool GATHER, int BNT = BN, bool SMALL = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmO,
                        const int32_t *__restrict__ offsets, int E, int N, int K,
                        bf16 *__restrict__ out, int ld_out, int n_valid, int32_t *status,
                        uint64_t wait_ns, const int32_t *__restrict__ row_token, int pf_kb)
{
    // The expert weights are inputs no earlier kernel writes, so they may be read
    // before the wait on the previous grid.  With at most one row tile per expert (the
    // host passes pf_kb > 0 only then) tile b is column tile b % n_tiles of expert
    // b / n_tiles whenever every expert has rows: the first pf_kb K blocks of that
    // weight tile go to L2 while the routing kernels still run (an expert without rows
    // only wastes its prefetch).
    if (pf_kb > 0 && threadIdx.x == 0) {
        const int nt = (N + BNT - 1) / BNT;
        if ((int)blockIdx.x < E * nt) {
            const int e = (int)blockIdx.x / nt, n0 = ((int)blockIdx.x % nt) * BNT;
            const int kbs = min(pf_kb, (K + BK - 1) / BK);
            for (int kb = 0; kb < kbs; ++kb)
                tma_prefetch_l2_3d(&tmB, kb * BK, n0, e);
        }
    }
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    using G = Geo<BNT, SMALL>;
    Aux *aux = reinterpret_cast<Aux *>(smem + G::TILE_BYTES + G::EPI_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int32_t *abort_flag = &aux->abort_flag;

    if (threadIdx.x == 0) {
        for (int s = 0; s < G::NSTAGES; ++s) {
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
    // The barriers and TMEM are set up before the wait on the previous grid: no kernel of
    // the library that holds TMEM can share an SM with this one (each takes more than half
    // of the shared memory), so the allocation cannot wait on a CTA that waits on us.
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&aux->tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    pdl_wait();
    pdl_trigger();
    const int n_tiles = (N + BNT - 1) / BNT;
    if (warp == 2) {
        for (int i = lane; i <= E; i += 32)
            aux->off[i] = offsets[i];
        __syncwarp();
        if (lane == 0) {
            int acc = 0;
            for (int e = 0; e < E; ++e) {
                aux->tstart[e] = acc;
                const int rows = aux->off[e + 1] - aux->off[e];
                acc += (rows + BM - 1) / BM * n_tiles;
            }
            aux->tstart[E] = acc;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = aux->tmem_base;
    const int total = aux->tstart[E];
    const int num_kb = (K + BK - 1) / BK;
    const uint32_t smem_base = smem_u32(smem);

    if (warp == 0) {
        // -------------------------------------------------------------- TMA producer
        // lane 0 waits for and arms each stage; in GATHER mode every lane then
        // fetches four A rows, otherwise lane 0 copies the A box
        int stage = 0;
        uint32_t phase = 0;
        int64_t fills = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            if (__shfl_sync(0xffffffffu, (int)*abort_flag, 0))
                break;
            const Tile t = decode_tile<BNT>(aux, tile, n_tiles);
            // A rows landing per stage: gather4 fills all BM rows; a SMALL stage has room
            // for one box (more rows than that: offsets no dispatch can give, reported)
            const bool big = t.row_end - t.row0 > kABoxRows;
            if (SMALL && big && lane == 0)
                set_status(status, MOE_ERR_DEVICE_BADINDEX);
            const int a_boxes = GATHER ? BM / kABoxRows : (big && !SMALL ? 2 : 1);
            int src[4] = {0, 0, 0, 0};
            if constexpr (GATHER) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = t.row0 + 4 * lane + i;
                    src[i] = row_token[r < t.row_end ? r : t.row_end - 1];
                }
            }
            bool ok = true;
            for (int kb = 0; kb < num_kb; ++kb) {
                int w_ok = 1;
                if (lane == 0)
                    w_ok = mbar_wait(smem_u32(&aux->empty[stage]), phase ^ 1u, wait_ns,
                                     abort_flag, status);
                if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = smem_u32(&aux->full[stage]);
                const uint32_t sa = smem_base + stage * G::STAGE_BYTES;
                if (lane == 0)
                    mbar_expect_tx(fb, (uint32_t)(a_boxes * kABoxRows * BK * 2 +
                                                  G::B_BYTES));
                __syncwarp();
                if constexpr (GATHER)
                    tma_gather4(&tmA, fb, sa + lane * 4 * 128, kb * BK, src[0], src[1], src[2],
                                src[3]);
                else if (lane == 0) {
                    tma_load_2d(&tmA, fb, sa, kb * BK, t.row0);
                    if (a_boxes == 2)
                        tma_load_2d(&tmA, fb, sa + kABoxRows * BK * 2, kb * BK,
                                    t.row0 + kABoxRows);
                }
                if (lane == 0)
                    tma_load_3d(&tmB, fb, sa + G::A_REGION, kb * BK, t.n0, t.e);
                ++fills;
                if (++stage == G::NSTAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok)
                break;
        }
        // drain: the last fill of every stage has landed before the CTA may exit
        if (lane == 0) {
            for (int s = 0; s < G::NSTAGES; ++s) {
                const int64_t n = fills / G::NSTAGES + (s < fills % G::NSTAGES ? 1 : 0);
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
                if (!mbar_wait(smem_u32(&aux->tempty[acc]), acc_phase ^ 1u, wait_ns, abort_flag,
                               status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(smem_u32(&aux->full[stage]), phase, wait_ns, abort_flag,
                                   status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_base + stage * G::STAGE_BYTES;
                    const uint64_t da = sdesc(sa), db = sdesc(sa + G::A_REGION);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)  // +32 bytes (16 bf16) per step
                        umma_f16(d_tmem, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k),
                                 G::IDESC, (kb | k) != 0);
                    umma_commit(smem_u32(&aux->empty[stage]));
                    if (++stage == G::NSTAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                umma_commit(smem_u32(&aux->tfull[acc]));
                if (++acc == ACC) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // drain: every MMA issued by this thread has completed
            umma_commit(smem_u32(&aux->drain));
            mbar_drain(smem_u32(&aux->drain), 0);
        }
    } else {
        // -------------------------------------------------------------- epilogue
        // warp w reads TMEM lanes 32*(w%4)..+31 (tile rows); warps 2-5 take the first
        // half of the accumulator's 32-column chunks (the larger half of an odd
        // count), warps 6-9 the rest
        const int wq = warp & 3;
        const int lane_base = wq * 32;
        constexpr int kChunks = BNT / 32, kHalf0 = (kChunks + 1) / 2;
        const bool upper = (warp - 2) / 4 != 0;
        const int c_first = upper ? kHalf0 : 0, n_chunks = upper ? kChunks - kHalf0 : kHalf0;
        EpiStore st{&tmO, smem_base + G::TILE_BYTES + (uint32_t)((warp - 2) * 2 * kStageSlotBytes), 0};
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const Tile t = decode_tile<BNT>(aux, tile, n_tiles);
            if (!mbar_wait(smem_u32(&aux->tfull[acc]), acc_phase, wait_ns, abort_flag, status))
                break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)lane_base << 16) + (uint32_t)(acc * BN);
            if (!SMALL || t.row0 + lane_base < t.row_end)  // SMALL: warps past the rows idle
                epilogue_slab<EPI, SMALL>(taddr, c_first, n_chunks, t.row0 + lane_base,
                                          t.row_end, t.n0, out, ld_out, n_valid, st);
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
            bulk_wait_all();  // this lane's output stores are done before the CTA exits
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
// The same grouped GEMM with cta_group::2: a cluster of two CTAs (two SMs) owns a
// 256 x 256 output tile.  CTA r of the pair loads rows [128r, 128r+128) of the A
// tile and rows [128r, 128r+128) of the B tile (half of N); the leader (r = 0)
// issues tcgen05.mma.cta_group::2 with M = 256, which reads A from each CTA's own
// shared memory and B from both, and writes each CTA's 128 accumulator rows
// (all 256 columns) into that CTA's TMEM.  Per CTA a K slab is 32 KB instead of
// 48 KB for the same 128 x 256 x 64 of MMA work, which relieves shared-memory
// bandwidth, the limit of the 1-SM kernel.
//   full[s]   leader only: the leader's producer expects both CTAs' bytes; both
//             CTAs' TMA loads complete on it
//   empty[s]  both CTAs: the leader's commit arrives on both (multicast commit)
//   tfull[a]  both CTAs: the leader's commit arrives on both
//   tempty[a] leader only: 4 epilogue warps of each CTA arrive (remote for r = 1)
// Loads carry no multicast qualifier.
namespace tc2 {

constexpr int BM = 128;   // rows per CTA (256 per pair)
constexpr int BN = 256;   // columns per pair tile
constexpr int BNH = 128;  // B rows loaded by each CTA
constexpr int BK = 64;
constexpr int STAGES = 6;
constexpr int ACC = 2;
constexpr int TMEM_COLS = ACC * BN;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BNH * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TILE_BYTES = STAGES * STAGE_BYTES;
constexpr int NUM_THREADS = 320;  // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue
constexpr int EPI_WARPS = 8;
constexpr uint64_t kAbortSettleNs = 200000ull;  // pause before exit after an abort

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
constexpr int SMEM_BYTES = 1024 + TILE_BYTES + tc::kEpiStageBytes + (int)sizeof(Aux);

// kind::f16, D f32, A/B bf16 K-major, N = 256, M = 256 (the pair)
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
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

// shared::cluster address of the same shared variable in CTA `rank` of the cluster
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

__device__ __forceinline__ void tma_gather4_pair(const CUtensorMap *map, uint32_t bar_cluster,
                                                 uint32_t dst, int col, int r0, int r1, int r2,
                                                 int r3)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile::gather4.mbarrier::"
        "complete_tx::bytes [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(col), "r"(r0), "r"(r1),
        "r"(r2), "r"(r3)
        : "memory");
}

__device__ __forceinline__ void umma_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(kIdesc), "r"(acc)
        : "memory");
}

// arrive on the barrier at this shared offset in both CTAs of the pair
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

struct PairTile {
    int e, row0, row_end, n0;
};

// Tile order inside an expert: bands of `band` m-tiles (0: the whole expert, split
// into equal bands), m-tiles fastest inside a band, then the band's n-tiles, then the
// next band.  Clusters working at the same time share one band of A rows (kept in L2
// while the band sweeps N) and the few B tiles of its current n-tiles.
__device__ __forceinline__ PairTile decode_pair_tile(const Aux *aux, int tile, int n_tiles,
                                                     int band)
{
    PairTile t;
    int e = 0;
    while (tile >= aux->tstart[e + 1])
        ++e;
    const int local = tile - aux->tstart[e];
    const int rows = aux->off[e + 1] - aux->off[e];
    const int mtiles = (rows + 2 * BM - 1) / (2 * BM);
    int G = (band > 0 && band < mtiles) ? band : mtiles;
    const int nbands = (mtiles + G - 1) / G;
    G = (mtiles + nbands - 1) / nbands;
    const int bi = local / (G * n_tiles);
    const int rem = local - bi * G * n_tiles;
    const int gr = mtiles - bi * G < G ? mtiles - bi * G : G;
    const int mt = bi * G + rem % gr, nt = rem / gr;
    t.e = e;
    t.row0 = aux->off[e] + mt * 2 * BM;
    t.row_end = aux->off[e + 1];
    t.n0 = nt * BN;
    return t;
}

template <int EPI, bool GATHER>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_2sm_kernel(const __grid_constant__ CUtensorMap tmA,
                            const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmO,
                            const int32_t *__restrict__ offsets, int E, int N, int K,
                            bf16 *__restrict__ out, int ld_out, int n_valid, int32_t *status,
                            uint64_t wait_ns, const int32_t *__restrict__ row_token, int band)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Aux *aux = reinterpret_cast<Aux *>(smem + TILE_BYTES + tc::kEpiStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int32_t *abort_flag = &aux->abort_flag;
    const uint32_t rank = cta_rank();
    const bool leader = rank == 0;
    const int cluster_id = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(tc::smem_u32(&aux->full[s]), 1);
            tc::mbar_init(tc::smem_u32(&aux->empty[s]), 1);
        }
        for (int a = 0; a < ACC; ++a) {
            tc::mbar_init(tc::smem_u32(&aux->tfull[a]), 1);
            tc::mbar_init(tc::smem_u32(&aux->tempty[a]), 2 * EPI_WARPS);
        }
        tc::mbar_init(tc::smem_u32(&aux->drain), 1);
        aux->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmO)) : "memory");
    }
    const int n_tiles = (N + BN - 1) / BN;
    if (warp == 2) {
        for (int i = lane; i <= E; i += 32)
            aux->off[i] = offsets[i];
        __syncwarp();
        if (lane == 0) {
            int acc = 0;
            for (int e = 0; e < E; ++e) {
                aux->tstart[e] = acc;
                const int rows = aux->off[e + 1] - aux->off[e];
                acc += (rows + 2 * BM - 1) / (2 * BM) * n_tiles;
            }
            aux->tstart[E] = acc;
        }
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         tc::smem_u32(&aux->tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc::tc_fence_before();
    cluster_sync();  // both CTAs' barriers exist before either signals the other's
    tc::tc_fence_after();
    const uint32_t tmem_base = aux->tmem_base;
    const int total = aux->tstart[E];
    const int num_kb = (K + BK - 1) / BK;
    const uint32_t smem_base = tc::smem_u32(smem);

    if (warp == 0) {
        // -------------------------------------------------------------- TMA producer (both)
        int stage = 0;
        uint32_t phase = 0;
        int64_t fills = 0;
        for (int tile = cluster_id; tile < total; tile += nclusters) {
            if (__shfl_sync(0xffffffffu, (int)*abort_flag, 0))
                break;
            const PairTile t = decode_pair_tile(aux, tile, n_tiles, band);
            int src[4] = {0, 0, 0, 0};
            if constexpr (GATHER) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = t.row0 + (int)rank * BM + 4 * lane + i;
                    src[i] = row_token[r < t.row_end ? r : t.row_end - 1];
                }
            }
            bool ok = true;
            for (int kb = 0; kb < num_kb; ++kb) {
                int w_ok = 1;
                if (lane == 0)
                    w_ok = tc::mbar_wait(tc::smem_u32(&aux->empty[stage]), phase ^ 1u, wait_ns,
                                         abort_flag, status);
                if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = tc::smem_u32(&aux->full[stage]);
                if (lane == 0 && leader)
                    tc::mbar_expect_tx(fb, 2 * STAGE_BYTES);
                __syncwarp();
                const uint32_t fb0 = map_rank(fb, 0);
                const uint32_t sa = smem_base + stage * STAGE_BYTES;
                if constexpr (GATHER)
                    tma_gather4_pair(&tmA, fb0, sa + lane * 4 * 128, kb * BK, src[0], src[1],
                                     src[2], src[3]);
                else if (lane == 0)
                    tma_load_2d_pair(&tmA, fb0, sa, kb * BK, t.row0 + (int)rank * BM);
                if (lane == 0)
                    tma_load_3d_pair(&tmB, fb0, sa + A_BYTES, kb * BK, t.n0 + (int)rank * BNH,
                                     t.e);
                ++fills;
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok)
                break;
        }
        if (lane == 0 && leader) {  // the leader's full barriers count both CTAs' bytes
            for (int s = 0; s < STAGES; ++s) {
                const int64_t n = fills / STAGES + (s < fills % STAGES ? 1 : 0);
                if (n > 0)
                    tc::mbar_drain(tc::smem_u32(&aux->full[s]), (uint32_t)((n - 1) & 1));
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---------------------------------------------------------- MMA issuer (leader)
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = cluster_id; tile < total && ok; tile += nclusters) {
                if (!tc::mbar_wait(tc::smem_u32(&aux->tempty[acc]), acc_phase ^ 1u, wait_ns,
                                   abort_flag, status)) {
                    ok = false;
                    break;
                }
                tc::tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!tc::mbar_wait(tc::smem_u32(&aux->full[stage]), phase, wait_ns,
                                       abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    const uint64_t da = tc::sdesc(sa), db = tc::sdesc(sa + A_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma_pair(d_tmem, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k),
                                  (kb | k) != 0);
                    umma_commit_both(tc::smem_u32(&aux->empty[stage]));
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                umma_commit_both(tc::smem_u32(&aux->tfull[acc]));
                if (++acc == ACC) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            umma_commit_own(tc::smem_u32(&aux->drain));
            tc::mbar_drain(tc::smem_u32(&aux->drain), 0);
        }
    } else {
        // -------------------------------------------------------------- epilogue (both)
        const int wq = warp & 3;
        const int lane_base = wq * 32;
        const int c_first = ((warp - 2) / 4) * (BN / 64);
        const uint32_t tempty0 = map_rank(tc::smem_u32(&aux->tempty[0]), 0);
        const uint32_t tempty1 = map_rank(tc::smem_u32(&aux->tempty[1]), 0);
        tc::EpiStore st{&tmO,
                        smem_base + TILE_BYTES + (uint32_t)((warp - 2) * 2 * tc::kStageSlotBytes),
                        0};
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = cluster_id; tile < total; tile += nclusters) {
            const PairTile t = decode_pair_tile(aux, tile, n_tiles, band);
            if (!tc::mbar_wait(tc::smem_u32(&aux->tfull[acc]), acc_phase, wait_ns, abort_flag,
                               status))
                break;
            tc::tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)lane_base << 16) + (uint32_t)(acc * BN);
            tc::epilogue_slab<EPI>(taddr, c_first, BN / 64, t.row0 + (int)rank * BM + lane_base,
                                   t.row_end, t.n0, out, ld_out, n_valid, st);
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(acc == 0 ? tempty0 : tempty1);
            if (++acc == ACC) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (lane == 0)
            tc::bulk_wait_all();  // this lane's output stores are done before the CTA exits
    }
    tc::tc_fence_before();
    cluster_sync();
    // after an abort, give copies still in flight time to land before either CTA of
    // the pair releases its shared memory (the other CTA's loads signal the leader)
    if (threadIdx.x == 0) {
        const int peer_abort =
            ld_cluster_s32(map_rank(tc::smem_u32(&aux->abort_flag), rank ^ 1u));
        if (*abort_flag || peer_abort) {
            const uint64_t t0 = globaltimer_ns();
            while (globaltimer_ns() - t0 < kAbortSettleNs) {
            }
        }
    }
    cluster_sync();
    if (warp == 1) {
        tc::tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(TMEM_COLS)
                     : "memory");
    }
}

}  // namespace tc2

// ------------------------------------------------------------------------ host side

struct DevInfo {
    int sms = 0;
    int pair_clusters = 0;
    bool attr[14] = {};
};
static std::mutex g_dev_mu;
static DevInfo g_dev[64];

template <typename Kern>
static cudaError_t set_smem_attr(Kern kern, int bytes, bool &done)
{
    if (done)
        return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        done = true;
    return e;
}

// SM count, dynamic shared memory opt-in of the GEMM kernels, and how many
// 2-CTA clusters of the pair kernel fit at once (per device, cached).
static cudaError_t prepare_device(DevInfo **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DevInfo &di = g_dev[dev];
    if (di.sms == 0) {
        e = cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess)
            return e;
    }
    if ((e = set_smem_attr(grouped_gemm_kernel<EPI_SWIGLU, false>, SMEM_BYTES, di.attr[0])) !=
            cudaSuccess ||
        (e = set_smem_attr(grouped_gemm_kernel<EPI_STORE, false>, SMEM_BYTES, di.attr[1])) !=
            cudaSuccess ||
        (e = set_smem_attr(grouped_gemm_kernel<EPI_SWIGLU, true>, SMEM_BYTES, di.attr[2])) !=
            cudaSuccess ||
        (e = set_smem_attr(grouped_gemm_kernel<EPI_STORE, true>, SMEM_BYTES, di.attr[3])) !=
            cudaSuccess ||
        (e = set_smem_attr(tc2::grouped_gemm_2sm_kernel<EPI_SWIGLU, false>, tc2::SMEM_BYTES,
                           di.attr[4])) != cudaSuccess ||
        (e = set_smem_attr(tc2::grouped_gemm_2sm_kernel<EPI_STORE, false>, tc2::SMEM_BYTES,
                           di.attr[5])) != cudaSuccess ||
        (e = set_smem_attr(tc2::grouped_gemm_2sm_kernel<EPI_SWIGLU, true>, tc2::SMEM_BYTES,
                           di.attr[6])) != cudaSuccess ||
        (e = set_smem_attr(tc2::grouped_gemm_2sm_kernel<EPI_STORE, true>, tc2::SMEM_BYTES,
                           di.attr[7])) != cudaSuccess ||
        (e = set_smem_attr(grouped_gemm_kernel<EPI_SWIGLU, false, kNarrowBN>,
                           Geo<kNarrowBN>::SMEM_BYTES, di.attr[8])) != cudaSuccess ||
        (e = set_smem_attr(grouped_gemm_kernel<EPI_STORE, false, kNarrowBN>,
                           Geo<kNarrowBN>::SMEM_BYTES, di.attr[9])) != cudaSuccess ||
        (e = set_smem_attr(grouped_gemm_kernel<EPI_SWIGLU, false, kNarrowBN, true>,
                           Geo<kNarrowBN, true>::SMEM_BYTES, di.attr[10])) != cudaSuccess ||
        (e = set_smem_attr(grouped_gemm_kernel<EPI_STORE, false, kNarrowBN, true>,
                           Geo<kNarrowBN, true>::SMEM_BYTES, di.attr[11])) != cudaSuccess ||
        (e = set_smem_attr(grouped_gemm_kernel<EPI_SWIGLU, false, BN, true>,
                           Geo<BN, true>::SMEM_BYTES, di.attr[12])) != cudaSuccess ||
        (e = set_smem_attr(grouped_gemm_kernel<EPI_STORE, false, BN, true>,
                           Geo<BN, true>::SMEM_BYTES, di.attr[13])) != cudaSuccess)
        return e;
    if (di.pair_clusters == 0) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * (di.sms / 2));
        cfg.blockDim = dim3(tc2::NUM_THREADS);
        cfg.dynamicSmemBytes = tc2::SMEM_BYTES;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, tc2::grouped_gemm_2sm_kernel<EPI_SWIGLU, false>,
                                           &cfg);
        if (e != cudaSuccess)
            return e;
        di.pair_clusters = n > 0 ? n : 1;
    }
    *out = &di;
    return cudaSuccess;
}

// Rows (T*k) from which the 2-SM kernel is used; below it the 1-SM kernel spreads
// the few tiles over more SMs.
constexpr int64_t kPairMinRows = 4096;

// Bytes of its first weight tile (KiB) that each CTA of a small-batch GEMM (at most one
// row tile per expert) brings into L2 before it waits for the routing kernels.
#ifndef MOE_L2_PREFETCH_KIB
#define MOE_L2_PREFETCH_KIB 400
#endif
constexpr int kL2PrefetchKiB = MOE_L2_PREFETCH_KIB;

// One grouped GEMM launch.  A: [a_rows][a_ld] activations (K extent a_k), read in
// expert-grouped row order, or -- when row_token is given -- gathered: tile row r is
// row row_token[r] of A; B: [E][b_rows][b_ld] expert weights (K extent b_k, N =
// b_rows); out: [rows][ld_out], first n_valid columns written; rows = T*k, k_rows = k
// (an expert has at most rows / k_rows rows).
template <int EPI>
static cudaError_t launch_gemm(const void *A, uint64_t a_k, uint64_t a_ld, uint64_t a_rows,
                               const int32_t *row_token, uint64_t rows, int k_rows, const void *B,
                               uint64_t b_k, uint64_t b_ld, uint64_t b_rows,
                               const int32_t *offsets, int E, bf16 *out, int ld_out, int n_valid,
                               int32_t *status, cudaStream_t s)
{
    DevInfo *di = nullptr;
    cudaError_t e = prepare_device(&di);
    if (e != cudaSuccess)
        return e;
    const bool pair = (int64_t)rows >= kPairMinRows;
    const bool gather = row_token != nullptr;
    CUtensorMap ta, tb;
    const uint64_t da[2] = {a_k, a_rows}, sa[1] = {a_ld * 2};
    const uint64_t db[3] = {b_k, b_rows, (uint64_t)E};
    const uint64_t sb[2] = {b_ld * 2, b_rows * b_ld * 2};
    // 1-SM tiles 160 wide instead of 256 when every expert has at most 128 rows (T <=
    // 128, one row tile each) and the narrower tiles still fit one wave of the SMs
    const int64_t T = (int64_t)rows / (k_rows > 0 ? k_rows : 1);
    const int64_t n_wide = (int64_t)E * (((int64_t)b_rows + BN - 1) / BN);
    const int64_t n_narrow = (int64_t)E * (((int64_t)b_rows + kNarrowBN - 1) / kNarrowBN);
    const bool narrow = !pair && !gather && T <= BM && n_wide < di->sms && n_narrow <= di->sms;
    // A boxes: one row high for gather4, 64 rows for the 1-SM kernel, BM for the pair
    const uint32_t ba[2] = {BK, gather ? 1u : (pair ? (uint32_t)BM : (uint32_t)kABoxRows)};
    const uint32_t bb[3] = {BK, pair ? (uint32_t)tc2::BNH : (uint32_t)(narrow ? kNarrowBN : BN),
                            1};
    if ((e = make_map(&ta, A, 2, da, sa, ba)) != cudaSuccess)
        return e;
    if ((e = make_map(&tb, B, 3, db, sb, bb)) != cudaSuccess)
        return e;
    // output boxes of 32 columns x 32 rows written by bulk tensor stores
    CUtensorMap to;
    const uint64_t dout[2] = {(uint64_t)n_valid, rows}, sout[1] = {(uint64_t)ld_out * 2};
    const uint32_t bout[2] = {32, 32};
    if ((e = make_map(&to, out, 2, dout, sout, bout, CU_TENSOR_MAP_SWIZZLE_64B)) != cudaSuccess)
        return e;
    const uint64_t wait_ns = wait_limit_ns();
    const int N = (int)b_rows, K = (int)a_k;
    // L2 prefetch depth of the first weight tile (K blocks), for one row tile per expert
    const int bnt = narrow ? kNarrowBN : BN;
    const int pf_kb = !pair && !gather && T <= BM
                          ? (int)((int64_t)kL2PrefetchKiB * 1024 / ((int64_t)bnt * BK * 2))
                          : 0;
    // at most 64 tokens: no expert has more than 64 rows (a token adds at most one row
    // per expert), so the small-batch stages apply
    const bool small = !pair && !gather && T <= kABoxRows;
    if (narrow && small) {
        launch_pdl(grouped_gemm_kernel<EPI, false, kNarrowBN, true>, dim3(di->sms),
                   dim3(NUM_THREADS), Geo<kNarrowBN, true>::SMEM_BYTES, s, ta, tb, to, offsets, E,
                   N, K, out, ld_out, n_valid, status, wait_ns, row_token, pf_kb);
        return cudaGetLastError();
    }
    if (small) {
        launch_pdl(grouped_gemm_kernel<EPI, false, BN, true>, dim3(di->sms), dim3(NUM_THREADS),
                   Geo<BN, true>::SMEM_BYTES, s, ta, tb, to, offsets, E, N, K, out, ld_out,
                   n_valid, status, wait_ns, row_token, pf_kb);
        return cudaGetLastError();
    }
    if (narrow) {
        launch_pdl(grouped_gemm_kernel<EPI, false, kNarrowBN>, dim3(di->sms), dim3(NUM_THREADS),
                   Geo<kNarrowBN>::SMEM_BYTES, s, ta, tb, to, offsets, E, N, K, out, ld_out,
                   n_valid, status, wait_ns, row_token, pf_kb);
        return cudaGetLastError();
    }
    if (!pair) {
        if (gather)
            launch_pdl(grouped_gemm_kernel<EPI, true>, dim3(di->sms), dim3(NUM_THREADS), SMEM_BYTES, s, 
                ta, tb, to, offsets, E, N, K, out, ld_out, n_valid, status, wait_ns, row_token, 0);
        else
            launch_pdl(grouped_gemm_kernel<EPI, false>, dim3(di->sms), dim3(NUM_THREADS), SMEM_BYTES, s, 
                ta, tb, to, offsets, E, N, K, out, ld_out, n_valid, status, wait_ns, row_token,
                pf_kb);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(2 * di->pair_clusters);
    cfg.blockDim = dim3(tc2::NUM_THREADS);
    cfg.dynamicSmemBytes = tc2::SMEM_BYTES;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    // band of A rows that concurrent clusters sweep N over, in pair m-tiles (0: the
    // whole expert)
    const int band_rows = gemm_band_rows();
    const int band = band_rows <= 0 ? 0 : (band_rows + 2 * BM - 1) / (2 * BM);
    if (gather)
        return cudaLaunchKernelEx(&cfg, tc2::grouped_gemm_2sm_kernel<EPI, true>, ta, tb, to,
                                  offsets, E, N, K, out, ld_out, n_valid, status, wait_ns,
                                  row_token, band);
    return cudaLaunchKernelEx(&cfg, tc2::grouped_gemm_2sm_kernel<EPI, false>, ta, tb, to, offsets,
                              E, N, K, out, ld_out, n_valid, status, wait_ns, row_token, band);
}

}  // namespace tc

using namespace tc;

cudaError_t launch_up_tc(const moe_params_t *p, const void *x_perm, const int32_t *offsets,
                         const void *W13, void *h, int32_t *status, cudaStream_t s)
{
    const uint64_t d = p->d, m = p->m, m16 = round_up(p->m, 16), m8 = round_up(p->m, 8);
    const uint64_t rows = (uint64_t)p->T * p->k;
    cudaError_t e = launch_gemm<EPI_SWIGLU>(x_perm, d, d, rows, nullptr, rows, p->k, W13, d, d, 2 * m16,
                                            offsets, p->E, (bf16 *)h, (int)m8, (int)m, status, s);
    count_launch();
    return e;
}

cudaError_t launch_up_tc_gather(const moe_params_t *p, const void *x, const int32_t *row_token,
                                const int32_t *offsets, const void *W13, void *h,
                                int32_t *status, cudaStream_t s)
{
    const uint64_t d = p->d, m = p->m, m16 = round_up(p->m, 16), m8 = round_up(p->m, 8);
    const uint64_t rows = (uint64_t)p->T * p->k;
    cudaError_t e = launch_gemm<EPI_SWIGLU>(x, d, d, (uint64_t)p->T, row_token, rows, p->k, W13, d, d,
                                            2 * m16, offsets, p->E, (bf16 *)h, (int)m8, (int)m,
                                            status, s);
    count_launch();
    return e;
}

cudaError_t launch_down_tc(const moe_params_t *p, const void *h, const int32_t *offsets,
                           const void *W2, void *out, int32_t *status, cudaStream_t s)
{
    const uint64_t d = p->d, m = p->m, m8 = round_up(p->m, 8);
    const uint64_t rows = (uint64_t)p->T * p->k;
    cudaError_t e = launch_gemm<EPI_STORE>(h, m, m8, rows, nullptr, rows, p->k, W2, m, m8, d, offsets,
                                           p->E, (bf16 *)out, (int)d, (int)d, status, s);
    count_launch();
    return e;
}

}  // namespace moe
