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
// Warp roles (192 threads, one CTA per SM, grid = #SMs):
//   warp 0     TMA producer (one lane)
//   warp 1     TMEM allocator and MMA issuer (one lane)
//   warps 2-5  epilogue: tcgen05.ld -> registers -> bf16 -> global; warp w reads
//              TMEM lanes 32*(w%4)..+31, i.e. tile rows, one row per thread.
// For a3 the packed W13 layout puts, in each 32-row group, 16 W1 rows and then the
// 16 W3 rows of the same 16 neurons, so each 32-column TMEM load holds the gate
// and up values of 16 neurons of the thread's row.
//
// Every mbarrier wait is bounded (%globaltimer): past the limit the kernel records
// MOE_ERR_DEVICE_TIMEOUT, every role stops, in-flight TMA copies and MMAs are
// drained (bounded again) and TMEM is freed before the CTA exits.  No TMA load here
// uses cluster multicast.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace tc {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;  // 64 bf16 = 128 bytes: one swizzle-128B row
constexpr int STAGES = 4;
constexpr int ACC = 2;
constexpr int TMEM_COLS = ACC * BN;  // 512
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TILE_BYTES = STAGES * STAGE_BYTES;
constexpr int NUM_THREADS = 192;
constexpr uint64_t kDrainNs = 1000000000ull;  // bound of the drain waits on exit

enum { EPI_SWIGLU = 0, EPI_STORE = 1 };

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
constexpr int SMEM_BYTES = 1024 + TILE_BYTES + (int)sizeof(Aux);

// kind::f16 instruction descriptor: D f32, A and B bf16, both K-major, N = BN, M = BM.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

// Shared-memory matrix descriptor of a K-major, 128B-swizzled tile whose rows are
// 128 bytes apart (8-row core groups 1024 bytes apart); tile base 1024-aligned.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address, 16-byte units
    d |= (uint64_t)1 << 16;                    // leading byte offset (unused for this layout)
    d |= (uint64_t)(1024 >> 4) << 32;          // stride byte offset: next 8-row group
    d |= (uint64_t)1 << 46;                    // descriptor version
    d |= (uint64_t)2 << 61;                    // 128-byte swizzle
    return d;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait; gives up when the limit passes or another role aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                          volatile int32_t *abort_flag, int32_t *status)
{
    if (mbar_try(bar, parity))
        return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try(bar, parity))
            return true;
        if (*abort_flag)
            return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            set_status(status, MOE_ERR_DEVICE_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
}

// Bounded wait used while draining on exit (ignores the abort flag).
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try(bar, parity))
        if (globaltimer_ns() - t0 > kDrainNs)
            return;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void tma_load_2d(const CUtensorMap *map, uint32_t bar, uint32_t dst,
                                            int c0, int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(const CUtensorMap *map, uint32_t bar, uint32_t dst,
                                            int c0, int c1, int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(kIdesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
          "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
          "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
          "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

struct Tile {
    int e, row0, row_end, n0;
};

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
    t.n0 = nt * BN;
    return t;
}

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const int32_t *__restrict__ offsets, int E, int N, int K,
                        bf16 *__restrict__ out, int ld_out, int n_valid, int32_t *status,
                        uint64_t wait_ns)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Aux *aux = reinterpret_cast<Aux *>(smem + TILE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int32_t *abort_flag = &aux->abort_flag;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&aux->full[s]), 1);
            mbar_init(smem_u32(&aux->empty[s]), 1);
        }
        for (int a = 0; a < ACC; ++a) {
            mbar_init(smem_u32(&aux->tfull[a]), 1);
            mbar_init(smem_u32(&aux->tempty[a]), 4);
        }
        mbar_init(smem_u32(&aux->drain), 1);
        aux->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
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
                acc += (rows + BM - 1) / BM * n_tiles;
            }
            aux->tstart[E] = acc;
        }
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
            for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
                const Tile t = decode_tile(aux, tile, n_tiles);
                bool ok = true;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(smem_u32(&aux->empty[stage]), phase ^ 1u, wait_ns, abort_flag,
                                   status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&aux->full[stage]);
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    mbar_expect_tx(fb, STAGE_BYTES);
                    tma_load_2d(&tmA, fb, sa, kb * BK, t.row0);
                    tma_load_3d(&tmB, fb, sa + A_BYTES, kb * BK, t.n0, t.e);
                    ++fills;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
            }
            // drain: the last fill of every stage has landed before the CTA may exit
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
                    const uint32_t sa = smem_base + stage * STAGE_BYTES;
                    const uint64_t da = sdesc(sa), db = sdesc(sa + A_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)  // +32 bytes (16 bf16) per step
                        umma_bf16(d_tmem, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k),
                                  (kb | k) != 0);
                    umma_commit(smem_u32(&aux->empty[stage]));
                    if (++stage == STAGES) {
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
        const int wq = warp & 3;
        const int lane_base = wq * 32;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const Tile t = decode_tile(aux, tile, n_tiles);
            if (!mbar_wait(smem_u32(&aux->tfull[acc]), acc_phase, wait_ns, abort_flag, status))
                break;
            tc_fence_after();
            const int row = t.row0 + lane_base + lane;
            const bool rv = row < t.row_end;
            const uint32_t taddr = tmem_base + ((uint32_t)lane_base << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(taddr + (uint32_t)(c * 32), v);
                if constexpr (EPI == EPI_SWIGLU) {
                    const int nb = t.n0 / 2 + c * 16;  // first neuron of this 32-column group
                    float hv[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float g = __uint_as_float(v[i]);
                        const float u = __uint_as_float(v[16 + i]);
                        hv[i] = g / (1.0f + __expf(-g)) * u;
                    }
                    if (rv && nb < n_valid) {
                        bf16 *dst = out + (int64_t)row * ld_out + nb;
                        if (nb + 16 <= n_valid) {
                            st_v4(dst, f32x8_to_bf16(hv));
                            st_v4(dst + 8, f32x8_to_bf16(hv + 8));
                        } else {
                            for (int i = 0; i < 16 && nb + i < n_valid; ++i)
                                dst[i] = __float2bfloat16_rn(hv[i]);
                        }
                    }
                } else {
                    const int col = t.n0 + c * 32;
                    if (rv) {
                        bf16 *dst = out + (int64_t)row * ld_out + col;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            if (col + q * 8 < n_valid) {  // n_valid is a multiple of 8
                                float f[8];
#pragma unroll
                                for (int i = 0; i < 8; ++i)
                                    f[i] = __uint_as_float(v[q * 8 + i]);
                                st_v4(dst + q * 8, f32x8_to_bf16(f));
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&aux->tempty[acc]));
            if (++acc == ACC) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
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

// ------------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encoder(cudaError_t *err)
{
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    static cudaError_t e0 = cudaSuccess;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        e0 = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                              cudaEnableDefault, &q);
        if (e0 == cudaSuccess && q != cudaDriverEntryPointSuccess)
            e0 = cudaErrorSymbolNotFound;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    *err = e0;
    return fn;
}

// rank-2 or rank-3 bf16 tensor map; dims/strides innermost first, strides in bytes.
static cudaError_t make_map(CUtensorMap *map, const void *base, int rank, const uint64_t *dims,
                            const uint64_t *strides, const uint32_t *box)
{
    cudaError_t err;
    EncodeTiledFn enc = get_encoder(&err);
    if (enc == nullptr)
        return err != cudaSuccess ? err : cudaErrorSymbolNotFound;
    cuuint64_t gd[3], gs[2];
    cuuint32_t bx[3], es[3] = {1, 1, 1};
    for (int i = 0; i < rank; ++i) {
        gd[i] = dims[i];
        bx[i] = box[i];
    }
    for (int i = 0; i < rank - 1; ++i)
        gs[i] = strides[i];
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank,
                     const_cast<void *>(base), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

struct DevInfo {
    int sms = 0;
    bool attr[2] = {false, false};
};
static std::mutex g_dev_mu;
static DevInfo g_dev[64];

static cudaError_t prepare_device(int which, int *sms)
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
    if (!di.attr[which]) {
        e = which == EPI_SWIGLU
                ? cudaFuncSetAttribute(grouped_gemm_kernel<EPI_SWIGLU>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)
                : cudaFuncSetAttribute(grouped_gemm_kernel<EPI_STORE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess)
            return e;
        di.attr[which] = true;
    }
    *sms = di.sms;
    return cudaSuccess;
}

}  // namespace tc

using namespace tc;

cudaError_t launch_up_tc(const moe_params_t *p, const void *x_perm, const int32_t *offsets,
                         const void *W13, void *h, int32_t *status, cudaStream_t s)
{
    const int d = p->d, m = p->m, m16 = round_up(m, 16), m8 = round_up(m, 8);
    const uint64_t rows = (uint64_t)p->T * p->k;
    CUtensorMap ta, tb;
    const uint64_t da[2] = {(uint64_t)d, rows}, sa[1] = {(uint64_t)d * 2};
    const uint32_t ba[2] = {BK, BM};
    const uint64_t db[3] = {(uint64_t)d, (uint64_t)2 * m16, (uint64_t)p->E};
    const uint64_t sb[2] = {(uint64_t)d * 2, (uint64_t)2 * m16 * d * 2};
    const uint32_t bb[3] = {BK, BN, 1};
    cudaError_t e;
    if ((e = make_map(&ta, x_perm, 2, da, sa, ba)) != cudaSuccess)
        return e;
    if ((e = make_map(&tb, W13, 3, db, sb, bb)) != cudaSuccess)
        return e;
    int sms = 0;
    if ((e = prepare_device(EPI_SWIGLU, &sms)) != cudaSuccess)
        return e;
    grouped_gemm_kernel<EPI_SWIGLU><<<sms, NUM_THREADS, SMEM_BYTES, s>>>(
        ta, tb, offsets, p->E, 2 * m16, d, (bf16 *)h, m8, m, status, wait_limit_ns());
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_down_tc(const moe_params_t *p, const void *h, const int32_t *offsets,
                           const void *W2, void *out, int32_t *status, cudaStream_t s)
{
    const int d = p->d, m = p->m, m8 = round_up(m, 8);
    const uint64_t rows = (uint64_t)p->T * p->k;
    CUtensorMap ta, tb;
    const uint64_t da[2] = {(uint64_t)m, rows}, sa[1] = {(uint64_t)m8 * 2};
    const uint32_t ba[2] = {BK, BM};
    const uint64_t db[3] = {(uint64_t)m, (uint64_t)d, (uint64_t)p->E};
    const uint64_t sb[2] = {(uint64_t)m8 * 2, (uint64_t)d * m8 * 2};
    const uint32_t bb[3] = {BK, BN, 1};
    cudaError_t e;
    if ((e = make_map(&ta, h, 2, da, sa, ba)) != cudaSuccess)
        return e;
    if ((e = make_map(&tb, W2, 3, db, sb, bb)) != cudaSuccess)
        return e;
    int sms = 0;
    if ((e = prepare_device(EPI_STORE, &sms)) != cudaSuccess)
        return e;
    grouped_gemm_kernel<EPI_STORE><<<sms, NUM_THREADS, SMEM_BYTES, s>>>(
        ta, tb, offsets, p->E, d, m, (bf16 *)out, d, d, status, wait_limit_ns());
    count_launch();
    return cudaGetLastError();
}

}  // namespace moe
