// common.cuh -- helpers shared by the kernels of libmoe.so (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libmoe targets sm_100a (B200) only"
#endif

namespace moe {

typedef __nv_bfloat16 bf16;

// ---------------------------------------------------------------- workspace
// The first 256 bytes of the caller's workspace are a header; word 0 is the
// device status word (0 or a MOE_ERR_DEVICE_* code; the first error sticks).
constexpr size_t kWsHeader = 256;
// Word 1 of the header: ticket counter of the dispatch count kernel (zero between calls).
constexpr int kWsCounterWord = 1;
// Word 2: ticket counter of the tensor-core router (zero between calls).
constexpr int kWsRouterCounterWord = 2;
// Words 4-5: grid barrier of the decode forward kernel (arrival count, zero between
// calls; generation, counting up).
constexpr int kWsDecodeBarrierWord = 4;
// Words 6-7: grid barriers of the small-batch front kernel (arrivals over both
// barriers; CTAs past both; zero between calls).
constexpr int kWsFrontBarrierWord = 6;
// Header bytes that clearing the status resets (status word and counters).
constexpr size_t kWsResetBytes = 32;
// Words 8-9: offsets {0, T} of the shared block's one-expert GEMMs (residual MoE).
constexpr int kWsTokenRangeWord = 8;

// Programmatic dependent launch.  Every kernel of the library is launched with
// programmatic stream serialization allowed (launch_pdl): it may be scheduled
// while the previous kernel on the stream is still running, so it calls
// pdl_wait() before it touches global memory (the wait returns once the
// previous grid has completed and its writes are visible), and pdl_trigger() to
// let the next kernel be scheduled early in turn.  A kernel that triggers before
// its own wait lets the next one start while the previous grid still runs; that
// one still sees every earlier grid complete at its wait, since this grid cannot
// complete before its own wait has returned.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void set_status(int32_t *status, int32_t code)
{
    if (status != nullptr)
        atomicCAS(status, 0, code);
}

__device__ __forceinline__ int32_t ld_acquire_gpu(const int32_t *p)
{
    int32_t v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- element I/O
template <typename T> struct Vec;  // 16-byte vector of T
template <> struct Vec<float> {
    static constexpr int N = 4;
};
template <> struct Vec<bf16> {
    static constexpr int N = 8;
};

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

// 16-byte global loads.  nc: read-only path, no L1 allocation (streamed once).
// Not volatile: a pure load the compiler may hoist and batch, so unrolled loops
// keep several loads in flight.
__device__ __forceinline__ uint4 ld_nc_na(const void *p)
{
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}
__device__ __forceinline__ uint4 ld_nc(const void *p)
{
    return __ldg(reinterpret_cast<const uint4 *>(p));
}
__device__ __forceinline__ void st_v4(void *p, uint4 v)
{
    *reinterpret_cast<uint4 *>(p) = v;
}

// unpack 8 bf16 held in a uint4 to f32 / pack back
__device__ __forceinline__ void bf16x8_to_f32(uint4 v, float *f)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint4 f32x8_to_bf16(const float *f)
{
    uint4 v;
    v.x = pack_bf16x2(f[0], f[1]);
    v.y = pack_bf16x2(f[2], f[3]);
    v.z = pack_bf16x2(f[4], f[5]);
    v.w = pack_bf16x2(f[6], f[7]);
    return v;
}

// D += A * B on the tensor cores, m16n8k16, bf16 inputs, f32 accumulators
// (A row-major 16x16 in a0..a3, B column-major 16x8 in b0..b1).
// B fragment of mma m16n8k16 from a row-major [k][8] bf16 tile: lanes 0..15 give the
// addresses of rows 0..15 (16-byte aligned)
__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t &b0, uint32_t &b1)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
                 : "=r"(b0), "=r"(b1)
                 : "r"(addr));
}

// A fragment of mma m16n8k16 from a row-major [16][16] bf16 tile: lane l gives the
// address of row l % 16 at column 8 * (l / 16) (16-byte aligned)
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &a0, uint32_t &a1, uint32_t &a2,
                                        uint32_t &a3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float *c, uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

}  // namespace moe
