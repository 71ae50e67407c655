// router_tc.cu -- a1 for bf16 batches above decode size on the tcgen05 tensor cores
// ("Llama 3 Meets MoE: Efficient Upcycling", section 3 "核心公式": H_i = (x W_g)_i +
// StandardNormal() * Softplus((x W_noise)_i), G = Softmax(KeepTopK(H, k)); section 5:
// the ST router takes KeepTopK of the full softmax instead).
//
// The logits x.[W_g | W_noise] are a T x d x NOUT product (NOUT = E or 2E padded to
// 16..128) that must run at HBM speed.  A persistent kernel streams 128-token tiles
// of x through a TMA ring (box 64 K x 128 tokens, 128-byte swizzle) together with
// the router weights packed K-major (box 64 K x NOUT; packed once per weight set by
// router_pack_tc_kernel), and tcgen05.mma (M = 128, N = NOUT) accumulates the logits
// in TMEM (two buffers, so one tile's gate overlaps the next tile's loads).  The
// epilogue gives each thread one token row: it reads the NOUT logits from TMEM and
// runs the gate in f32: noise, KeepTopK (ties to the lower expert index), Mixtral or
// ST weights, and the token's contributions to the per-expert sums of softmax(H) and
// of G, which are reduced over the CTA in a fixed order (warp butterflies, then the
// four warps in order) and written as one partial per CTA.  Each gate warp also
// counts, per expert, the tokens of its 32-token chunk routed there (the count step
// of a2's counting sort).  The CTA that finishes last adds the CTA partials in CTA
// order (f64) and scans the chunk counts into rank bases and routed counts, so a
// dispatch that follows needs no count pass of its own.
//
// Warps: 0 TMA producer (one lane), 1 TMEM allocator and MMA issuer (one lane),
// 2-5 gate (warp w reads TMEM lanes 32*(w%4)..+31 = tokens of the tile).
// Packed router weight rows: noisy -> row 2e = W_g[:, e], row 2e+1 = W_noise[:, e];
// otherwise row e = W_g[:, e]; the other rows are zero.
#include <math.h>

#include "dispatch_scan.cuh"
#include "tc_common.cuh"

namespace moe {
namespace rtc {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int MAX_STAGES = 12;
constexpr int NUM_THREADS = 192;

// The ring is as deep as shared memory allows (the kernel streams x once, so bytes
// in flight per SM set its speed): 11 stages of 18 KB for 16 outputs, 6 of 32 KB
// for 128.
template <int NOUT> struct Cfg {
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = NOUT * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = (200 * 1024 / STAGE_BYTES) < MAX_STAGES ? (200 * 1024 / STAGE_BYTES)
                                                                          : MAX_STAGES;
    static constexpr int TILE_BYTES = STAGES * STAGE_BYTES;
    static constexpr int TMEM_COLS = 2 * NOUT < 32 ? 32 : 2 * NOUT;
    // kind::f16, D f32, A/B bf16 K-major, N = NOUT, M = 128
    static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) |
                                      ((uint32_t)(NOUT >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
    static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment");
};

struct Aux {
    uint64_t full[MAX_STAGES];
    uint64_t empty[MAX_STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int32_t abort_flag;
    float red[4][2 * MOE_MAX_EXPERTS];  // per-warp sums of one tile
    float acc[2 * MOE_MAX_EXPERTS];     // this CTA's running sums
    int32_t last;                       // this CTA finished last
};

__device__ __forceinline__ void tmem_ld16_async(uint32_t taddr, uint32_t (&v)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}

__device__ __forceinline__ float softplus_f(float z) { return fmaxf(z, 0.f) + log1pf(expf(-fabsf(z))); }

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int s = 16; s > 0; s >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, s);
    return v;
}

// named barrier over the 4 gate warps (128 threads)
__device__ __forceinline__ void gate_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
struct GateBar {
    __device__ void operator()() const { gate_bar(); }
};

// the same barrier, returning whether v held on every gate thread: the gate warps
// leave their tile loop together, so their barrier counts never diverge
__device__ __forceinline__ bool gate_all(bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, 1, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

template <int NOUT, bool NOISY>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                     const __grid_constant__ CUtensorMap tmW, int T, int d, int E, int k,
                     const float *__restrict__ noise, const float *__restrict__ bias,
                     int router_type, int32_t *__restrict__ idx_out, float *__restrict__ w_out,
                     float *__restrict__ part, int32_t *counter, float *__restrict__ probs_sum,
                     float *__restrict__ importance, int32_t *__restrict__ hist,
                     int32_t *__restrict__ dcounts, int32_t *status, uint64_t wait_ns)
{
    using C = Cfg<NOUT>;
    constexpr int STAGES = C::STAGES;
    constexpr int EMAX = NOISY ? NOUT / 2 : NOUT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Aux *aux = reinterpret_cast<Aux *>(smem + C::TILE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int32_t *abort_flag = &aux->abort_flag;
    const int n_tiles = (T + BM - 1) / BM;
    const int num_kb = (d + BK - 1) / BK;
    const int nch = (T + kDispatchChunk - 1) / kDispatchChunk;
    // CTA b sweeps K starting at block kstart and wraps around: the CTAs' concurrent
    // TMA reads (128 rows of 128 bytes, 8 KB apart in x) then differ in their low
    // address bits instead of all landing on the same few DRAM channels
    const int kstart = (int)((int64_t)blockIdx.x * num_kb / gridDim.x);

    // set-up that touches no global memory overlaps the previous kernel's tail
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(tc::smem_u32(&aux->full[s]), 1);
            tc::mbar_init(tc::smem_u32(&aux->empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            tc::mbar_init(tc::smem_u32(&aux->tfull[a]), 1);
            tc::mbar_init(tc::smem_u32(&aux->tempty[a]), 4);
        }
        tc::mbar_init(tc::smem_u32(&aux->drain), 1);
        aux->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW)) : "memory");
    }
    for (int i = threadIdx.x; i < 2 * MOE_MAX_EXPERTS; i += blockDim.x)
        aux->acc[i] = 0.f;
    pdl_wait();
    pdl_trigger();
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         tc::smem_u32(&aux->tmem_base)),
                     "r"(C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_base = aux->tmem_base;
    const uint32_t smem_base = tc::smem_u32(smem);

    if (warp == 0) {
        if (lane == 0) {
            // -------------------------------------------------------------- TMA producer (A)
            int stage = 0;
            uint32_t phase = 0;
            int64_t fills = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
                for (int i = 0; i < num_kb; ++i) {
                    const int kb = kstart + i < num_kb ? kstart + i : kstart + i - num_kb;
                    if (!tc::mbar_wait(tc::smem_u32(&aux->empty[stage]), phase ^ 1u, wait_ns,
                                       abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = tc::smem_u32(&aux->full[stage]);
                    const uint32_t sa = smem_base + stage * C::STAGE_BYTES;
                    tc::mbar_expect_tx(fb, C::STAGE_BYTES);
                    tc::tma_load_2d(&tmX, fb, sa, kb * BK, tile * BM);
                    tc::tma_load_2d(&tmW, fb, sa + C::A_BYTES, kb * BK, 0);
                    ++fills;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // every issued copy has landed before the CTA can exit (bounded)
            for (int s = 0; s < STAGES; ++s) {
                const int64_t n = fills / STAGES + (s < fills % STAGES ? 1 : 0);
                if (n > 0)
                    tc::mbar_drain(tc::smem_u32(&aux->full[s]), (uint32_t)((n - 1) & 1));
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // -------------------------------------------------------------- MMA issuer
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
                if (!tc::mbar_wait(tc::smem_u32(&aux->tempty[acc]), acc_phase ^ 1u, wait_ns,
                                   abort_flag, status))
                    break;
                tc::tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * NOUT);
                for (int i = 0; i < num_kb; ++i) {  // the producer's K order
                    if (!tc::mbar_wait(tc::smem_u32(&aux->full[stage]), phase, wait_ns,
                                       abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint32_t sa = smem_base + stage * C::STAGE_BYTES;
                    const uint64_t da = tc::sdesc(sa), db = tc::sdesc(sa + C::A_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        tc::umma_f16(d_tmem, da + (uint64_t)(2 * kk), db + (uint64_t)(2 * kk),
                                     C::IDESC, (i | kk) != 0);
                    tc::umma_commit(tc::smem_u32(&aux->empty[stage]));
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                tc::umma_commit(tc::smem_u32(&aux->tfull[acc]));
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            tc::umma_commit(tc::smem_u32(&aux->drain));
            tc::mbar_drain(tc::smem_u32(&aux->drain), 0);
        }
    } else {
        // ------------------------------------------------------------------ gate
        const int wq = warp & 3;
        const int lane_base = wq * 32;
        const int gt = threadIdx.x - 64;  // 0..127 over the gate warps
        float bias_r[EMAX];
#pragma unroll
        for (int e = 0; e < EMAX; ++e)
            bias_r[e] = (bias != nullptr && e < E) ? bias[e] : 0.f;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
            const int64_t t = (int64_t)tile * BM + lane_base + lane;
            const bool tv = t < T;
            // the token's noise draws are loaded before the logits are ready
            float nz[EMAX];
#pragma unroll
            for (int e = 0; e < EMAX; ++e)
                nz[e] = (NOISY && tv && e < E) ? __ldg(noise + t * E + e) : 0.f;
            const bool got = tc::mbar_wait(tc::smem_u32(&aux->tfull[acc]), acc_phase, wait_ns,
                                           abort_flag, status);
            if (!gate_all(got))
                break;
            tc::tc_fence_after();
            const uint32_t taddr =
                tmem_base + ((uint32_t)lane_base << 16) + (uint32_t)(acc * NOUT);
            float lg[NOUT];
#pragma unroll
            for (int c = 0; c < NOUT / 16; ++c) {
                uint32_t v[16];
                tmem_ld16_async(taddr + (uint32_t)(16 * c), v);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    lg[16 * c + i] = __uint_as_float(v[i]);
            }
            // the accumulator is in registers: release it to the MMA warp
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0)
                tc::mbar_arrive(tc::smem_u32(&aux->tempty[acc]));
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }

            float H[EMAX];
            bool bad = false;
#pragma unroll
            for (int e = 0; e < EMAX; ++e) {
                float h = -INFINITY;
                if (e < E) {
                    h = NOISY ? lg[2 * e] : lg[e];
                    if (bias)
                        h += bias_r[e];
                    if (NOISY && tv)
                        h += nz[e] * softplus_f(lg[2 * e + 1]);
                    bad |= !isfinite(h);
                }
                H[e] = h;
            }
            bad = bad && tv;
            // KeepTopK: j-th pick = largest remaining H, ties to the lower index
            int sel[MOE_MAX_TOPK];
            float selv[MOE_MAX_TOPK];
            uint64_t taken = 0;
#pragma unroll
            for (int j = 0; j < MOE_MAX_TOPK; ++j) {
                sel[j] = -1;
                selv[j] = -INFINITY;
                if (j < k) {
                    int bi = -1;
                    float best = -INFINITY;
#pragma unroll
                    for (int e = 0; e < EMAX; ++e) {
                        if (e < E && !((taken >> e) & 1ull) && (bi < 0 || H[e] > best)) {
                            best = H[e];
                            bi = e;
                        }
                    }
                    sel[j] = bi;
                    selv[j] = best;
                    taken |= 1ull << (bi & 63);
                }
            }
            const float hmax = selv[0];
            float z = 0.f;
#pragma unroll
            for (int e = 0; e < EMAX; ++e)
                if (e < E)
                    z += expf(H[e] - hmax);
            const float invz = 1.f / z;
            float wsel[MOE_MAX_TOPK];
            if (router_type == MOE_ROUTER_MIXTRAL) {
                float zs = 0.f;
#pragma unroll
                for (int j = 0; j < MOE_MAX_TOPK; ++j)
                    if (j < k)
                        zs += expf(selv[j] - hmax);
                const float is = 1.f / zs;
#pragma unroll
                for (int j = 0; j < MOE_MAX_TOPK; ++j)
                    wsel[j] = j < k ? expf(selv[j] - hmax) * is : 0.f;
            } else {
#pragma unroll
                for (int j = 0; j < MOE_MAX_TOPK; ++j)
                    wsel[j] = j < k ? expf(selv[j] - hmax) * invz : 0.f;
            }
            if (tv) {
                if (bad)
                    set_status(status, MOE_ERR_DEVICE_BADINDEX);
#pragma unroll
                for (int j = 0; j < MOE_MAX_TOPK; ++j)
                    if (j < k) {
                        idx_out[t * k + j] = bad ? -1 : sel[j];
                        w_out[t * k + j] = bad ? 0.f : wsel[j];
                    }
            }
            const bool contrib = tv && !bad;
            // a2's chunk histogram: this warp's 32 tokens are chunk tile*4 + wq
            const int chunk = tile * (BM / kDispatchChunk) + wq;
#pragma unroll
            for (int e = 0; e < EMAX; ++e) {
                if (e < E) {  // E is uniform: every lane takes part in the ballot
                    bool has = false;
#pragma unroll
                    for (int j = 0; j < MOE_MAX_TOPK; ++j)
                        has |= contrib && j < k && sel[j] == e;
                    const unsigned b = __ballot_sync(0xffffffffu, has);
                    if (lane == (e & 31) && chunk < nch)
                        hist[(int64_t)e * nch + chunk] = __popc(b);
                }
            }
            // per-expert sums over the tile's tokens: softmax(H) and gate weights
            gate_bar();  // red[][] of the previous tile has been consumed
#pragma unroll
            for (int e = 0; e < EMAX; ++e) {
                if (e < E) {
                    float p = contrib ? expf(H[e] - hmax) * invz : 0.f;
                    float g = 0.f;
#pragma unroll
                    for (int j = 0; j < MOE_MAX_TOPK; ++j)
                        g += (contrib && j < k && sel[j] == e) ? wsel[j] : 0.f;
                    p = warp_sum(p);
                    g = warp_sum(g);
                    if (lane == 0) {
                        aux->red[wq][e] = p;
                        aux->red[wq][E + e] = g;
                    }
                }
            }
            gate_bar();
            for (int i = gt; i < 2 * E; i += 128)
                aux->acc[i] += ((aux->red[0][i] + aux->red[1][i]) + aux->red[2][i]) + aux->red[3][i];
        }
        gate_bar();
        for (int i = gt; i < 2 * E; i += 128)
            part[(int64_t)blockIdx.x * 2 * E + i] = aux->acc[i];
        // the CTA that finishes last adds every CTA's partials in CTA order (f64) and
        // scans the chunk histogram; its ring is idle by now (every stage it loaded was
        // consumed before its last tile's logits were ready), so both are staged there
        __threadfence();
        gate_bar();
        if (gt == 0)
            aux->last = atomicAdd(counter, 1) == (int)gridDim.x - 1;
        gate_bar();
        if (aux->last) {
            __threadfence();
            float *s_part = reinterpret_cast<float *>(smem);
            const int np = (int)gridDim.x * 2 * E;  // <= 148 x 128 floats: fits the ring
            stage_words(s_part, part, np, gt, 128);
            gate_bar();
            for (int o = gt; o < 2 * E; o += 128) {
                double sum = 0.0;
                for (int b = 0; b < (int)gridDim.x; ++b)
                    sum += (double)s_part[b * 2 * E + o];
                if (o < E)
                    probs_sum[o] = (float)sum;
                else
                    importance[o - E] = (float)sum;
            }
            gate_bar();
            scan_chunk_counts(hist, E, nch, dcounts, reinterpret_cast<int32_t *>(smem),
                              C::TILE_BYTES / 4, gt, 128, GateBar());
            if (gt == 0)
                *counter = 0;
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(C::TMEM_COLS)
                     : "memory");
    }
}

// Router weights into the packed layout the kernel reads (see the file comment).
__global__ void router_pack_tc_kernel(const bf16 *__restrict__ Wg, const bf16 *__restrict__ Wn,
                                      int d, int E, int rows, bf16 *__restrict__ Wt)
{
    pdl_wait();
    pdl_trigger();
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)rows * d)
        return;
    const int o = (int)(i / d), c = (int)(i % d);
    bf16 v = __float2bfloat16_rn(0.f);
    if (Wn != nullptr) {
        if (o < 2 * E)
            v = (o & 1) ? Wn[(int64_t)c * E + (o >> 1)] : Wg[(int64_t)c * E + (o >> 1)];
    } else if (o < E) {
        v = Wg[(int64_t)c * E + o];
    }
    Wt[i] = v;
}

template <int NOUT, bool NOISY>
static cudaError_t run(const moe_params_t *p, const void *x, const bf16 *Wt,
                       const float *noise, const float *bias, int32_t *idx, float *w,
                       float *part, int32_t *counter, float *probs_sum, float *importance,
                       int32_t *hist, int32_t *dcounts, int32_t *status, cudaStream_t s)
{
    using C = Cfg<NOUT>;
    constexpr int SMEM = 1024 + C::TILE_BYTES + (int)sizeof(Aux);
    static_assert(SMEM <= 227 * 1024, "router shared memory");
    static_assert(148 * 2 * MOE_MAX_EXPERTS * 4 <= C::TILE_BYTES, "CTA partials fit the ring");
    static bool attr_done[64] = {false};
    static int sms_cached[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    if (!attr_done[dev]) {
        e = cudaFuncSetAttribute(router_tc_kernel<NOUT, NOISY>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
        if (e != cudaSuccess)
            return e;
        e = cudaDeviceGetAttribute(&sms_cached[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess)
            return e;
        if (sms_cached[dev] > 148)  // the staged CTA partials are sized for 148 CTAs
            sms_cached[dev] = 148;
        attr_done[dev] = true;
    }
    CUtensorMap tx, tw;
    const uint64_t dx[2] = {(uint64_t)p->d, (uint64_t)p->T}, sx[1] = {(uint64_t)p->d * 2};
    const uint32_t bx[2] = {BK, BM};
    const uint64_t dw[2] = {(uint64_t)p->d, (uint64_t)NOUT}, sw[1] = {(uint64_t)p->d * 2};
    const uint32_t bw[2] = {BK, NOUT};
    if ((e = tc::make_map(&tx, x, 2, dx, sx, bx)) != cudaSuccess)
        return e;
    if ((e = tc::make_map(&tw, Wt, 2, dw, sw, bw)) != cudaSuccess)
        return e;
    const int n_tiles = ceil_div(p->T, BM);
    const int grid = n_tiles < sms_cached[dev] ? n_tiles : sms_cached[dev];
    launch_pdl(router_tc_kernel<NOUT, NOISY>, dim3(grid), dim3(NUM_THREADS), SMEM, s, tx, tw,
               p->T, p->d, p->E, p->k, noise, bias, p->router_type, idx, w, part, counter,
               probs_sum, importance, hist, dcounts, status, wait_limit_ns());
    return cudaGetLastError();
}

}  // namespace rtc

int router_packed_rows(int E, bool noisy)
{
    const int nout = noisy ? 2 * E : E;
    return nout <= 16 ? 16 : nout <= 32 ? 32 : nout <= 64 ? 64 : 128;
}

cudaError_t launch_router_pack(const moe_params_t *p, const void *Wg, const void *Wnoise, void *Wt,
                               cudaStream_t s)
{
    const int rows = router_packed_rows(p->E, Wnoise != nullptr);
    const int64_t n = (int64_t)rows * p->d;
    launch_pdl(rtc::router_pack_tc_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s,
               (const bf16 *)Wg, (const bf16 *)Wnoise, p->d, p->E, rows, (bf16 *)Wt);
    count_launch();
    return cudaGetLastError();
}

// Routes a bf16 batch on the tensor cores with packed router weights, token sums and
// a2's chunk counts included.
cudaError_t launch_route_tc(const moe_params_t *p, const void *x, const void *Wt, bool noisy,
                            const float *noise, const float *bias, int32_t *idx, float *w,
                            float *probs_sum, float *importance, float *part, int32_t *counter,
                            int32_t *hist, int32_t *dcounts, int32_t *status, cudaStream_t s)
{
    const int rows = router_packed_rows(p->E, noisy);
    const bf16 *t = (const bf16 *)Wt;
    cudaError_t e;
#define MOE_RTC(NO)                                                                          \
    (noisy ? rtc::run<NO, true>(p, x, t, noise, bias, idx, w, part, counter, probs_sum,         \
                                importance, hist, dcounts, status, s)                           \
           : rtc::run<NO, false>(p, x, t, noise, bias, idx, w, part, counter, probs_sum,        \
                                 importance, hist, dcounts, status, s))
    if (rows == 16)
        e = MOE_RTC(16);
    else if (rows == 32)
        e = MOE_RTC(32);
    else if (rows == 64)
        e = MOE_RTC(64);
    else
        e = MOE_RTC(128);
#undef MOE_RTC
    count_launch();
    return e;
}

}  // namespace moe
