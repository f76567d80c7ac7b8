// sa_attn.cu -- fused low-bit attention forward for sm_100a.
//
// Two kernels, both with two 128-query tiles per persistent CTA (one softmax warpgroup per
// tile, a thread owning one query row and all 128 keys of a step):
//   attn_pairs_kernel   (sa_attn_pairs.cuh) every call without a keep mask; the two tiles
//                       read one K/V stream (causal and variable-length forms included);
//   attn_mpairs_kernel  (sa_attn_mpairs.cuh) calls with a keep mask; each tile has its own
//                       kept blocks, and their steps take turns in one K/V ring.
//
// Sources: "AIGC weekend special 5.10" section 1.2 Method, items (1) and (2)
// (SageAttention2++ INT8 Q.K^T on tensor cores; SLA sparse attention on top);
// "Video-Generation-101 research log" section 5.5 (INT Q.K^T, FP8 P.V); NetEase
// TurboDiffusion article, SLA figure caption (only critical blocks are computed);
// FlashAttention (digest timeline 2022.06) for the tiled online softmax.
//
// Shared by both: S = Q.K^T with tcgen05 kind::i8 into tensor memory; row maxima on int32
// S; P = 448 * exp(...) packed to e4m3 into a 128B-swizzled shared tile for the PV MMA
// (kind::f8f6f4); O rescaled in tensor memory when a row max grows.  The row sum l of the
// FP8 weights comes from the tensor core: each V^T stage carries 16 extra rows (row 128 =
// e4m3 1.0, rows 129-143 = 0), so the PV MMA (N = 144) writes sum_t p8_t into O column 128,
// rescaled together with O.  Every mbarrier wait is bounded; on expiry the kernel records
// SA_ERR_DEVICE_TIMEOUT in the device status word, skips all remaining work and exits.
//
// This file also holds the debug kernels (int32 S tiles, the bounded-wait test) and the
// launchers.
#include <cstdint>
#include <cuda_bf16.h>

#include "sa_internal.h"
#include "sa_ptx.cuh"

namespace sa {

__device__ int g_device_status;  // 0 = OK, 6 = a bounded wait expired

namespace {

constexpr int kOCols = 144;  // O accumulator columns: 128 channels + the row-sum column

constexpr uint32_t kQTileBytes = 128 * 128;      // 128 rows x 128 B (int8), 128B swizzle
constexpr uint32_t kKHalfBytes = 64 * 128;       // 64 keys x 128 B
constexpr uint32_t kKTileBytes = 2 * kKHalfBytes;
constexpr uint32_t kVHalfData = 128 * 64;        // 128 channels x 64 keys, 64B swizzle
constexpr uint32_t kVHalfBytes = 144 * 64;       // + 16 constant rows (row sum)
constexpr uint32_t kPTileBytes = 128 * 128;
static_assert(kVHalfBytes % 1024 == 0, "V half tiles stay 1024-B aligned");

constexpr uint32_t kIdescQK = idesc_s8_s32(128, 128);
constexpr uint32_t kIdescPV = idesc_e4m3_f32(128, kOCols);

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLog2_448 = 8.807354922057604f;

__device__ __forceinline__ void record_timeout()
{
    atomicExch(&g_device_status, int(6));
}

__device__ __forceinline__ float i2f(uint32_t x) { return __int2float_rn(int(x)); }

// In-order asm forms of the P steps: their relative order is kept as written.
__device__ __forceinline__ float cvt_s32_f32_ord(uint32_t x)
{
    float y;
    asm volatile("cvt.rn.f32.s32 %0, %1;" : "=f"(y) : "r"(x));
    return y;
}
__device__ __forceinline__ float fma_ord(float a, float b, float c)
{
    float y;
    asm volatile("fma.rn.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
    return y;
}
__device__ __forceinline__ float ex2_ord(float x)
{
    float y;
    asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ uint32_t pack_e4m3x2_ord(float lo, float hi)
{
    uint16_t r;
    asm volatile("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// ---------------------------------------------------------------------------------
// Debug: int32 S tiles through the same TMA + tcgen05 kind::i8 path.  One CTA per
// (query tile, 128-key tile, head); 128 threads; S tile stored to global.
constexpr uint32_t kDbgOffQ = 0, kDbgOffK = 16384, kDbgOffBar = 32768;
constexpr uint32_t kDbgSmem = kDbgOffBar + 64 + 1024;

__global__ void __launch_bounds__(128, 1)
    debug_qk_s32_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k, int Npad,
                        int32_t *__restrict__ s_out)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar_load = sbase + kDbgOffBar, bar_mma = sbase + kDbgOffBar + 8;
    volatile uint32_t *slot = reinterpret_cast<volatile uint32_t *>(smem + kDbgOffBar + 16);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kDbgOffBar + 20);
    const int qt = blockIdx.x, kt = blockIdx.y, bh = blockIdx.z;
    if (threadIdx.x == 0) {
        mbar_init(bar_load, 1);
        mbar_init(bar_mma, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(sbase + kDbgOffBar + 16, 128);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    bool ok = true;
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(bar_load, kQTileBytes + kKTileBytes);
        tma_load_2d(sbase + kDbgOffQ, &tm_q, bar_load, 0, bh * Npad + qt * 128);
        tma_load_2d(sbase + kDbgOffK, &tm_k, bar_load, 0, bh * Npad + kt * 128);
        tma_load_2d(sbase + kDbgOffK + kKHalfBytes, &tm_k, bar_load, 0, bh * Npad + kt * 128 + 64);
        ok = mbar_wait(bar_load, 0, abort_flag);
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_i8(tmem, sdesc(sbase + kDbgOffQ + 32 * kk, 1024, SWZ_128B),
                       sdesc(sbase + kDbgOffK + 32 * kk, 1024, SWZ_128B), kIdescQK, kk > 0);
            tc_commit(bar_mma);
        } else {
            *abort_flag = 1;
        }
    }
    __syncwarp();
    if (ok) ok = mbar_wait(bar_mma, 0, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
        tc_fence_after();
        const int r = warp * 32 + lane;
        int32_t *dst = s_out + (int64_t(bh) * Npad + qt * 128 + r) * Npad + kt * 128;
        for (int cb = 0; cb < 4; ++cb) {
            uint32_t v[32];
            tmem_ld32_wait(tmem + (uint32_t(warp * 32) << 16) + 32 * cb, v);
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<uint4 *>(dst + 32 * cb + i) = make_uint4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
    } else if (lane == 0) {
        record_timeout();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

// Debug: a wait that can never complete (no thread arrives on the barrier), bounded by
// timeout_ns; records the timeout status and returns.
__global__ void debug_wait_timeout_kernel(unsigned long long timeout_ns)
{
    __shared__ __align__(8) uint64_t barrier;
    const uint32_t b = smem_u32(&barrier);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_barrier_init();
        const uint64_t t0 = globaltimer_ns();
        bool done = false;
        while (!done && globaltimer_ns() - t0 < timeout_ns) done = mbar_try_wait(b, 0);
        if (!done) record_timeout();
    }
}

#include "sa_attn_pairs.cuh"
#include "sa_attn_mpairs.cuh"

}  // namespace

// Without a mask: two query tiles per CTA (attn_pairs_kernel).
static cudaError_t launch_attention_pairs(const AttnArgs &a, cudaStream_t st)
{
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && !attr_set[dev]) {
        if ((e = cudaFuncSetAttribute(attn_pairs_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(pairs::kSmemAlloc))) != cudaSuccess ||
            (e = cudaFuncSetAttribute(attn_pairs_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(pairs::kSmemAlloc))) != cudaSuccess)
            return e;
        attr_set[dev] = true;
    }
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int npairs = a.BH * ((a.nq + 1) / 2);
    const int grid = npairs < sms ? npairs : sms;
    if (a.seq.len)
        attn_pairs_kernel<true><<<grid, pairs::kThreads, pairs::kSmemAlloc, st>>>(
            a.tm_q, a.tm_k, a.tm_v, a.q_scale, a.k_scale, a.v_scale, a.o, a.BH, a.N, a.Npad, a.nq, a.nk,
            a.sm_scale, a.causal, a.seq);
    else
        attn_pairs_kernel<false><<<grid, pairs::kThreads, pairs::kSmemAlloc, st>>>(
            a.tm_q, a.tm_k, a.tm_v, a.q_scale, a.k_scale, a.v_scale, a.o, a.BH, a.N, a.Npad, a.nq, a.nk,
            a.sm_scale, a.causal, a.seq);
    return cudaGetLastError();
}

cudaError_t launch_attention(const AttnArgs &a, cudaStream_t st)
{
    // without a keep mask (causal or not): two query tiles per CTA on one K/V stream
    if (!a.mask) return launch_attention_pairs(a, st);
    // with one: two query tiles per CTA, each on its own kept blocks
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && !attr_set[dev]) {
        e = cudaFuncSetAttribute(attn_mpairs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(mpairs::kSmemAlloc));
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int npairs = a.BH * ((a.nq + 1) / 2);
    const int grid = npairs < sms ? npairs : sms;
    attn_mpairs_kernel<<<grid, pairs::kThreads, mpairs::kSmemAlloc, st>>>(
        a.tm_q, a.tm_k, a.tm_v, a.q_scale, a.k_scale, a.v_scale, a.mask, a.o, a.BH, a.N, a.Npad, a.nq, a.nk,
        a.sm_scale, a.causal, a.addend);
    return cudaGetLastError();
}

cudaError_t launch_debug_qk_s32(const CUtensorMap &tm_q, const CUtensorMap &tm_k, int BH, int Npad,
                                int32_t *s_out, cudaStream_t st)
{
    cudaError_t e = cudaFuncSetAttribute(debug_qk_s32_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(kDbgSmem));
    if (e != cudaSuccess) return e;
    const dim3 grid(Npad / 128, Npad / 128, BH);
    debug_qk_s32_kernel<<<grid, 128, kDbgSmem, st>>>(tm_q, tm_k, Npad, s_out);
    return cudaGetLastError();
}

cudaError_t launch_debug_wait_timeout(int timeout_us, cudaStream_t st)
{
    debug_wait_timeout_kernel<<<1, 32, 0, st>>>(1000ull * (unsigned long long)timeout_us);
    return cudaGetLastError();
}

cudaError_t read_and_clear_status(int *status)
{
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(status, g_device_status, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
}

}  // namespace sa
