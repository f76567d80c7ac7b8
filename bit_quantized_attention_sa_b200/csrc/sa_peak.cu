// sa_peak.cu -- measured 8-bit tensor-core peak of this device: the denominator of the
// attention kernel's roofline.  One CTA per SM issues back-to-back tcgen05 MMAs of
// M = 128, N = 256, K = 32 (kind::i8 or kind::f8f6f4 with e4m3 operands) from shared-memory
// tiles into two tensor-memory accumulators, in chains of four (one K = 128 contraction,
// as the attention kernel issues them).  The host times the launch; every MMA does
// 2 * 128 * 256 * 32 operations.  Operand values do not matter for the rate; the tiles hold
// a fixed non-zero pattern.
#include <cstdint>

#include "sa_internal.h"
#include "sa_ptx.cuh"

namespace sa {

__device__ int g_peak_status;  // 0 = OK, 6 = the final bounded wait expired

namespace {

constexpr uint32_t kPeakA = 0, kPeakB = 128 * 128;            // A: 128 rows, B: 256 rows, 128 B each
constexpr uint32_t kPeakBar = kPeakB + 256 * 128;
constexpr uint32_t kPeakSmem = kPeakBar + 64 + 1024;

__global__ void __launch_bounds__(128, 1) mma_peak_kernel(int kind, int reps)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    volatile uint32_t *slot = reinterpret_cast<volatile uint32_t *>(smem + kPeakBar + 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kPeakBar + 12);
    for (uint32_t i = threadIdx.x; i < kPeakBar / 4; i += blockDim.x)
        reinterpret_cast<uint32_t *>(smem)[i] = 0x11223344u ^ (i * 0x9E3779B9u);
    fence_proxy_async_smem();
    if (threadIdx.x == 0) {
        mbar_init(sbase + kPeakBar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (threadIdx.x < 32) tmem_alloc(sbase + kPeakBar + 8, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    if (threadIdx.x == 0) {
        const uint32_t idesc_i8 = idesc_s8_s32(128, 256), idesc_f8 = idesc_e4m3_f32(128, 256);
        for (int r = 0; r < reps; ++r) {
            const uint32_t d = tmem + 256u * uint32_t(r & 1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t a = sdesc(sbase + kPeakA + 32 * kk, 1024, SWZ_128B);
                const uint64_t b = sdesc(sbase + kPeakB + 32 * kk, 1024, SWZ_128B);
                if (kind == 0)
                    mma_i8(d, a, b, idesc_i8, kk > 0);
                else
                    mma_f8(d, a, b, idesc_f8, kk > 0);
            }
        }
        tc_commit(sbase + kPeakBar);
        if (!mbar_wait(sbase + kPeakBar, 0, abort_flag)) atomicExch(&g_peak_status, 6);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x < 32) tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_mma_peak(int kind, int reps, cudaStream_t st)
{
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(mma_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kPeakSmem))) !=
        cudaSuccess)
        return e;
    mma_peak_kernel<<<sms, 128, kPeakSmem, st>>>(kind, reps);
    return cudaGetLastError();
}

cudaError_t read_and_clear_peak_status(int *status)
{
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(status, g_peak_status, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_peak_status, &zero, sizeof(int));
}

}  // namespace sa
