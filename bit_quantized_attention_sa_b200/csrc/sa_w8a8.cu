// sa_w8a8.cu -- W8A8 linear layer: INT8 activations and weights with one scale per
// 128 x 128 block, products on the tcgen05 INT8 tensor cores.
//
// Sources: NetEase article on the TurboDiffusion release, W8A8 linear-layer quantisation
// section (weights and activations of the linear layers to 8 bits in 128 x 128 blocks, on
// INT8 tensor cores); "AIGC weekend special 5.10" section 1.2 Method item (4).
//
// y[m, n] = sum over 128-wide k-blocks b, ascending, of (float)S_b * (sx[m/128, b] *
// sw[n/128, b]), accumulated by fused multiply-add in fp32, then rounded to bf16, where
// S_b is the exact int32 product of the block's INT8 codes.
//
// w8a8_gemm_kernel: persistent clusters of two CTAs (a CTA pair on two SMs) over 256 x 256
// output tiles; the pair issues one kind::i8 MMA of M = 256, N = 256, K = 32 across both
// SMs' tensor cores (cta_group::2), so each instruction does twice the work of a one-SM MMA
// and each SM stages only half of the w tile.
//   CTA r of the pair holds rows 128 r .. 128 r + 127 of the tile's x rows and of its w
//   rows (w row = output column) for every k-block, and its 128 output rows in its own
//   tensor memory.
//   Tiles are visited in groups of 16 row tiles (column-major inside a group) so that
//   the x and w tiles in flight at once stay in L2.
//   warp 8      producer (both CTAs): TMA loads of this CTA's x half (128 rows x 128 B)
//               and w half (128 rows x 128 B) of each k-block into a 6-stage ring; both
//               halves complete on the full barrier of CTA 0.
//   warps 9-10  MMA issuers (lane 0 of each, in CTA 0): warp 9 takes the even k-blocks
//               and warp 10 the odd ones, each into its own int32 accumulator (256
//               columns), 4 MMAs per k-block, committed to the stage's empty barrier and
//               the accumulator's full barrier in both CTAs.  Two issuing threads keep
//               the tensor pipe fed where one thread's issue rate falls short.
//   warps 0-7   epilogue (both CTAs): warp w owns TMEM lane quarter w % 4 and columns
//               128 * (w / 4) .. +127 (one weight block); per k-block it reads its int32
//               block 16 columns at a time, the next load in flight while the previous
//               16 columns are converted and folded into 128 fp32 registers with the
//               block's scale, releases the accumulator (to CTA 0's empty barrier) as soon
//               as the last load has landed, and after the last k-block stores bf16 rows.
// Every mbarrier wait is bounded (sa_ptx.cuh); on expiry the kernel records the device
// timeout status and exits.
#include <cstdint>
#include <cuda_bf16.h>

#include "sa_internal.h"
#include "sa_ptx.cuh"

namespace sa {

__device__ int g_w8a8_status;  // 0 = OK, 6 = a bounded wait expired

namespace {

constexpr int kThreads = 352;  // 8 epilogue warps, the producer and two MMA issuers
constexpr int kStages = 6;
constexpr int kPairM = 256, kTileN = 256, kKB = 128, kHalf = 128;
constexpr int kWarpProducer = 8, kWarpMma = 9, kNumIssuers = 2;
constexpr uint32_t kHalfTileBytes = kHalf * kKB;              // 16 KB: 128 rows of one k-block
static_assert(kW8a8BoxRows == kHalf, "each TMA load fills one half tile");
constexpr uint32_t kStageBytes = 2 * kHalfTileBytes;           // this CTA's x half + w half
constexpr uint32_t kOffBar = kStages * kStageBytes;
constexpr int kBarFull = 0, kBarEmpty = kStages, kBarAccFull = 2 * kStages, kBarAccEmpty = kBarAccFull + 2,
              kNumBars = kBarAccEmpty + 2;
constexpr uint32_t kOffMisc = kOffBar + 8 * kNumBars;
constexpr uint32_t kSmemAlloc = kOffMisc + 16 + 1024;
static_assert(kSmemAlloc <= 227 * 1024, "shared memory per CTA");
constexpr uint32_t kIdesc = idesc_s8_s32(kPairM, kTileN);
constexpr int kEpilogueWarps = 8;
static_assert(kStages % kNumIssuers == 0, "each stage is always consumed by the same issuer");

__device__ __forceinline__ void record_timeout() { atomicExch(&g_w8a8_status, int(6)); }

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// INT8 code of x under scale s (r = 1/s): round-half-even of the IEEE quotient x/s,
// clamped to [-127, 127].  y = x*r differs from fl(x/s) by < |x/s| * 3 * 2^-24 < 2.3e-5,
// so unless y is within 2^-14 of a half-integer both round alike; otherwise the exact
// division decides.
__device__ __forceinline__ int int8_code(float x, float s, float r)
{
    if (s == 0.0f) return 0;
    const float y = __fmul_rn(x, r);
    float n = rintf(y);
    if (fabsf(fabsf(__fsub_rn(y, n)) - 0.5f) < 6.103515625e-05f) n = rintf(__fdiv_rn(x, s));
    return max(-127, min(127, int(n)));
}

// grid (ceil(cols/128), ceil(rows/128)), 256 threads: one 128 x 128 block of x (bf16,
// row stride cols) -> codes (row stride kpad, the block's padding columns zero) and its
// scale.  cols is a multiple of 8 (16-byte rows of 8 values).
__global__ void __launch_bounds__(256, 2)
    w8a8_quant_kernel(const uint16_t *__restrict__ x, int64_t rows, int64_t cols, int64_t kpad,
                      int8_t *__restrict__ codes, float *__restrict__ scales)
{
    __shared__ float red[8];
    const int tid = threadIdx.x, cg = tid & 15, rs = tid >> 4;
    const int64_t r0 = int64_t(blockIdx.y) * 128, c0 = int64_t(blockIdx.x) * 128;
    const int64_t col = c0 + cg * 8;
    const bool cvalid = col < cols;
    uint4 raw[8];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t r = r0 + rs + 16 * i;
        raw[i] = (r < rows && cvalid) ? __ldg(reinterpret_cast<const uint4 *>(x + r * cols + col))
                                      : make_uint4(0, 0, 0, 0);
        const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            amax = fmaxf(amax, fmaxf(fabsf(bf16_bits_to_f32(w[e] & 0xFFFFu)), fabsf(bf16_bits_to_f32(w[e] >> 16))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
    const float s = __fdiv_rn(amax, 127.0f);
    const float rcp = s == 0.0f ? 0.0f : __frcp_rn(s);
    if (tid == 0) scales[int64_t(blockIdx.y) * gridDim.x + blockIdx.x] = s;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t r = r0 + rs + 16 * i;
        if (r >= rows) continue;
        const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint32_t a = uint8_t(int8_code(bf16_bits_to_f32(w[e] & 0xFFFFu), s, rcp));
            const uint32_t b = uint8_t(int8_code(bf16_bits_to_f32(w[e] >> 16), s, rcp));
            if (e < 2) lo |= (a | (b << 8)) << (16 * e);
            else hi |= (a | (b << 8)) << (16 * (e - 2));
        }
        *reinterpret_cast<uint2 *>(codes + r * kpad + col) = make_uint2(lo, hi);
    }
}

// ------------------------------------------------------------------ CTA-pair primitives
// (cluster of two CTAs; every tcgen05 instruction of the kernel uses cta_group::2)

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// All threads of both CTAs; orders earlier shared-memory writes (barrier initialisation)
// before the peer's later accesses.
__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The shared::cluster address of the object at shared::cta address `addr` in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// Arrive with no memory ordering: for releases whose only prior accesses are tensor-memory
// loads already waited for (ordered by tcgen05.fence::before_thread_sync).
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t caddr)
{
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}

// 16 columns of this warp's TMEM lanes, without waiting: the registers are valid only
// after tmem_wait_ld() and regs_ready16().
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Makes the compiler treat r as produced here, after the wait, so no use of the loaded
// values is scheduled before it.
__device__ __forceinline__ void regs_ready16(uint32_t (&r)[16])
{
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
}

// 2-D tiled TMA load into this CTA's shared memory whose byte count completes on the
// mbarrier at shared::cluster address `bar_c` (this CTA's or its peer's).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void *tmap, uint32_t bar_c, int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar_c), "r"(x), "r"(y)
        : "memory");
}

// Collective over one warp in each CTA of the pair: both get the same base address.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D (both CTAs' tensor memory) (+)= A (128 rows in each CTA) * B^T (N/2 rows in each CTA).
__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives once on the mbarrier at shared::cluster address `bar_c` when every tcgen05
// operation issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar_c)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_c)
                 : "memory");
}

// Tile t -> (mt, nt): tiles go in groups of kGroupM row tiles, column-major inside a group,
// so that the tiles in flight at once (consecutive t) share a few row tiles of x and
// column tiles of w, and each x tile is read from DRAM once while its group runs.
constexpr int kGroupM = 16;
__device__ __forceinline__ void tile_coords(int t, int nmt, int nnt, int &mt, int &nt)
{
    const int per_group = kGroupM * nnt;
    const int grp = t / per_group, idx = t - grp * per_group;
    const int gm = min(kGroupM, nmt - grp * kGroupM);
    mt = grp * kGroupM + idx % gm;
    nt = idx / gm;
}

// grid: 2 x (number of co-resident pairs), clusters of 2; 384 threads.  x8 [M, kpad] and
// w8 [N, kpad] through the tensor maps (box 128 B x 128 rows), sx [ceil(M/128), nkb],
// sw [ceil(N/128), nkb]; y bf16 [M, N] (N a multiple of 8).
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    w8a8_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     const float *__restrict__ sx, const float *__restrict__ sw, int M, int N, int nkb,
                     __nv_bfloat16 *__restrict__ y)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
    auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * uint32_t(i); };
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(kBarFull + s), 1);   // CTA 0's: its producer's arrive + both CTAs' bytes
            mbar_init(bar(kBarEmpty + s), 1);  // one commit of the MMA issuer
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(kBarAccFull + b), 1);
            mbar_init(bar(kBarAccEmpty + b), 2 * kEpilogueWarps);  // CTA 0's: both CTAs' epilogue warps
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) tmem_alloc_pair(sbase + kOffMisc, 512);
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int nmt = (M + kPairM - 1) / kPairM, nnt = (N + kTileN - 1) / kTileN, ntiles = nmt * nnt;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (warp >= kWarpProducer) {
        if (warp == kWarpProducer && lane == 0) {
            prefetch_tmap(&tm_x);
            prefetch_tmap(&tm_w);
            bool ok = true;
            uint32_t g = 0;
            for (int t = pair; t < ntiles && ok; t += npairs) {
                int mt, nt;
                tile_coords(t, nmt, nnt, mt, nt);
                for (int b = 0; b < nkb && ok; ++b, ++g) {
                    const uint32_t st = g % kStages;
                    if (g >= kStages) ok = mbar_wait(bar(kBarEmpty + st), ((g / kStages) - 1) & 1, abort_flag);
                    if (!ok) break;
                    const uint32_t xs = sbase + st * kStageBytes, ws = xs + kHalfTileBytes;
                    const uint32_t full0 = cluster_addr(bar(kBarFull + st), 0);
                    if (rank == 0) mbar_arrive_expect_tx(bar(kBarFull + st), 2 * kStageBytes);
                    tma_load_2d_pair(xs, &tm_x, full0, b * kKB, mt * kPairM + int(rank) * kHalf);
                    tma_load_2d_pair(ws, &tm_w, full0, b * kKB, nt * kTileN + int(rank) * kHalf);
                }
            }
            // drain: the issuer's last commits to this CTA's empty barriers have landed
            for (uint32_t d = g > kStages ? g - kStages : 0; d < g && ok; ++d)
                ok = mbar_wait(bar(kBarEmpty + d % kStages), (d / kStages) & 1, abort_flag);
            if (!ok) { *abort_flag = 1; record_timeout(); }
        } else if (warp >= kWarpMma && warp < kWarpMma + kNumIssuers && lane == 0 && rank == 0) {
            bool ok = true;
            uint32_t g = 0;
            const uint32_t me = uint32_t(warp - kWarpMma);  // this issuer's k-blocks: g % 2 == me
            for (int t = pair; t < ntiles && ok; t += npairs) {
                for (int b = 0; b < nkb && ok; ++b, ++g) {
                    if ((g & 1) != me) continue;
                    const uint32_t st = g % kStages, ab = g & 1;
                    ok = mbar_wait(bar(kBarFull + st), (g / kStages) & 1, abort_flag);
                    if (ok && g >= 2) ok = mbar_wait(bar(kBarAccEmpty + ab), ((g >> 1) - 1) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t xs = sbase + st * kStageBytes, ws = xs + kHalfTileBytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_i8_pair(tmem + ab * kTileN, sdesc(xs + 32 * kk, 1024, SWZ_128B),
                                    sdesc(ws + 32 * kk, 1024, SWZ_128B), kIdesc, kk > 0);
                    tc_commit_pair(cluster_addr(bar(kBarEmpty + st), 0));
                    tc_commit_pair(cluster_addr(bar(kBarEmpty + st), 1));
                    tc_commit_pair(cluster_addr(bar(kBarAccFull + ab), 0));
                    tc_commit_pair(cluster_addr(bar(kBarAccFull + ab), 1));
                }
            }
            if (!ok) { *abort_flag = 1; record_timeout(); }
        }
    } else {
        // ---------------------------------------------------------------- epilogue warps 0-7
        const int wq = warp & 3, half = warp >> 2;
        const uint32_t lane_addr = uint32_t(wq * 32) << 16;
        const int nbm = (M + kHalf - 1) / kHalf, nbn = (N + kHalf - 1) / kHalf;
        bool ok = true;
        uint32_t g = 0;
        for (int t = pair; t < ntiles; t += npairs) {
            int mt, nt;
            tile_coords(t, nmt, nnt, mt, nt);
            const int mb = mt * 2 + int(rank), nb = nt * 2 + half;  // this warp's x and w block rows
            const bool live = mb < nbm && nb < nbn;
            float acc[128];
#pragma unroll
            for (int c = 0; c < 128; ++c) acc[c] = 0.0f;
            // the block scales of k-block b + 1 load while k-block b is processed
            const float *sxr = sx + int64_t(live ? mb : 0) * nkb, *swr = sw + int64_t(live ? nb : 0) * nkb;
            float sx_next = live ? sxr[0] : 0.0f, sw_next = live ? swr[0] : 0.0f;
            for (int b = 0; b < nkb; ++b, ++g) {
                const uint32_t ab = g & 1;
                const float s = sx_next * sw_next;  // the block's scale product, as in the definition
                if (live && b + 1 < nkb) {
                    sx_next = sxr[b + 1];
                    sw_next = swr[b + 1];
                }
                if (ok) ok = mbar_wait(bar(kBarAccFull + ab), (g >> 1) & 1, abort_flag);
                ok = __all_sync(0xffffffffu, ok);
                const uint32_t acc_empty = cluster_addr(bar(kBarAccEmpty + ab), 0);
                if (!ok) {
                    if (lane == 0) mbar_arrive_cluster_relaxed(acc_empty);
                    continue;
                }
                tc_fence_after();
                const uint32_t ta = tmem + lane_addr + ab * kTileN + half * 128;
                // 16-column chunks: chunk q + 1 is loading while chunk q is folded in
                uint32_t va[16], vb[16];
                tmem_ld16_nowait(ta, va);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    uint32_t(&cur)[16] = (q & 1) ? vb : va;
                    uint32_t(&nxt)[16] = (q & 1) ? va : vb;
                    tmem_wait_ld();
                    regs_ready16(cur);
                    if (q == 7) {
                        // the warp's whole block is in registers: release the accumulator
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster_relaxed(acc_empty);
                    } else {
                        tmem_ld16_nowait(ta + 16 * (q + 1), nxt);
                    }
#pragma unroll
                    for (int i = 0; i < 16; i += 2)
                        fma2(acc[16 * q + i], acc[16 * q + i + 1], __int2float_rn(int(cur[i])),
                             __int2float_rn(int(cur[i + 1])), s, s, acc[16 * q + i], acc[16 * q + i + 1]);
                }
            }
            // bf16 row of 128 columns: 16-byte stores, columns < N
            const int64_t m = int64_t(mb) * kHalf + wq * 32 + lane;
            const int n0 = nb * kHalf;
            if (m < M && ok) {
                __nv_bfloat16 *yr = y + m * N + n0;
#pragma unroll
                for (int c = 0; c < 128; c += 8) {
                    if (n0 + c >= N) break;
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[c + 2 * e], acc[c + 2 * e + 1]);
                        w[e] = *reinterpret_cast<const uint32_t *>(&h2);
                    }
                    *reinterpret_cast<uint4 *>(yr + c) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
        if (lane == 0 && !ok) { *abort_flag = 1; record_timeout(); }
    }
    __syncwarp();
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    if (warp == kWarpMma) tmem_dealloc_pair(tmem, 512);
}

}  // namespace

cudaError_t launch_w8a8_quantize(const void *x, int64_t rows, int64_t cols, int8_t *codes, float *scales,
                                 cudaStream_t st)
{
    const int64_t cb = (cols + 127) / 128;
    const dim3 g(unsigned(cb), unsigned((rows + 127) / 128));
    w8a8_quant_kernel<<<g, 256, 0, st>>>(static_cast<const uint16_t *>(x), rows, cols, cb * 128, codes, scales);
    return cudaGetLastError();
}

cudaError_t launch_w8a8_gemm(const CUtensorMap &tm_x, const CUtensorMap &tm_w, const float *sx,
                             const float *sw, int M, int N, int nkb, void *y, cudaStream_t st)
{
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        e = cudaFuncSetAttribute(w8a8_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemAlloc));
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    // co-resident CTA pairs (clusters of two), computed once per device
    static int max_pairs[64] = {0};
    int pairs = dev >= 0 && dev < 64 ? max_pairs[dev] : 0;
    if (pairs <= 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = kSmemAlloc;
        e = cudaOccupancyMaxActiveClusters(&pairs, w8a8_gemm_kernel, &cfg);
        if (e != cudaSuccess) return e;
        if (pairs < 1) return cudaErrorInvalidConfiguration;
        if (dev >= 0 && dev < 64) max_pairs[dev] = pairs;
    }
    const int ntiles = ((M + kPairM - 1) / kPairM) * ((N + kTileN - 1) / kTileN);
    const int grid = 2 * (ntiles < pairs ? ntiles : pairs);
    w8a8_gemm_kernel<<<grid, kThreads, kSmemAlloc, st>>>(tm_x, tm_w, sx, sw, M, N, nkb,
                                                          static_cast<__nv_bfloat16 *>(y));
    return cudaGetLastError();
}

cudaError_t read_and_clear_w8a8_status(int *status)
{
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(status, g_w8a8_status, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_w8a8_status, &zero, sizeof(int));
}

}  // namespace sa
