// sa_attn.cu -- fused low-bit attention forward for sm_100a.
//
// Two kernels: attn_pairs_kernel (sa_attn_pairs.cuh) runs every call without a keep mask,
// two query tiles per CTA; attn_fwd_kernel below runs masked calls, one query tile per
// CTA, since two tiles generally keep different key blocks.
//
// Sources: "AIGC weekend special 5.10" section 1.2 Method, items (1) and (2)
// (SageAttention2++ INT8 Q.K^T on tensor cores; SLA sparse attention on top);
// "Video-Generation-101 research log" section 5.5 (INT Q.K^T, FP8 P.V); NetEase
// TurboDiffusion article, SLA figure caption (only critical blocks are computed);
// FlashAttention (digest timeline 2022.06) for the tiled online softmax.
//
// One persistent CTA per SM walks (head, 128-query tile) work items.  Roles:
//   warp 8      producer: scans the tile's keep-mask row, pairs consecutive kept 64-key
//               blocks into 128-key steps and TMA-loads the K (INT8) and V^T (FP8) tiles
//               of each step into a STAGES-deep ring; loads the Q tile once per item.
//   warp 9      QK issuer (one thread): S = Q.K^T with tcgen05 kind::i8 into one of two
//               tensor-memory S buffers.
//   warp 10     PV issuer (one thread): O += P.V with kind::f8f6f4 into the O buffer.
//               A tcgen05.mma holds its issuing warp for ~200 cycles whatever its shape,
//               so the two streams are issued from two warps to overlap in the tensor core.
//   warps 0-7   softmax: two warpgroups share each S tile by key half (warpgroup w owns
//               the step's w-th 64-key block, so one K scale per thread); each thread owns
//               one query row (its TMEM lane).  Row maxima are taken on int32 S and
//               exchanged between the two warps that own the same rows; P = 448 * exp(...)
//               is packed to e4m3 into a 128B-swizzled shared tile for the PV MMA; O is
//               rescaled in tensor memory when a row max grows; the epilogue normalises
//               and stores bf16 rows.
// The row sum l of the FP8 weights comes from the tensor core: each V^T stage carries
// 16 extra rows (row 128 = e4m3 1.0, rows 129-143 = 0), so the PV MMA (N = 144) writes
// sum_t p8_t into O column 128, rescaled together with O.
//
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O [256,400).
// Every mbarrier wait is bounded; on expiry the kernel records SA_ERR_DEVICE_TIMEOUT in
// the device status word, skips all remaining work and exits.
#include <cstdint>
#include <cuda_bf16.h>

#include "sa_internal.h"
#include "sa_ptx.cuh"

namespace sa {

__device__ int g_device_status;  // 0 = OK, 6 = a bounded wait expired

namespace {

constexpr int kStages = 4;
constexpr int kThreads = 352;
constexpr int kWarpProducer = 8;
constexpr int kWarpMmaQK = 9;
constexpr int kWarpMmaPV = 10;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
constexpr int kOCols = 144;

constexpr uint32_t kQTileBytes = 128 * 128;      // 128 rows x 128 B (int8), 128B swizzle
constexpr uint32_t kKHalfBytes = 64 * 128;       // 64 keys x 128 B
constexpr uint32_t kKTileBytes = 2 * kKHalfBytes;
constexpr uint32_t kVHalfData = 128 * 64;        // 128 channels x 64 keys, 64B swizzle
constexpr uint32_t kVHalfBytes = 144 * 64;       // + 16 constant rows (row sum)
constexpr uint32_t kPTileBytes = 128 * 128;

constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + 2 * kQTileBytes;
constexpr uint32_t kOffV = kOffK + kStages * kKTileBytes;
constexpr uint32_t kOffP = kOffV + kStages * 2 * kVHalfBytes;
constexpr uint32_t kOffBar = kOffP + 2 * kPTileBytes;
// barrier indices
constexpr int kBarQFull = 0, kBarQEmpty = 2, kBarKvFull = 4, kBarKvEmpty = 4 + kStages,
              kBarSFull = 4 + 2 * kStages, kBarSEmpty = kBarSFull + 2, kBarPFull = kBarSEmpty + 2,
              kBarPvDone = kBarPFull + 2, kBarOFull = kBarPvDone + 2, kBarOEmpty = kBarOFull + 1,
              kNumBars = kBarOEmpty + 1;
constexpr uint32_t kOffInfo = kOffBar + 8 * kNumBars;            // int2 [kStages]
constexpr uint32_t kOffXch = kOffInfo + 8 * kStages;             // float [2][2][128]
constexpr uint32_t kOffMisc = kOffXch + 4 * 2 * 2 * 128;         // tmem base, abort flag
constexpr uint32_t kSmemBytes = kOffMisc + 16;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;               // 1024-B alignment slack

static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffP % 1024 == 0, "tile alignment");
static_assert(kVHalfBytes % 1024 == 0, "V half tiles stay 1024-B aligned");

constexpr uint32_t kIdescQK = idesc_s8_s32(128, 128);
constexpr uint32_t kIdescPV = idesc_e4m3_f32(128, kOCols);

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLog2_448 = 8.807354922057604f;

__device__ __forceinline__ void record_timeout()
{
    atomicExch(&g_device_status, int(6));
}

// Number of kept 64-key blocks in a mask row (warp-wide; all lanes must call).
__device__ __forceinline__ int count_kept(const uint8_t *mrow, int nk, int lane)
{
    if (!mrow) return nk;
    int cnt = 0;
    for (int base = 0; base < nk; base += 32) {
        const int j = base + lane;
        const bool keep = j < nk && mrow[j] != 0;
        cnt += __popc(__ballot_sync(0xffffffffu, keep));
    }
    return cnt;
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

// 64 keys of S (a: keys 0-31, b: keys 32-63) -> 16 words of e4m3 P = 448 * 2^(S*k +
// nbias); with MASK, bytes of keys at or past nvalid are zero.  Computed as a software
// pipeline (exponent arguments of word w+1, ex2 of word w, packing of word w-1), as the
// 128-key row of the pair kernel, so that a warp alone in this phase keeps the
// multi-function unit busier.
template <bool MASK>
__device__ __forceinline__ void p_half_impl(const uint32_t (&a)[32], const uint32_t (&b)[32], float k,
                                            float nbias, int nvalid, uint32_t (&pw)[16])
{
#define SA_HV(key) ((key) < 32 ? a[(key)] : b[(key) - 32])
    float y[2][4], e[2][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) y[0][i] = fma_ord(cvt_s32_f32_ord(SA_HV(i)), k, nbias);
#pragma unroll
    for (int w = 0; w < 17; ++w) {
        const int cur = w & 1, nxt = cur ^ 1;
        if (w + 1 < 16) {
#pragma unroll
            for (int i = 0; i < 4; ++i) y[nxt][i] = fma_ord(cvt_s32_f32_ord(SA_HV(4 * (w + 1) + i)), k, nbias);
        }
        if (w < 16) {
#pragma unroll
            for (int i = 0; i < 4; ++i) e[cur][i] = ex2_ord(y[cur][i]);
        }
        if (w >= 1) {
            uint32_t x = pack_e4m3x2_ord(e[nxt][0], e[nxt][1]) | (pack_e4m3x2_ord(e[nxt][2], e[nxt][3]) << 16);
            if (MASK) {
                const int kb = nvalid - 4 * (w - 1);  // bytes of this word to keep
                x = kb >= 4 ? x : (kb <= 0 ? 0u : (x & ((1u << (8 * kb)) - 1u)));
            }
            pw[w - 1] = x;
        }
    }
#undef SA_HV
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ q_scale,
                    const float *__restrict__ k_scale, const float *__restrict__ v_scale,
                    const uint8_t *__restrict__ mask, __nv_bfloat16 *__restrict__ out, int BH,
                    int N, int Npad, int nq, int nk, float sm_scale, int causal,
                    const float *__restrict__ addend)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int2 *info = reinterpret_cast<int2 *>(smem + kOffInfo);
    float *xch = reinterpret_cast<float *>(smem + kOffXch);
    volatile uint32_t *tmem_base_slot = reinterpret_cast<volatile uint32_t *>(smem + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
    auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * uint32_t(i); };

    // ---- set-up: barriers, constant V rows, tensor memory
    if (threadIdx.x == 0) {
        mbar_init(bar(kBarQFull + 0), 1);
        mbar_init(bar(kBarQFull + 1), 1);
        mbar_init(bar(kBarQEmpty + 0), 1);
        mbar_init(bar(kBarQEmpty + 1), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(kBarKvFull + s), 1);
            mbar_init(bar(kBarKvEmpty + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(kBarSFull + b), 1);
            mbar_init(bar(kBarSEmpty + b), 8);
            mbar_init(bar(kBarPFull + b), 8);
            mbar_init(bar(kBarPvDone + b), 1);
        }
        mbar_init(bar(kBarOFull), 1);
        mbar_init(bar(kBarOEmpty), 8);
        *abort_flag = 0;
        fence_barrier_init();
    }
    // rows 128..143 of every V half tile: row 128 all e4m3 1.0 (0x38), the rest zero
    for (int i = threadIdx.x; i < kStages * 2 * 16 * 16; i += kThreads) {
        const int half = i / (16 * 16), w = i % (16 * 16);  // 16 rows x 16 words
        uint32_t *p = reinterpret_cast<uint32_t *>(smem + kOffV + half * kVHalfBytes + kVHalfData);
        p[w] = (w < 16) ? 0x38383838u : 0u;
    }
    fence_proxy_async_smem();
    if (warp == kWarpMmaQK) tmem_alloc(sbase + kOffMisc, kTmemCols);
    if (warp == kWarpProducer && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_slot;

    const int ntiles = BH * nq;

    if (warp == kWarpProducer) {
        // ------------------------------------------------------------ producer
        bool ok = true;
        uint32_t g = 0, tl = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tl) {
            const int bh = tile / nq, qt = tile % nq;
            const uint8_t *mrow = mask ? mask + (int64_t(bh) * nq + qt) * nk : nullptr;
            const uint32_t qb = tl & 1;
            if (lane == 0) {
                if (tl >= 2 && ok) ok = mbar_wait(bar(kBarQEmpty + qb), ((tl >> 1) - 1) & 1, abort_flag);
                if (ok) {
                    mbar_arrive_expect_tx(bar(kBarQFull + qb), kQTileBytes);
                    tma_load_2d(sbase + kOffQ + qb * kQTileBytes, &tm_q, bar(kBarQFull + qb), 0,
                                bh * Npad + qt * 128);
                }
            }
            int pending = -1;
            for (int base = 0; base < nk; base += 32) {
                const int jj = base + lane;
                const bool keep = jj < nk && (!mrow || mrow[jj] != 0);
                uint32_t bits = __ballot_sync(0xffffffffu, keep);
                if (lane == 0) {
                    while (bits) {
                        const int j = base + __ffs(bits) - 1;
                        bits &= bits - 1;
                        if (pending < 0) { pending = j; continue; }
                        // issue the step (pending, j)
                        const uint32_t st = g % kStages;
                        if (g >= kStages && ok)
                            ok = mbar_wait(bar(kBarKvEmpty + st), ((g / kStages) - 1) & 1, abort_flag);
                        if (ok) {
                            info[st] = make_int2(pending, j);
                            const uint32_t kb = sbase + kOffK + st * kKTileBytes;
                            const uint32_t vb = sbase + kOffV + st * 2 * kVHalfBytes;
                            mbar_arrive_expect_tx(bar(kBarKvFull + st), 2 * (kKHalfBytes + kVHalfData));
                            tma_load_2d(kb, &tm_k, bar(kBarKvFull + st), 0, bh * Npad + pending * 64);
                            tma_load_2d(kb + kKHalfBytes, &tm_k, bar(kBarKvFull + st), 0, bh * Npad + j * 64);
                            tma_load_2d(vb, &tm_v, bar(kBarKvFull + st), pending * 64, bh * 128);
                            tma_load_2d(vb + kVHalfBytes, &tm_v, bar(kBarKvFull + st), j * 64, bh * 128);
                        }
                        pending = -1;
                        ++g;
                    }
                }
            }
            if (lane == 0 && pending >= 0) {
                const uint32_t st = g % kStages;
                if (g >= kStages && ok)
                    ok = mbar_wait(bar(kBarKvEmpty + st), ((g / kStages) - 1) & 1, abort_flag);
                if (ok) {
                    info[st] = make_int2(pending, -1);
                    const uint32_t kb = sbase + kOffK + st * kKTileBytes;
                    const uint32_t vb = sbase + kOffV + st * 2 * kVHalfBytes;
                    mbar_arrive_expect_tx(bar(kBarKvFull + st), kKHalfBytes + kVHalfData);
                    tma_load_2d(kb, &tm_k, bar(kBarKvFull + st), 0, bh * Npad + pending * 64);
                    tma_load_2d(vb, &tm_v, bar(kBarKvFull + st), pending * 64, bh * 128);
                }
                ++g;
            }
            __syncwarp();
        }
        if (lane == 0 && !ok) { *abort_flag = 1; record_timeout(); }
    } else if (warp == kWarpMmaQK) {
        // ------------------------------------------------------------ QK issuer
        // A tcgen05.mma blocks its issuing warp for roughly 200 cycles whatever its size,
        // so S = Q.K^T and O += P.V are issued from two warps and overlap in the tensor
        // core; each warp commits only its own operations.
        bool ok = true;
        uint32_t g = 0, tl = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tl) {
            const int bh = tile / nq, qt = tile % nq;
            const uint8_t *mrow = mask ? mask + (int64_t(bh) * nq + qt) * nk : nullptr;
            const int n = (count_kept(mrow, nk, lane) + 1) / 2;
            const uint32_t qb = tl & 1;
            if (lane == 0) {
                if (ok) ok = mbar_wait(bar(kBarQFull + qb), (tl >> 1) & 1, abort_flag);
                tc_fence_after();
                const uint32_t qa = sbase + kOffQ + qb * kQTileBytes;
                for (int s = 0; s < n; ++s) {
                    const uint32_t gg = g + s, st = gg % kStages, sb = gg & 1;
                    if (ok) ok = mbar_wait(bar(kBarKvFull + st), (gg / kStages) & 1, abort_flag);
                    if (gg >= 2 && ok) ok = mbar_wait(bar(kBarSEmpty + sb), ((gg >> 1) - 1) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t kb = sbase + kOffK + st * kKTileBytes;
                    const uint32_t dcol = tmem + (sb ? kColS1 : kColS0);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_i8(dcol, sdesc(qa + 32 * kk, 1024, SWZ_128B),
                               sdesc(kb + 32 * kk, 1024, SWZ_128B), kIdescQK, kk > 0);
                    tc_commit(bar(kBarSFull + sb));
                }
                if (ok) tc_commit(bar(kBarQEmpty + qb));
            }
            __syncwarp();
            g += n;
        }
        if (lane == 0 && !ok) { *abort_flag = 1; record_timeout(); }
    } else if (warp == kWarpMmaPV) {
        // ------------------------------------------------------------ PV issuer
        bool ok = true;
        uint32_t g = 0, otile = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
            const int bh = tile / nq, qt = tile % nq;
            const uint8_t *mrow = mask ? mask + (int64_t(bh) * nq + qt) * nk : nullptr;
            const int n = (count_kept(mrow, nk, lane) + 1) / 2;
            if (lane == 0 && n > 0) {
                for (int s = 0; s < n; ++s) {
                    const uint32_t gg = g + s, st = gg % kStages, sb = gg & 1;
                    // V of the stage (already complete: the softmax's P implies it) and P
                    if (ok) ok = mbar_wait(bar(kBarKvFull + st), (gg / kStages) & 1, abort_flag);
                    if (ok) ok = mbar_wait(bar(kBarPFull + sb), (gg >> 1) & 1, abort_flag);
                    if (s == 0 && otile >= 1 && ok)
                        ok = mbar_wait(bar(kBarOEmpty), (otile - 1) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const int nk_step = info[st].y >= 0 ? 4 : 2;
                    const uint32_t pa = sbase + kOffP + sb * kPTileBytes;
                    const uint32_t vb = sbase + kOffV + st * 2 * kVHalfBytes;
                    for (int kk = 0; kk < nk_step; ++kk)
                        mma_f8(tmem + kColO, sdesc(pa + 32 * kk, 1024, SWZ_128B),
                               sdesc(vb + (kk >> 1) * kVHalfBytes + 32 * (kk & 1), 512, SWZ_64B),
                               kIdescPV, (s > 0 || kk > 0) ? 1u : 0u);
                    // QK of this step completed before its P existed, so the stage is free
                    // once this PV completes
                    tc_commit(bar(kBarKvEmpty + st));
                    tc_commit(bar(kBarPvDone + sb));
                }
                if (ok) tc_commit(bar(kBarOFull));
            }
            __syncwarp();
            g += n;
            if (n > 0) ++otile;
        }
        if (lane == 0 && !ok) { *abort_flag = 1; record_timeout(); }
    } else {
        // ------------------------------------------------------------ softmax warps 0-7
        const int wg = warp >> 2;        // key half owned by this warpgroup
        const int wq = warp & 3;         // TMEM lane quarter
        const int row = wq * 32 + lane;  // query row within the tile
        const uint32_t lane_addr = uint32_t(wq * 32) << 16;
        bool ok = true;
        uint32_t g = 0, otile = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
            const int bh = tile / nq, qt = tile % nq;
            const uint8_t *mrow = mask ? mask + (int64_t(bh) * nq + qt) * nk : nullptr;
            const int n = (count_kept(mrow, nk, lane) + 1) / 2;
            const int qrow = qt * 128 + row;
            __nv_bfloat16 *orow = out + (int64_t(bh) * N + qrow) * kD + 64 * wg;
            // the addend's half row (fp32), added before the one rounding to bf16
            const float *arow = addend ? addend + (int64_t(bh) * N + qrow) * kD + 64 * wg : nullptr;
            if (n == 0) {
                if (qrow < N) {
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        uint32_t w[4] = {0u, 0u, 0u, 0u};
                        if (arow) {
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const __nv_bfloat162 h2 = __floats2bfloat162_rn(arow[8 * c + 2 * e], arow[8 * c + 2 * e + 1]);
                                w[e] = *reinterpret_cast<const uint32_t *>(&h2);
                            }
                        }
                        reinterpret_cast<uint4 *>(orow)[c] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
                continue;
            }
            const float sq = q_scale[int64_t(bh) * nq + qt];
            float m = -INFINITY;
            for (int s = 0; s < n; ++s) {
                const uint32_t gg = g + s, st = gg % kStages, sb = gg & 1;
                if (ok) ok = mbar_wait(bar(kBarKvFull + st), (gg / kStages) & 1, abort_flag);
                if (ok) ok = mbar_wait(bar(kBarSFull + sb), (gg >> 1) & 1, abort_flag);
                ok = __all_sync(0xffffffffu, ok);
                const int2 jp = info[st];
                const int j = ok ? (wg ? jp.y : jp.x) : -1;  // info is only valid once loaded
                int nvalid = j >= 0 ? min(64, N - 64 * j) : 0;
                // causal: row qrow keeps the keys t <= qrow of this block
                if (causal && j >= 0) nvalid = max(0, min(nvalid, qrow - 64 * j + 1));
                const uint32_t taddr = tmem + lane_addr + (sb ? kColS1 : kColS0) + 64 * wg;

                // S of this half is read from tensor memory once and kept in registers;
                // keys past the end of the sequence (last block only) are set to INT_MIN,
                // so they drop out of the max and their weight underflows (their P bytes
                // are also cleared below, which covers a zero scale)
                float c = 0.0f, pmax = -INFINITY;
                uint32_t a[32], b[32];
                if (j >= 0) {
                    c = (sq * k_scale[int64_t(bh) * nk + j]) * sm_scale;
                    tc_fence_after();
                    tmem_ld64_wait(taddr, a, b);
                    if (nvalid < 64) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            if (i >= nvalid) a[i] = uint32_t(INT_MIN);
                            if (i + 32 >= nvalid) b[i] = uint32_t(INT_MIN);
                        }
                    }
                    // row max on int32 S (the scale is positive, so max commutes with it)
                    int acc[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) acc[k] = max(int(a[k]), int(b[k]));
#pragma unroll
                    for (int i = 8; i < 32; i += 8)
#pragma unroll
                        for (int k = 0; k < 8; ++k) acc[k] = max(acc[k], max(int(a[i + k]), int(b[i + k])));
                    const int imax = max(max(max(acc[0], acc[1]), max(acc[2], acc[3])),
                                         max(max(acc[4], acc[5]), max(acc[6], acc[7])));
                    // a block with no key left (ragged tail, causal) gives no maximum,
                    // whatever its scale
                    pmax = nvalid > 0 ? i2f(uint32_t(imax)) * c : -INFINITY;
                }
                // S has been read: its buffer may take QK of step gg+2
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarSEmpty + sb));

                float *x = xch + sb * 256;
                x[wg * 128 + row] = pmax;
                named_bar_sync(1 + wq, 64);
                const float other = x[(wg ^ 1) * 128 + row];
                const float mnew = fmaxf(m, fmaxf(pmax, other));

                // P = e4m3(448 * 2^(S*c*log2e - mnew*log2e)) for this half: 64 keys -> 16 words
                uint32_t pw[16];
                if (j >= 0) {
                    const float c2 = c * kLog2e;
                    const float nb = kLog2_448 - mnew * kLog2e;
                    // the masked form only where some row of the warp has a partial block
                    if (__any_sync(0xffffffffu, nvalid < 64))
                        p_half_impl<true>(a, b, c2, nb, nvalid, pw);
                    else
                        p_half_impl<false>(a, b, c2, nb, nvalid, pw);
                } else {
#pragma unroll
                    for (int w = 0; w < 16; ++w) pw[w] = 0u;
                }
                // the P buffer is free once the PV MMA of step gg-2 has completed
                if (gg >= 2 && ok) ok = mbar_wait(bar(kBarPvDone + sb), ((gg >> 1) - 1) & 1, abort_flag);
                ok = __all_sync(0xffffffffu, ok);
                {
                    // 128B-swizzled P tile: 16-byte chunk k of row r at position k ^ (r & 7)
                    uint8_t *prow = smem + kOffP + sb * kPTileBytes + row * 128;
#pragma unroll
                    for (int cidx = 0; cidx < 4; ++cidx) {
                        const int chunk = 4 * wg + cidx;
                        *reinterpret_cast<uint4 *>(prow + ((chunk ^ (row & 7)) << 4)) =
                            make_uint4(pw[4 * cidx], pw[4 * cidx + 1], pw[4 * cidx + 2], pw[4 * cidx + 3]);
                    }
                }
                // rescale O (and its row-sum column) when the running max grew
                if (s > 0) {
                    const bool need = mnew > m;
                    if (__any_sync(0xffffffffu, need)) {
                        const uint32_t pg = gg - 1;
                        if (ok) ok = mbar_wait(bar(kBarPvDone + (pg & 1)), (pg >> 1) & 1, abort_flag);
                        ok = __all_sync(0xffffffffu, ok);
                        if (ok) {
                            tc_fence_after();
                            const float alpha = need ? ex2_approx((m - mnew) * kLog2e) : 1.0f;
                            const uint32_t oa = tmem + lane_addr + kColO;
                            uint32_t r0[32], r1[32];
                            tmem_ld64_wait(oa + 64 * wg, r0, r1);
#pragma unroll
                            for (int i = 0; i < 32; i += 2) {
                                float f0, f1;
                                mul2(f0, f1, __uint_as_float(r0[i]), __uint_as_float(r0[i + 1]), alpha, alpha);
                                r0[i] = __float_as_uint(f0);
                                r0[i + 1] = __float_as_uint(f1);
                                mul2(f0, f1, __uint_as_float(r1[i]), __uint_as_float(r1[i + 1]), alpha, alpha);
                                r1[i] = __float_as_uint(f0);
                                r1[i + 1] = __float_as_uint(f1);
                            }
                            tmem_st32(oa + 64 * wg, r0);
                            tmem_st32(oa + 64 * wg + 32, r1);
                            uint32_t r8[8];
                            tmem_ld8_wait(oa + 128 + 8 * wg, r8);
#pragma unroll
                            for (int i = 0; i < 8; ++i) r8[i] = __float_as_uint(__uint_as_float(r8[i]) * alpha);
                            tmem_st8(oa + 128 + 8 * wg, r8);
                            tmem_st_wait();
                        }
                    }
                }
                m = mnew;
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarPFull + sb));
            }
            // ---- epilogue: O = acc * scale_v / l, bf16, 32 channels at a time
            if (ok) ok = mbar_wait(bar(kBarOFull), otile & 1, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                tc_fence_after();
                const uint32_t base = tmem + lane_addr + kColO;
                uint32_t lbits;
                tmem_ld1_wait(base + 128, lbits);
                const float l = __uint_as_float(lbits);
                const float inv_l = l > 0.0f ? __frcp_rn(l) : 0.0f;  // a row with no kept key gives 0
                const float *svp = v_scale + int64_t(bh) * kD + 64 * wg;
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    uint32_t o[32];
                    tmem_ld32_wait(base + 64 * wg + 32 * h, o);
                    if (qrow < N) {
#pragma unroll
                        for (int cidx = 0; cidx < 4; ++cidx) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int i = 8 * cidx + 2 * e;
                                float y0 = (__uint_as_float(o[i]) * svp[32 * h + i]) * inv_l;
                                float y1 = (__uint_as_float(o[i + 1]) * svp[32 * h + i + 1]) * inv_l;
                                if (arow) {
                                    y0 += arow[32 * h + i];
                                    y1 += arow[32 * h + i + 1];
                                }
                                const __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
                                w[e] = *reinterpret_cast<const uint32_t *>(&h2);
                            }
                            reinterpret_cast<uint4 *>(orow)[4 * h + cidx] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarOEmpty));
            g += n;
            ++otile;
        }
        if (lane == 0 && !ok) { *abort_flag = 1; record_timeout(); }
    }

    // ---- teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMmaQK) tmem_dealloc(tmem, kTmemCols);
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
    // without a keep mask (causal or not): two query tiles per CTA
    if (!a.mask) return launch_attention_pairs(a, st);
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && !attr_set[dev]) {
        e = cudaFuncSetAttribute(attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(kSmemAlloc));
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int ntiles = a.BH * a.nq;
    const int grid = ntiles < sms ? ntiles : sms;
    attn_fwd_kernel<<<grid, kThreads, kSmemAlloc, st>>>(a.tm_q, a.tm_k, a.tm_v, a.q_scale, a.k_scale,
                                                        a.v_scale, a.mask, a.o, a.BH, a.N, a.Npad,
                                                        a.nq, a.nk, a.sm_scale, a.causal, a.addend);
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
