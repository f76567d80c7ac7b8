// sa_sla.cu -- the linear-attention branch of Sparse-Linear Attention (SLA).
//
// Sources: NetEase article on the TurboDiffusion release, attention-acceleration section:
// SLA combines sparse attention with linear attention, and its figure caption splits the
// attention weights into three classes handled at different costs; "AIGC weekend special
// 5.10" section 1.2 Method item (2): SLA, a trainable sparse-linear attention used on top
// of SageAttention.  The pages give no formula for the linear part; the reading built
// here is kernelised linear attention over each row's marginal (class 1) key blocks:
//     O_lin[r] = phi(q_r)^T A_i / (phi(q_r) . z_i),   A_i = sum_{j marginal} H_j,
//     H_j = sum_{t in block j} phi(k_t) v_t^T,          z_i = sum_{j marginal} Z_j,
//     Z_j = sum_{t in block j} phi(k_t),
// projected by a d x d matrix W (out = O_lin W^T, identity if none) and added to the sparse
// quantised attention of the critical (class >= 2) blocks.  phi is the softmax over the
// d features of a row, or elu + 1.
//
// Kernels, over groups of heads whose states fit a bounded workspace:
//   sla_state_mma_kernel  one CTA per (head, 64-key block): H_j (128 x 128) and Z_j as one
//                         TF32 tcgen05 GEMM of phi(K_j)^T with [V_j | 1], phi split into hi +
//                         lo; stored as one 128 x 136 block whose column 128 is Z_j (columns
//                         129-135 zero), so that the apply step gets the normaliser from the
//                         same product as the numerator.
//   sla_marginal_kernel   the 0/1 matrix C[i][j] = (class == 1) in fp32.
//   sla_sum_mma_kernel    A_i = sum_j C[i][j] H_j for every query block: a TF32 tcgen05 GEMM
//                         (K = key blocks) with the states split into hi + lo terms.
//   sla_apply_mma_kernel  one CTA per (head, 128-query block): phi(Q_i) [A_i | z_i] and the
//                         projection as TF32 tcgen05 GEMMs with both operands split into hi +
//                         lo (three products each), the division by the normaliser between
//                         them, fp32 out.  The SLA forward hands that output to the attention
//                         kernel's epilogue, which adds it before the one bf16 rounding.
//   sla_critical_kernel   the keep mask (class >= 2) of the sparse part.
// The hi/lo splits carry about 22 significant bits into every product; accumulation is
// fp32, so the branch stays within fp32-level error of the factorised form.
#include <cstdint>
#include <cuda_bf16.h>

#include "sa_internal.h"
#include "sa_ptx.cuh"

namespace sa {
namespace {

constexpr int kStateCols = 136;                      // H_j columns, then Z_j, then zeros
constexpr int kStateFloats = kD * kStateCols;        // 17408 per key (or query) block

__device__ int g_sla_status;  // 0 = OK, 6 = a bounded wait expired

// A wait bounded by time alone (not by the abort flag): used to let this CTA's own
// copies and MMAs land before it frees its memory.
__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > SA_WAIT_LIMIT_NS) return false;
    return true;
}

// hi keeps the sign, exponent and top 10 mantissa bits (exact in TF32); lo = x - hi exactly.
__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

// ---- the per-block states on the tensor cores
// H_j[a][b] = sum_{t in block j} phi(k_t)[a] [v_t, 1, 0...][b]: M = 128 features a, N = 144
// (the 128 value channels, the ones column that gives Z_j, zeros), K = the block's 64
// tokens; kind::tf32 with phi split into hi + lo (two products; v is bf16, exact in TF32),
// fp32 accumulation in tensor memory.  Both operands are MN-major (feature a, resp. channel
// b, contiguous) in the 128-byte swizzle of 32-byte granules: an atom is 4 token rows of 128
// bytes (32 values), granule g of row t at granule position g ^ (t & 3); atom columns of
// 64 rows are 8 KB apart, 4-row groups 512 bytes apart.
//   all 8 warps  token t = 8 * warp + lane / 4 and atom column c = lane % 4 (32 features
//                or channels): phi over the row's 128 features (the 4 lanes of a token
//                exchange the maximum and the sum), phi hi/lo and v into the tiles; column
//                4 of v holds the ones column.
//   thread 0     the 16 MMAs, committed to one barrier.
//   all 8 warps  the epilogue: warp w reads tensor-memory lanes 32 (w % 4) .., columns
//                0-63 (w < 4) or 64-135 (w >= 4), and stores the state rows.
namespace stm {
constexpr uint32_t kCol = 64 * 128;                                 // one atom column, 8 KB
constexpr uint32_t kOffPhiHi = 0, kOffPhiLo = 4 * kCol, kOffV = 8 * kCol;  // V: 5 columns
constexpr uint32_t kOffBar = kOffV + 5 * kCol;
constexpr uint32_t kSmem = kOffBar + 16 + 1024;
constexpr int kN = 144;
static_assert(kSmem <= 116 * 1024, "two CTAs per SM");
}  // namespace stm

// byte offset of the 8-value granule g of token row t in an MN-major atom column
__device__ __forceinline__ uint32_t mn32_off(int t, int g)
{
    return uint32_t(t >> 2) * 512u + uint32_t(t & 3) * 128u + (uint32_t(g ^ (t & 3)) << 5);
}

// grid (nk, heads), 256 threads, stm::kSmem bytes (two CTAs per SM).
__global__ void __launch_bounds__(256, 2)
    sla_state_mma_kernel(const uint16_t *__restrict__ k, const uint16_t *__restrict__ v, int N, int nk, int phi,
                         float *__restrict__ state)
{
    using namespace stm;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = blockIdx.x, bh = blockIdx.y;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + kOffBar + 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffBar + 12);
    const uint32_t bar = sbase + kOffBar;
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(sbase + kOffBar + 8, 256);

    // ---- operands: token t, atom column c (features / channels 32c .. 32c + 31)
    {
        const int t = 8 * warp + (lane >> 2), c = lane & 3;
        const int64_t tok = int64_t(j) * kKBlk + t;
        const bool valid = tok < N;
        const int64_t row = (int64_t(bh) * N + (valid ? tok : 0)) * kD + 32 * c;
        float x[32];
        uint4 vr[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint4 kw = valid ? __ldg(reinterpret_cast<const uint4 *>(k + row) + u) : make_uint4(0u, 0u, 0u, 0u);
            vr[u] = valid ? __ldg(reinterpret_cast<const uint4 *>(v + row) + u) : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t w4[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                x[8 * u + 2 * e] = __uint_as_float(w4[e] << 16);
                x[8 * u + 2 * e + 1] = __uint_as_float(w4[e] & 0xFFFF0000u);
            }
        }
        if (phi == 0) {
            float m = x[0];
#pragma unroll
            for (int f = 1; f < 32; ++f) m = fmaxf(m, x[f]);
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
            float sum = 0.0f;
#pragma unroll
            for (int f = 0; f < 32; ++f) {
                x[f] = expf(x[f] - m);
                sum += x[f];
            }
            sum += __shfl_xor_sync(0xffffffffu, sum, 1);
            sum += __shfl_xor_sync(0xffffffffu, sum, 2);
#pragma unroll
            for (int f = 0; f < 32; ++f) x[f] = __fdiv_rn(x[f], sum);
        } else {
#pragma unroll
            for (int f = 0; f < 32; ++f) x[f] = x[f] > 0.0f ? x[f] + 1.0f : expf(x[f]);
        }
        if (!valid) {
#pragma unroll
            for (int f = 0; f < 32; ++f) x[f] = 0.0f;  // rows past N take no part
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            float4 h0, h1, l0, l1, v0, v1;
            h0 = make_float4(tf32_hi(x[8 * g]), tf32_hi(x[8 * g + 1]), tf32_hi(x[8 * g + 2]), tf32_hi(x[8 * g + 3]));
            h1 = make_float4(tf32_hi(x[8 * g + 4]), tf32_hi(x[8 * g + 5]), tf32_hi(x[8 * g + 6]), tf32_hi(x[8 * g + 7]));
            l0 = make_float4(x[8 * g] - h0.x, x[8 * g + 1] - h0.y, x[8 * g + 2] - h0.z, x[8 * g + 3] - h0.w);
            l1 = make_float4(x[8 * g + 4] - h1.x, x[8 * g + 5] - h1.y, x[8 * g + 6] - h1.z, x[8 * g + 7] - h1.w);
            const uint32_t w4[4] = {vr[g].x, vr[g].y, vr[g].z, vr[g].w};
            v0 = make_float4(__uint_as_float(w4[0] << 16), __uint_as_float(w4[0] & 0xFFFF0000u),
                             __uint_as_float(w4[1] << 16), __uint_as_float(w4[1] & 0xFFFF0000u));
            v1 = make_float4(__uint_as_float(w4[2] << 16), __uint_as_float(w4[2] & 0xFFFF0000u),
                             __uint_as_float(w4[3] << 16), __uint_as_float(w4[3] & 0xFFFF0000u));
            const uint32_t off = uint32_t(c) * kCol + mn32_off(t, g);
            *reinterpret_cast<float4 *>(smem + kOffPhiHi + off) = h0;
            *reinterpret_cast<float4 *>(smem + kOffPhiHi + off + 16) = h1;
            *reinterpret_cast<float4 *>(smem + kOffPhiLo + off) = l0;
            *reinterpret_cast<float4 *>(smem + kOffPhiLo + off + 16) = l1;
            *reinterpret_cast<float4 *>(smem + kOffV + off) = v0;
            *reinterpret_cast<float4 *>(smem + kOffV + off + 16) = v1;
        }
        // V column 4 (channels 128-159): the ones column 128 (zero past N), then zeros
        const float one = valid ? 1.0f : 0.0f;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            if (g != c) continue;  // the token's 4 lanes write one granule each
            const uint32_t off = 4u * kCol + mn32_off(t, g);
            *reinterpret_cast<float4 *>(smem + kOffV + off) = make_float4(g == 0 ? one : 0.0f, 0.0f, 0.0f, 0.0f);
            *reinterpret_cast<float4 *>(smem + kOffV + off + 16) = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (threadIdx.x == 0) {
        const uint32_t idesc = idesc_tf32_f32(128, kN, true, true);
#pragma unroll
        for (int kk = 0; kk < kKBlk / 8; ++kk) {
            const uint64_t bd = sdesc_mn32(sbase + kOffV + 1024u * kk, kCol, 512);
            mma_tf32(tmem, sdesc_mn32(sbase + kOffPhiHi + 1024u * kk, kCol, 512), bd, idesc, kk > 0);
            mma_tf32(tmem, sdesc_mn32(sbase + kOffPhiLo + 1024u * kk, kCol, 512), bd, idesc, 1);
        }
        tc_commit(bar);
    }
    bool ok = mbar_wait(bar, 0, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
        tc_fence_after();
        const int a = 32 * (warp & 3) + lane;
        const uint32_t ta = tmem + (uint32_t(32 * (warp & 3)) << 16);
        float *out = state + ((int64_t(bh) * nk + j) * kD + a) * kStateCols;
        uint32_t r[32];
        if (warp < 4) {
            for (int c0 = 0; c0 < 64; c0 += 32) {
                tmem_ld32_wait(ta + c0, r);
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4 *>(out + c0 + e) =
                        make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]), __uint_as_float(r[e + 2]),
                                    __uint_as_float(r[e + 3]));
            }
        } else {
            for (int c0 = 64; c0 < 128; c0 += 32) {
                tmem_ld32_wait(ta + c0, r);
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4 *>(out + c0 + e) =
                        make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]), __uint_as_float(r[e + 2]),
                                    __uint_as_float(r[e + 3]));
            }
            uint32_t r8[8];
            tmem_ld8_wait(ta + 128, r8);  // Z_j, then the zero columns 129-135
            *reinterpret_cast<float4 *>(out + 128) =
                make_float4(__uint_as_float(r8[0]), __uint_as_float(r8[1]), __uint_as_float(r8[2]), __uint_as_float(r8[3]));
            *reinterpret_cast<float4 *>(out + 132) =
                make_float4(__uint_as_float(r8[4]), __uint_as_float(r8[5]), __uint_as_float(r8[6]), __uint_as_float(r8[7]));
        }
    } else if (lane == 0) {
        *abort_flag = 1;
        atomicExch(&g_sla_status, 6);
    }
    if (threadIdx.x == 0 && !drain_wait(bar, 0)) atomicExch(&g_sla_status, 6);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// ---- the class-weighted state sum on the tensor cores
// D[n][i] = sum_j H[j][n] C[i][j] with C[i][j] = (classes[i][j] == 1), for one head: the
// GEMM of the states (K = key blocks j, M = the 17408 state entries n) with the 0/1 class
// rows of up to 256 query blocks i (N).  kind::tf32 with fp32 accumulation in tensor
// memory.  C is exact in TF32; the states are split in shared memory into hi (the top 11
// significant bits, exact in TF32) and lo = H - hi (exact in fp32, of which the tensor core
// uses the top 11 bits), and both halves are multiplied, so every product carries about 22
// significant bits of H: far below fp32 accumulation error relative to the 1e-4 bound.
//
// One CTA per (query-block tile, 128 state entries, head), query-block tiles fastest so
// that the CTAs reading one chunk of states run together and share it through L2.
//   warps 0-3  per k-block of 32 key blocks: split the landed state tile into hi and lo;
//              then the epilogue (warp w owns tensor-memory lanes 32w .. 32w+31, i.e. state
//              entries n0 + 32w + lane).
//   warp 4     TMA producer: the state tile, 4 boxes of 32 entries x 32 key blocks, in the
//              MN-major layout with 32-byte swizzle granules that TF32 operands need; and
//              the tile of C (fp32 0/1, written once per call by sla_marginal_kernel),
//              K-major with the usual 128-byte swizzle.
//   warp 5     MMA issuer: per k-block, 4 steps of K = 8, each hi and lo.
namespace summ {
constexpr int kM = 128;        // state entries per tile (MMA M)
constexpr int kKb = 32;        // key blocks per k-block: 128 bytes of fp32
constexpr int kStages = 3;
constexpr int kMaxNT = 256;    // query blocks per tile (MMA N)
constexpr int kThreads = 192;
constexpr int kWarpTma = 4, kWarpMma = 5;
constexpr uint32_t kABytes = kM * kKb * 4;      // 16 KB: 4 atoms of 32 entries x 32 rows
constexpr uint32_t kBBytes = kMaxNT * kKb * 4;  // 32 KB
constexpr uint32_t kOffAhi = 0;
constexpr uint32_t kOffAlo = kOffAhi + kStages * kABytes;
constexpr uint32_t kOffB = kOffAlo + kStages * kABytes;
constexpr uint32_t kOffBar = kOffB + kStages * kBBytes;
constexpr int kBarFull = 0, kBarEmpty = kStages, kBarReady = 2 * kStages, kBarAcc = 3 * kStages;
constexpr uint32_t kOffMisc = kOffBar + 8 * (3 * kStages + 1);
constexpr uint32_t kSmem = kOffMisc + 16 + 1024;  // + slack for the 1024-byte alignment
static_assert(kOffB % 1024 == 0 && kABytes % 1024 == 0 && kBBytes % 1024 == 0, "swizzle atoms");
static_assert(kSmem <= 232448, "shared memory");
}  // namespace summ

// grid (ceil(nq / nt), 17408 / 128, BH), summ::kThreads threads, summ::kSmem bytes.
// nt: query blocks per tile, a multiple of 16 in [16, 256].
__global__ void __launch_bounds__(summ::kThreads, 1)
    sla_sum_mma_kernel(const __grid_constant__ CUtensorMap tm_state, const __grid_constant__ CUtensorMap tm_c,
                       int nq, int nk, int nt, float *__restrict__ sums)
{
    using namespace summ;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i0 = blockIdx.x * nt, n0 = blockIdx.y * kM, bh = blockIdx.z;
    const int nkb = (nk + kKb - 1) / kKb;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
    auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * uint32_t(i); };
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(kBarFull + s), 1);
            mbar_init(bar(kBarEmpty + s), 1);
            mbar_init(bar(kBarReady + s), 4);
        }
        mbar_init(bar(kBarAcc), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) tmem_alloc(sbase + kOffMisc, kMaxNT);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kWarpTma) {
        if (lane == 0) {
            prefetch_tmap(&tm_state);
            prefetch_tmap(&tm_c);
            bool ok = true;
            int kb = 0;
            for (; kb < nkb; ++kb) {
                const int s = kb % kStages;
                if (kb >= kStages) ok = mbar_wait(bar(kBarEmpty + s), ((kb / kStages) & 1) ^ 1, abort_flag);
                if (!ok) break;
                const uint32_t dst = sbase + kOffAhi + uint32_t(s) * kABytes;
                mbar_arrive_expect_tx(bar(kBarFull + s), kABytes + uint32_t(nt) * 128u);
#pragma unroll
                for (int c = 0; c < kM / 32; ++c)
                    tma_load_3d(dst + 4096u * c, &tm_state, bar(kBarFull + s), n0 + 32 * c, kb * kKb, bh);
                tma_load_3d(sbase + kOffB + uint32_t(s) * kBBytes, &tm_c, bar(kBarFull + s), kb * kKb, i0, bh);
            }
            // the last loads issued have landed before the CTA's memory is released
            bool drained = true;
            for (int d = kb > kStages ? kb - kStages : 0; d < kb; ++d)
                drained = drain_wait(bar(kBarFull + d % kStages), (d / kStages) & 1) && drained;
            if (!ok || !drained) {
                *abort_flag = 1;
                atomicExch(&g_sla_status, 6);
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            const uint32_t idesc = idesc_tf32_f32(kM, nt, true, false);
            bool ok = true;
            int kb = 0;
            for (; kb < nkb; ++kb) {
                const int s = kb % kStages;
                ok = mbar_wait(bar(kBarReady + s), (kb / kStages) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t ahi = sbase + kOffAhi + uint32_t(s) * kABytes;
                const uint32_t alo = sbase + kOffAlo + uint32_t(s) * kABytes;
                const uint32_t bt = sbase + kOffB + uint32_t(s) * kBBytes;
#pragma unroll
                for (int kk = 0; kk < kKb / 8; ++kk) {
                    // A: rows 8kk .. 8kk+7 (two 4-row atoms, 512 bytes apart) of each column
                    // of 32 entries, the columns 4096 bytes apart; B: 32 bytes of K per step
                    const uint64_t bdesc = sdesc(bt + 32u * kk, 1024, SWZ_128B);
                    mma_tf32(tmem, sdesc_mn32(ahi + 1024u * kk, 4096, 512), bdesc, idesc, (kb | kk) != 0);
                    mma_tf32(tmem, sdesc_mn32(alo + 1024u * kk, 4096, 512), bdesc, idesc, 1);
                }
                tc_commit(bar(kBarEmpty + s));
            }
            if (ok) tc_commit(bar(kBarAcc));
            // this thread's MMAs have completed before the tensor memory is freed
            if (kb > 0 && !drain_wait(bar(kBarEmpty + (kb - 1) % kStages), ((kb - 1) / kStages) & 1)) ok = false;
            if (!ok) {
                *abort_flag = 1;
                atomicExch(&g_sla_status, 6);
            }
        }
    } else {
        // ---- warps 0-3: the hi/lo split, then the epilogue.  The full barrier of a stage
        // completes only after the producer's wait for that stage's previous MMAs, so the
        // lo tile is free to overwrite once the loads have landed.
        bool ok = true;
        for (int kb = 0; kb < nkb && ok; ++kb) {
            const int s = kb % kStages;
            ok = mbar_wait(bar(kBarFull + s), (kb / kStages) & 1, abort_flag);
            if (!ok) break;
            // hi keeps the sign, exponent and top 10 mantissa bits; lo = H - hi exactly
            float4 *ahi = reinterpret_cast<float4 *>(smem + kOffAhi + uint32_t(s) * kABytes);
            float4 *alo = reinterpret_cast<float4 *>(smem + kOffAlo + uint32_t(s) * kABytes);
#pragma unroll
            for (int u = 0; u < int(kABytes / 16) / 128; ++u) {
                const int e = threadIdx.x + 128 * u;
                const float4 x = ahi[e];
                float4 h;
                h.x = __uint_as_float(__float_as_uint(x.x) & 0xFFFFE000u);
                h.y = __uint_as_float(__float_as_uint(x.y) & 0xFFFFE000u);
                h.z = __uint_as_float(__float_as_uint(x.z) & 0xFFFFE000u);
                h.w = __uint_as_float(__float_as_uint(x.w) & 0xFFFFE000u);
                ahi[e] = h;
                alo[e] = make_float4(x.x - h.x, x.y - h.y, x.z - h.z, x.w - h.w);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarReady + s));
        }
        if (ok) ok = mbar_wait(bar(kBarAcc), 0, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc_fence_after();
            const int n = n0 + 32 * warp + lane;
            float *dst = sums + int64_t(bh) * nq * int64_t(kStateFloats) + n;
            for (int c0 = 0; c0 < nt; c0 += 32) {
                uint32_t r[32];
                tmem_ld32_wait(tmem + (uint32_t(32 * warp) << 16) + uint32_t(c0), r);
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int i = i0 + c0 + c;
                    if (c0 + c < nt && i < nq) dst[int64_t(i) * kStateFloats] = __uint_as_float(r[c]);
                }
            }
        } else if (lane == 0) {
            *abort_flag = 1;
            atomicExch(&g_sla_status, 6);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) tmem_dealloc(tmem, kMaxNT);
}

// C of the state sum: cm[bh][i][j] = (classes[bh][i][j] == 1) as fp32, for j < nk4 (a
// multiple of 4, so that rows are 16-byte aligned for TMA); zero for j >= nk.
__global__ void sla_marginal_kernel(const uint8_t *__restrict__ classes, int64_t rows, int nk, int nk4,
                                    float *__restrict__ cm)
{
    const int64_t n = rows * nk4;
    for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < n; e += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = e / nk4;
        const int j = int(e - r * nk4);
        cm[e] = (j < nk && classes[r * nk + j] == 1) ? 1.0f : 0.0f;
    }
}

// ---- the apply step on the tensor cores
// For one (head, 128-query block i):
//   GEMM1  D1[r][b] = sum_a phi(q_r)[a] A_i[a][b]   (M = 128 rows, N = 144: the 128 value
//          columns, the normaliser column 128 and zeros, K = 128 features)
//   O_lin[r][f] = D1[r][f] / D1[r][128]  (0 when the normaliser is not positive)
//   GEMM2  out[r][c] = sum_f O_lin[r][f] W[c][f]     (M = 128, N = 128, K = 128; skipped
//          without a projection, when out = O_lin)
// Both are kind::tf32 with both operands split into hi + lo and three products (hi*hi,
// hi*lo, lo*hi), about 22 significant bits per product, fp32 accumulation in tensor memory.
//   warps 0-3  thread r owns row r: phi(q_r) into the phi tiles, then O_lin from D1 into the
//              O tiles, then out from D2 (tensor-memory lanes of warp w: 32w .. 32w+31).
//   warps 4-7  split the A_i halves (TMA) into hi/lo; load W halves and split them.
//   warp 8     lane 0 issues the TMA loads and the MMAs.
// Shared memory: region R0 holds phi (hi, lo: 4 K-atoms of 128 rows x 128 bytes each) for
// GEMM1 and then, per K half of GEMM2, the O and W tiles (hi, lo: 2 K-atoms each); region R1
// holds one K half (64 features) of A_i (hi, lo), MN-major with 32-byte swizzle granules:
// 5 columns of 32 entries x 64 rows.
namespace appm {
constexpr int kThreads = 288;
constexpr int kWarpIssue = 8;
constexpr uint32_t kAtom = 128 * 128;            // 128 rows x 128 bytes, K-major
constexpr uint32_t kOffPhiHi = 0, kOffPhiLo = 4 * kAtom;
constexpr uint32_t kOffOHi = 0, kOffOLo = 2 * kAtom, kOffWHi = 4 * kAtom, kOffWLo = 6 * kAtom;
constexpr uint32_t kAColBytes = 64 * 128;         // one column of 32 entries, 64 rows
constexpr uint32_t kAHalfBytes = 5 * kAColBytes;  // N = 144 needs 5 columns (160 entries)
constexpr uint32_t kOffAHi = 8 * kAtom, kOffALo = kOffAHi + kAHalfBytes;
constexpr uint32_t kOffBar = kOffALo + kAHalfBytes;
enum { kBarFullA, kBarReadyPhi, kBarReadyA, kBarFreeA, kBarAcc1, kBarReadyO, kBarReadyW, kBarFreeR0, kBarAcc2,
       kNumBars };
constexpr uint32_t kOffMisc = kOffBar + 8 * kNumBars;
constexpr uint32_t kSmem = kOffMisc + 16 + 1024;
constexpr uint32_t kColAcc1 = 0, kColAcc2 = 256;  // D1: 144 columns; D2: 128 columns
static_assert(kOffAHi % 1024 == 0 && kSmem <= 232448, "apply shared memory");
}  // namespace appm

// Writes 4 consecutive K values (chunk c of 8 in a 128-byte row) of row r of a K-major,
// 128-byte swizzled atom, as hi and lo.
__device__ __forceinline__ void put_hilo(uint8_t *hi, uint8_t *lo, int r, int c, float4 x)
{
    const float4 h = make_float4(tf32_hi(x.x), tf32_hi(x.y), tf32_hi(x.z), tf32_hi(x.w));
    const uint32_t off = uint32_t(r) * 128u + (uint32_t(c ^ (r & 7)) << 4);
    *reinterpret_cast<float4 *>(hi + off) = h;
    *reinterpret_cast<float4 *>(lo + off) = make_float4(x.x - h.x, x.y - h.y, x.z - h.z, x.w - h.w);
}

// grid (nq, heads), appm::kThreads threads, appm::kSmem bytes.  tm_sums: map of the summed
// states as rows of 136 floats (row (bh * nq + i) * 128 + a; third dimension 1), box {32, 64}.
__global__ void __launch_bounds__(appm::kThreads, 1)
    sla_apply_mma_kernel(const __grid_constant__ CUtensorMap tm_sums, const uint16_t *__restrict__ q,
                         const float *__restrict__ proj, int N, int nq, int phi, float *__restrict__ out)
{
    using namespace appm;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x, bh = blockIdx.y;
    const bool has_proj = proj != nullptr;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
    auto bar = [&](int b) -> uint32_t { return sbase + kOffBar + 8u * uint32_t(b); };
    if (threadIdx.x == 0) {
        for (int b = 0; b < kNumBars; ++b)
            mbar_init(bar(b), (b == kBarReadyPhi || b == kBarReadyA || b == kBarReadyO || b == kBarReadyW) ? 4 : 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kWarpIssue) tmem_alloc(sbase + kOffMisc, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int64_t arow = (int64_t(bh) * nq + i) * 128;  // first row of A_i in the summed states

    if (warp == kWarpIssue) {
        if (lane == 0) {
            prefetch_tmap(&tm_sums);
            bool ok = true;
            int loads = 0;  // A halves issued
            const uint32_t id1 = idesc_tf32_f32(128, 144, false, true), id2 = idesc_tf32_f32(128, 128, false, false);
            for (int h = 0; h < 2 && ok; ++h) {
                if (h == 1) ok = mbar_wait(bar(kBarFreeA), 0, abort_flag);  // half 0's MMAs done
                if (!ok) break;
                mbar_arrive_expect_tx(bar(kBarFullA), kAHalfBytes);
#pragma unroll
                for (int c = 0; c < 5; ++c)
                    tma_load_3d(sbase + kOffAHi + uint32_t(c) * kAColBytes, &tm_sums, bar(kBarFullA), 32 * c,
                                int(arow + 64 * h), 0);
                ++loads;
                ok = (h > 0 || mbar_wait(bar(kBarReadyPhi), 0, abort_flag)) && mbar_wait(bar(kBarReadyA), h, abort_flag);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    // phi: K-atom 2h + kk/4, 32 bytes per step; A_i: 8 rows (two 4-row atoms)
                    const uint32_t pa = uint32_t(2 * h + kk / 4) * kAtom + 32u * uint32_t(kk & 3);
                    const uint64_t ahi = sdesc(sbase + kOffPhiHi + pa, 1024, SWZ_128B);
                    const uint64_t alo = sdesc(sbase + kOffPhiLo + pa, 1024, SWZ_128B);
                    const uint64_t bhi = sdesc_mn32(sbase + kOffAHi + 1024u * kk, kAColBytes, 512);
                    const uint64_t blo = sdesc_mn32(sbase + kOffALo + 1024u * kk, kAColBytes, 512);
                    mma_tf32(tmem + kColAcc1, ahi, bhi, id1, (h | kk) != 0);
                    mma_tf32(tmem + kColAcc1, ahi, blo, id1, 1);
                    mma_tf32(tmem + kColAcc1, alo, bhi, id1, 1);
                }
                tc_commit(bar(h == 0 ? kBarFreeA : kBarAcc1));
            }
            for (int h = 0; h < 2 && ok && has_proj; ++h) {
                ok = mbar_wait(bar(kBarReadyO), h, abort_flag) && mbar_wait(bar(kBarReadyW), h, abort_flag);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t pa = uint32_t(kk / 4) * kAtom + 32u * uint32_t(kk & 3);
                    const uint64_t ahi = sdesc(sbase + kOffOHi + pa, 1024, SWZ_128B);
                    const uint64_t alo = sdesc(sbase + kOffOLo + pa, 1024, SWZ_128B);
                    const uint64_t bhi = sdesc(sbase + kOffWHi + pa, 1024, SWZ_128B);
                    const uint64_t blo = sdesc(sbase + kOffWLo + pa, 1024, SWZ_128B);
                    mma_tf32(tmem + kColAcc2, ahi, bhi, id2, (h | kk) != 0);
                    mma_tf32(tmem + kColAcc2, ahi, blo, id2, 1);
                    mma_tf32(tmem + kColAcc2, alo, bhi, id2, 1);
                }
                tc_commit(bar(h == 0 ? kBarFreeR0 : kBarAcc2));
            }
            // the loads and MMAs issued have completed before the CTA's memory is released
            bool drained = loads == 0 || drain_wait(bar(kBarFullA), uint32_t(loads - 1) & 1u);
            if (ok) drained = drain_wait(bar(has_proj ? kBarAcc2 : kBarAcc1), 0) && drained;
            if (!ok || !drained) {
                *abort_flag = 1;
                atomicExch(&g_sla_status, 6);
            }
        }
    } else if (warp >= 4) {
        // ---- operand warps: A_i halves, then W halves
        const int t = threadIdx.x - 128;
        bool ok = true;
        for (int h = 0; h < 2 && ok; ++h) {
            ok = mbar_wait(bar(kBarFullA), h, abort_flag);
            if (!ok) break;
            float4 *ahi = reinterpret_cast<float4 *>(smem + kOffAHi), *alo = reinterpret_cast<float4 *>(smem + kOffALo);
            for (int e = t; e < int(kAHalfBytes / 16); e += 128) {
                const float4 x = ahi[e];
                const float4 hh = make_float4(tf32_hi(x.x), tf32_hi(x.y), tf32_hi(x.z), tf32_hi(x.w));
                ahi[e] = hh;
                alo[e] = make_float4(x.x - hh.x, x.y - hh.y, x.z - hh.z, x.w - hh.w);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarReadyA));
        }
        for (int h = 0; h < 2 && ok && has_proj; ++h) {
            // R0 is free once GEMM1 (half 0) or the first half of GEMM2 (half 1) is done
            ok = mbar_wait(bar(h == 0 ? kBarAcc1 : kBarFreeR0), 0, abort_flag);
            if (!ok) break;
            // row c = t of W, features 64h .. 64h+63
            const float4 *wr = reinterpret_cast<const float4 *>(proj + int64_t(t) * kD + 64 * h);
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    put_hilo(smem + kOffWHi + a * kAtom, smem + kOffWLo + a * kAtom, t, c, __ldg(wr + 8 * a + c));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarReadyW));
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            atomicExch(&g_sla_status, 6);
        }
    } else {
        // ---- row warps: thread r = row r of the query block.  The row of q stays packed
        // (bf16 pairs) in registers; values are unpacked 4 features (one 16-byte chunk of the
        // phi tile) at a time.
        const int r = threadIdx.x;
        const int64_t tok = int64_t(i) * kQBlk + r;
        uint4 qp[kD / 8];
        {
            const uint4 *src = reinterpret_cast<const uint4 *>(q + (int64_t(bh) * N + (tok < N ? tok : 0)) * kD);
#pragma unroll
            for (int u = 0; u < kD / 8; ++u) qp[u] = tok < N ? __ldg(src + u) : make_uint4(0u, 0u, 0u, 0u);
        }
        auto unpack4 = [&](int c4) -> float4 {  // features 4 c4 .. 4 c4 + 3
            const uint4 &w = qp[c4 >> 1];
            const uint32_t lo = (c4 & 1) ? w.z : w.x, hi = (c4 & 1) ? w.w : w.y;
            return make_float4(__uint_as_float(lo << 16), __uint_as_float(lo & 0xFFFF0000u),
                               __uint_as_float(hi << 16), __uint_as_float(hi & 0xFFFF0000u));
        };
        // phi = softmax over the features: exp(x - max) / sum.  The 1/sum factor multiplies
        // the numerator and the normaliser of O_lin alike, so it is not applied here (the
        // ratio is the same); elu + 1 has no such factor.
        float m = 0.0f;
        if (phi == 0) {
            m = -INFINITY;
#pragma unroll
            for (int c4 = 0; c4 < kD / 4; ++c4) {
                const float4 x = unpack4(c4);
                m = fmaxf(m, fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w)));
            }
        }
        // exponentials as ex2.approx of the argument times log2(e) (a few ulp, far inside
        // the branch's 1e-4 bound)
        constexpr float kL2e = 1.4426950408889634f;
        auto phi1 = [&](float v) -> float {
            return phi == 0 ? ex2_approx((v - m) * kL2e) : (v > 0.0f ? v + 1.0f : ex2_approx(v * kL2e));
        };
#pragma unroll
        for (int c4 = 0; c4 < kD / 4; ++c4) {
            float4 x = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (tok < N) {
                x = unpack4(c4);
                x = make_float4(phi1(x.x), phi1(x.y), phi1(x.z), phi1(x.w));
            }
            put_hilo(smem + kOffPhiHi + (c4 >> 3) * kAtom, smem + kOffPhiLo + (c4 >> 3) * kAtom, r, c4 & 7, x);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarReadyPhi));
        // O_lin = D1 / normaliser
        bool ok = mbar_wait(bar(kBarAcc1), 0, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        const uint32_t lrow = uint32_t(32 * warp) << 16;
        float4 *o = reinterpret_cast<float4 *>(out + (int64_t(bh) * N + tok) * kD);
        if (ok) {
            tc_fence_after();
            uint32_t dn;
            tmem_ld1_wait(tmem + lrow + kColAcc1 + 128, dn);
            const float den = __uint_as_float(dn);
            const float rden = den > 0.0f ? __frcp_rn(den) : 0.0f;  // 0: no marginal key, O_lin = 0
            // 32 columns of O_lin (chunk cb) -> hi/lo O tile (GEMM2) or the output
            for (int cb = 0; cb < 4; ++cb) {
                if (has_proj && (cb & 1) == 0) {
                    // a K half of GEMM2 starts: its O tiles reuse R0 once the MMAs before are done
                    if (cb == 2) ok = mbar_wait(bar(kBarFreeR0), 0, abort_flag);
                    if (!ok) break;
                }
                uint32_t v[32];
                tmem_ld32_wait(tmem + lrow + kColAcc1 + 32 * cb, v);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float4 x = make_float4(__uint_as_float(v[4 * c]) * rden, __uint_as_float(v[4 * c + 1]) * rden,
                                                 __uint_as_float(v[4 * c + 2]) * rden,
                                                 __uint_as_float(v[4 * c + 3]) * rden);
                    if (has_proj)
                        put_hilo(smem + kOffOHi + (cb & 1) * kAtom, smem + kOffOLo + (cb & 1) * kAtom, r, c, x);
                    else if (tok < N)
                        o[8 * cb + c] = x;
                }
                if (has_proj && (cb & 1) == 1) {
                    tc_fence_before();
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(kBarReadyO));
                }
            }
            ok = __all_sync(0xffffffffu, ok);
            if (ok && has_proj) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar(kBarAcc2), 0, abort_flag));
                if (ok) {
                    tc_fence_after();
                    for (int cb = 0; cb < 4; ++cb) {
                        uint32_t v[32];
                        tmem_ld32_wait(tmem + lrow + kColAcc2 + 32 * cb, v);
                        if (tok < N) {
#pragma unroll
                            for (int c = 0; c < 8; ++c)
                                o[8 * cb + c] = make_float4(__uint_as_float(v[4 * c]), __uint_as_float(v[4 * c + 1]),
                                                            __uint_as_float(v[4 * c + 2]), __uint_as_float(v[4 * c + 3]));
                        }
                    }
                }
            }
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            atomicExch(&g_sla_status, 6);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpIssue) tmem_dealloc(tmem, 512);
}

__global__ void sla_critical_kernel(const uint8_t *__restrict__ classes, int64_t n, uint8_t *__restrict__ keep)
{
    for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < n; e += int64_t(gridDim.x) * blockDim.x)
        keep[e] = classes[e] >= 2 ? 1 : 0;
}

}  // namespace

// The branch runs over groups of heads whose states and summed states together take at
// most kChunkBudget bytes (at least one head per group), so its workspace does not grow
// with the number of heads.
constexpr size_t kChunkBudget = size_t(1) << 30;

static size_t head_state_bytes(const Shape &s) { return size_t(s.nk()) * kStateFloats * sizeof(float); }
static size_t head_sum_bytes(const Shape &s) { return size_t(s.nq()) * kStateFloats * sizeof(float); }
static int nk4_of(const Shape &s) { return int((s.nk() + 3) / 4 * 4); }
static size_t head_c_bytes(const Shape &s) { return size_t(s.nq()) * size_t(nk4_of(s)) * sizeof(float); }
static size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

static int64_t chunk_heads(const Shape &s)
{
    const int64_t per = int64_t(head_state_bytes(s) + head_sum_bytes(s) + head_c_bytes(s));
    int64_t g = int64_t(kChunkBudget) / per;
    if (g > 65535) g = 65535;  // the group is a grid dimension of every launch
    return g < 1 ? 1 : (g > s.BH() ? s.BH() : g);
}

// workspace: [states | summed states | C], each for chunk_heads(s) heads
size_t sla_workspace_bytes(const Shape &s)
{
    const size_t g = size_t(chunk_heads(s));
    return up256(g * head_state_bytes(s)) + up256(g * head_sum_bytes(s)) + g * head_c_bytes(s);
}

cudaError_t launch_sla_linear(const void *q, const void *k, const void *v, const uint8_t *classes, const Shape &s,
                              int phi, const float *proj, void *workspace, float *out, cudaStream_t st)
{
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        if ((e = cudaFuncSetAttribute(sla_state_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(stm::kSmem))) != cudaSuccess ||
            (e = cudaFuncSetAttribute(sla_sum_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(summ::kSmem))) != cudaSuccess ||
            (e = cudaFuncSetAttribute(sla_apply_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(appm::kSmem))) != cudaSuccess)
            return e;
        attr_set[dev] = true;
    }
    const int nq = int(s.nq()), nk = int(s.nk()), N = int(s.N), nk4 = nk4_of(s);
    const int64_t G = chunk_heads(s), tok = int64_t(N) * kD;
    uint8_t *w = static_cast<uint8_t *>(workspace);
    float *state = reinterpret_cast<float *>(w);
    float *sums = reinterpret_cast<float *>(w + up256(size_t(G) * head_state_bytes(s)));
    float *cm = reinterpret_cast<float *>(w + up256(size_t(G) * head_state_bytes(s)) +
                                          up256(size_t(G) * head_sum_bytes(s)));
    // query-block tiles of nt <= 256 (a multiple of 16), as even as the count allows
    const int ntiles = (nq + summ::kMaxNT - 1) / summ::kMaxNT;
    const int nt = ((nq + ntiles - 1) / ntiles + 15) / 16 * 16;
    for (int64_t h0 = 0; h0 < s.BH(); h0 += G) {
        const int64_t g = s.BH() - h0 < G ? s.BH() - h0 : G;
        sla_state_mma_kernel<<<dim3(unsigned(nk), unsigned(g)), 256, stm::kSmem, st>>>(
            static_cast<const uint16_t *>(k) + h0 * tok, static_cast<const uint16_t *>(v) + h0 * tok, N, nk, phi,
            state);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int64_t crows = g * nq, celems = crows * nk4;
        const int cblocks = int(celems / 1024 + 1 < 4096 ? celems / 1024 + 1 : 4096);
        sla_marginal_kernel<<<cblocks, 256, 0, st>>>(classes + h0 * nq * int64_t(nk), crows, nk, nk4, cm);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        CUtensorMap tm_state, tm_c;
        if (!encode_tmap_3d_f32(&tm_state, state, kStateFloats, uint64_t(nk), uint64_t(g),
                                uint64_t(kStateFloats) * sizeof(float), head_state_bytes(s), 32, summ::kKb,
                                CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B) ||
            !encode_tmap_3d_f32(&tm_c, cm, uint64_t(nk4), uint64_t(nq), uint64_t(g), uint64_t(nk4) * sizeof(float),
                                head_c_bytes(s), summ::kKb, uint32_t(nt), CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        sla_sum_mma_kernel<<<dim3(unsigned((nq + nt - 1) / nt), unsigned(kStateFloats / summ::kM), unsigned(g)),
                             summ::kThreads, summ::kSmem, st>>>(tm_state, tm_c, nq, nk, nt, sums);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        CUtensorMap tm_sums;
        const uint64_t srows = uint64_t(g) * uint64_t(nq) * kD;
        if (!encode_tmap_3d_f32(&tm_sums, sums, kStateCols, srows, 1, kStateCols * sizeof(float),
                                srows * kStateCols * sizeof(float), 32, 64, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B))
            return cudaErrorInvalidValue;
        sla_apply_mma_kernel<<<dim3(unsigned(nq), unsigned(g)), appm::kThreads, appm::kSmem, st>>>(
            tm_sums, static_cast<const uint16_t *>(q) + h0 * tok, proj, N, nq, phi, out + h0 * tok);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t read_and_clear_sla_status(int *status)
{
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(status, g_sla_status, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_sla_status, &zero, sizeof(int));
}

cudaError_t launch_sla_critical(const uint8_t *classes, int64_t n, uint8_t *keep, cudaStream_t st)
{
    const int blocks = int(n / 1024 + 1 < 4096 ? n / 1024 + 1 : 4096);
    sla_critical_kernel<<<blocks, 256, 0, st>>>(classes, n, keep);
    return cudaGetLastError();
}

}  // namespace sa
