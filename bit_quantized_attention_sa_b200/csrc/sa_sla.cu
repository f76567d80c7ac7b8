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
// Kernels (fp32 throughout):
//   sla_state_kernel      one CTA per (head, 64-key block): H_j (128 x 128) and Z_j, stored
//                         as one 128 x 136 block whose column 128 is Z_j (columns 129-135
//                         zero), so that the apply step gets the normaliser from the same
//                         product as the numerator.
//   sla_state_sum_kernel  A_i = sum of the marginal blocks' states, for 16 query blocks at a
//                         time (each H_j chunk is read once for all 16 rows of classes).
//   sla_apply_kernel      one CTA per (head, 128-query block): phi(Q_i) A_i in shared memory,
//                         division by the normaliser column, the projection, and the fp32
//                         store.  The SLA forward hands that fp32 output to the attention
//                         kernel's epilogue, which adds it before the one bf16 rounding.
//   sla_critical_kernel   the keep mask (class >= 2) of the sparse part.
#include <cstdint>
#include <cuda_bf16.h>

#include "sa_internal.h"
#include "sa_ptx.cuh"

namespace sa {
namespace {

constexpr int kStateCols = 136;                      // H_j columns, then Z_j, then zeros
constexpr int kStateFloats = kD * kStateCols;        // 17408 per key (or query) block

// phi of one 128-feature row held by a warp, 4 features per lane (features 4 lane .. +3).
__device__ __forceinline__ void phi_row_warp(float (&x)[4], int phi)
{
    if (phi == 0) {
        float m = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float s = 0.0f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[e] = expf(x[e] - m);
            s += x[e];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = __fdiv_rn(x[e], s);
    } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = x[e] > 0.0f ? x[e] + 1.0f : expf(x[e]);
    }
}

// Loads row t of a head (bf16, 128 features) into 4 floats per lane; zeros past N.
__device__ __forceinline__ void load_row4(const uint16_t *base, int64_t t, int64_t N, int lane, float (&x)[4])
{
    if (t < N) {
        const uint2 w = *reinterpret_cast<const uint2 *>(base + t * kD + 4 * lane);
        x[0] = __uint_as_float(w.x << 16);
        x[1] = __uint_as_float(w.x & 0xFFFF0000u);
        x[2] = __uint_as_float(w.y << 16);
        x[3] = __uint_as_float(w.y & 0xFFFF0000u);
    } else {
        x[0] = x[1] = x[2] = x[3] = 0.0f;
    }
}

// grid (nk, BH), 256 threads, dynamic shared memory 2 x 64 x 128 floats.
__global__ void __launch_bounds__(256)
    sla_state_kernel(const uint16_t *__restrict__ k, const uint16_t *__restrict__ v, int N, int nk, int phi,
                     float *__restrict__ state)
{
    extern __shared__ __align__(16) float sm[];
    float *pk = sm;               // [64][128] phi(k) rows of the block (zero past N)
    float *vv = sm + kKBlk * kD;  // [64][128] v rows
    const int64_t bh = blockIdx.y;
    const int j = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint16_t *kh = k + bh * int64_t(N) * kD, *vh = v + bh * int64_t(N) * kD;
    for (int t = warp; t < kKBlk; t += 8) {
        const int64_t tok = int64_t(j) * kKBlk + t;
        float x[4], y[4];
        load_row4(kh, tok, N, lane, x);
        load_row4(vh, tok, N, lane, y);
        if (tok < N) phi_row_warp(x, phi);
        *reinterpret_cast<float4 *>(pk + t * kD + 4 * lane) = make_float4(x[0], x[1], x[2], x[3]);
        *reinterpret_cast<float4 *>(vv + t * kD + 4 * lane) = make_float4(y[0], y[1], y[2], y[3]);
    }
    __syncthreads();
    // H[a][c] for a in [8 ty, 8 ty + 8), c in [8 tx, 8 tx + 8), over the block's 64 tokens
    const int ty = tid >> 4, tx = tid & 15;
    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[a][c] = 0.0f;
    for (int t = 0; t < kKBlk; ++t) {
        const float4 p0 = *reinterpret_cast<const float4 *>(pk + t * kD + 8 * ty);
        const float4 p1 = *reinterpret_cast<const float4 *>(pk + t * kD + 8 * ty + 4);
        const float4 v0 = *reinterpret_cast<const float4 *>(vv + t * kD + 8 * tx);
        const float4 v1 = *reinterpret_cast<const float4 *>(vv + t * kD + 8 * tx + 4);
        const float pa[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
        const float vc[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[a][c] = fmaf(pa[a], vc[c], acc[a][c]);
    }
    float *out = state + (bh * nk + j) * int64_t(kStateFloats);
#pragma unroll
    for (int a = 0; a < 8; ++a) {
        float *row = out + (8 * ty + a) * kStateCols + 8 * tx;
        *reinterpret_cast<float4 *>(row) = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
        *reinterpret_cast<float4 *>(row + 4) = make_float4(acc[a][4], acc[a][5], acc[a][6], acc[a][7]);
    }
    if (tid < kD) {
        // column 128: Z_j[a] = sum over the block's tokens of phi(k_t)[a]; columns 129-135 zero
        float z = 0.0f;
        for (int t = 0; t < kKBlk; ++t) z += pk[t * kD + tid];
        float *row = out + tid * kStateCols + kD;
        *reinterpret_cast<float4 *>(row) = make_float4(z, 0.0f, 0.0f, 0.0f);
        *reinterpret_cast<float4 *>(row + 4) = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
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
            const uint32_t idesc = idesc_tf32_f32_amn(kM, nt);
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

// Shared memory of the apply kernel (floats): phi(Q) [128][132] (row-padded), then the
// summed state [128][136]; W^T [128][132] reuses the phi(Q) region and O_lin [128][132]
// the state region once they are consumed.
constexpr int kApplyLd = 132;
constexpr int kApplyPhi = 0, kApplyState = kD * kApplyLd, kApplyDen = kApplyState + kD * kStateCols;
constexpr int kApplySmemFloats = kApplyDen + kD;
constexpr size_t kApplySmemBytes = size_t(kApplySmemFloats) * sizeof(float);

// grid (nq, BH), 256 threads.  out: fp32 [BH, N, d].  proj: fp32 [d][d] or null (identity).
__global__ void __launch_bounds__(256)
    sla_apply_kernel(const uint16_t *__restrict__ q, const float *__restrict__ sums, const float *__restrict__ proj,
                     int N, int nq, int phi, float *__restrict__ out)
{
    extern __shared__ __align__(16) float sm[];
    float *pq = sm + kApplyPhi, *st = sm + kApplyState, *den = sm + kApplyDen;
    const int64_t bh = blockIdx.y;
    const int i = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint16_t *qh = q + bh * int64_t(N) * kD;
    for (int r = warp; r < kQBlk; r += 8) {
        const int64_t tok = int64_t(i) * kQBlk + r;
        float x[4];
        load_row4(qh, tok, N, lane, x);
        if (tok < N) phi_row_warp(x, phi);
        *reinterpret_cast<float4 *>(pq + r * kApplyLd + 4 * lane) = make_float4(x[0], x[1], x[2], x[3]);
    }
    const float4 *ssrc = reinterpret_cast<const float4 *>(sums + (bh * nq + i) * int64_t(kStateFloats));
    for (int e = tid; e < kStateFloats / 4; e += 256) reinterpret_cast<float4 *>(st)[e] = __ldg(ssrc + e);
    __syncthreads();
    // normaliser of each row: phi(q_r) . z_i (column 128 of the state), one warp per row
    for (int r = warp; r < kQBlk; r += 8) {
        float s = 0.0f;
#pragma unroll
        for (int e = 0; e < 4; ++e) s = fmaf(pq[r * kApplyLd + 4 * lane + e], st[(4 * lane + e) * kStateCols + kD], s);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) den[r] = s;
    }
    // numerator: rows r = ty + 16 m (m < 8), columns 8 tx .. 8 tx + 7
    const int ty = tid >> 4, tx = tid & 15;
    float acc[8][8];
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[m][c] = 0.0f;
    for (int a = 0; a < kD; a += 4) {
        float4 p[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) p[m] = *reinterpret_cast<const float4 *>(pq + (ty + 16 * m) * kApplyLd + a);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float4 s0 = *reinterpret_cast<const float4 *>(st + (a + e) * kStateCols + 8 * tx);
            const float4 s1 = *reinterpret_cast<const float4 *>(st + (a + e) * kStateCols + 8 * tx + 4);
            const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const float pm = e == 0 ? p[m].x : e == 1 ? p[m].y : e == 2 ? p[m].z : p[m].w;
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[m][c] = fmaf(pm, sv[c], acc[m][c]);
            }
        }
    }
    __syncthreads();  // phi(Q) and the state are consumed
    // O_lin = numerator / normaliser (0 for a row without marginal keys) into the state
    // region; W^T into the phi(Q) region
    float *ol = st, *wt = pq;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const int r = ty + 16 * m;
        const float dn = den[r];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[m][c] = dn > 0.0f ? __fdiv_rn(acc[m][c], dn) : 0.0f;
        *reinterpret_cast<float4 *>(ol + r * kApplyLd + 8 * tx) = make_float4(acc[m][0], acc[m][1], acc[m][2], acc[m][3]);
        *reinterpret_cast<float4 *>(ol + r * kApplyLd + 8 * tx + 4) =
            make_float4(acc[m][4], acc[m][5], acc[m][6], acc[m][7]);
    }
    if (proj) {
        for (int e = tid; e < kD * kD; e += 256) {
            const int c = e / kD, f = e % kD;  // W[c][f] -> W^T[f][c]
            wt[f * kApplyLd + c] = __ldg(proj + e);
        }
        __syncthreads();
        // out[r][c] = sum_f O_lin[r][f] W[c][f]
#pragma unroll
        for (int m = 0; m < 8; ++m)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[m][c] = 0.0f;
        for (int f = 0; f < kD; f += 4) {
            float4 o4[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) o4[m] = *reinterpret_cast<const float4 *>(ol + (ty + 16 * m) * kApplyLd + f);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float4 w0 = *reinterpret_cast<const float4 *>(wt + (f + e) * kApplyLd + 8 * tx);
                const float4 w1 = *reinterpret_cast<const float4 *>(wt + (f + e) * kApplyLd + 8 * tx + 4);
                const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const float om = e == 0 ? o4[m].x : e == 1 ? o4[m].y : e == 2 ? o4[m].z : o4[m].w;
#pragma unroll
                    for (int c = 0; c < 8; ++c) acc[m][c] = fmaf(om, wv[c], acc[m][c]);
                }
            }
        }
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const int64_t tok = int64_t(i) * kQBlk + ty + 16 * m;
        if (tok >= N) continue;
        float *o = out + (bh * N + tok) * kD + 8 * tx;
        *reinterpret_cast<float4 *>(o) = make_float4(acc[m][0], acc[m][1], acc[m][2], acc[m][3]);
        *reinterpret_cast<float4 *>(o + 4) = make_float4(acc[m][4], acc[m][5], acc[m][6], acc[m][7]);
    }
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
    const int64_t g = int64_t(kChunkBudget) / per;
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
    const size_t state_smem = size_t(2) * kKBlk * kD * sizeof(float);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        if ((e = cudaFuncSetAttribute(sla_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(state_smem))) != cudaSuccess ||
            (e = cudaFuncSetAttribute(sla_sum_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(summ::kSmem))) != cudaSuccess ||
            (e = cudaFuncSetAttribute(sla_apply_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(kApplySmemBytes))) != cudaSuccess)
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
        sla_state_kernel<<<dim3(unsigned(nk), unsigned(g)), 256, state_smem, st>>>(
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
        sla_apply_kernel<<<dim3(unsigned(nq), unsigned(g)), 256, kApplySmemBytes, st>>>(
            static_cast<const uint16_t *>(q) + h0 * tok, sums, proj, N, nq, phi, out + h0 * tok);
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
