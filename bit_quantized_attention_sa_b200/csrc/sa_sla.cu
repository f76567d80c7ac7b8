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

namespace sa {
namespace {

constexpr int kStateCols = 136;                      // H_j columns, then Z_j, then zeros
constexpr int kStateFloats = kD * kStateCols;        // 17408 per key (or query) block
constexpr int kSumChunk = 1024;                      // floats of a state per sum CTA
constexpr int kSumChunks = kStateFloats / kSumChunk;  // 17
constexpr int kSumGroup = 16;                        // query blocks per sum CTA
static_assert(kStateFloats % kSumChunk == 0, "state chunks");

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

// grid (kSumChunks, ceil(nq / 16), BH), 256 threads; dynamic shared memory nk uint32.
// A_i (chunk) = sum over j ascending of the states of the blocks with classes[i][j] == 1.
__global__ void __launch_bounds__(256)
    sla_state_sum_kernel(const float *__restrict__ state, const uint8_t *__restrict__ classes, int nq, int nk,
                         float *__restrict__ sums)
{
    extern __shared__ uint32_t marg_bits[];  // bit g: query block i0 + g has class 1 at j
    const int64_t bh = blockIdx.z;
    const int cc = blockIdx.x, i0 = blockIdx.y * kSumGroup, tid = threadIdx.x;
    const int ng = min(kSumGroup, nq - i0);
    for (int j = tid; j < nk; j += blockDim.x) {
        uint32_t bits = 0;
        for (int g = 0; g < ng; ++g) bits |= uint32_t(classes[(bh * nq + i0 + g) * int64_t(nk) + j] == 1) << g;
        marg_bits[j] = bits;
    }
    __syncthreads();
    float4 acc[kSumGroup];
#pragma unroll
    for (int g = 0; g < kSumGroup; ++g) acc[g] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    const float *src = state + bh * int64_t(nk) * kStateFloats + cc * kSumChunk + 4 * tid;
    // 8 key blocks per step: their loads are all in flight before the first is added
    constexpr int kAhead = 8;
    for (int j0 = 0; j0 < nk; j0 += kAhead) {
        uint32_t bits[kAhead];
        float4 h[kAhead];
#pragma unroll
        for (int u = 0; u < kAhead; ++u) {
            bits[u] = j0 + u < nk ? marg_bits[j0 + u] : 0u;
            h[u] = bits[u] ? __ldg(reinterpret_cast<const float4 *>(src + int64_t(j0 + u) * kStateFloats))
                           : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
        // keeps the compiler from sinking each load to its first use
#pragma unroll
        for (int u = 0; u < kAhead; ++u) asm volatile("" ::"f"(h[u].x), "f"(h[u].y), "f"(h[u].z), "f"(h[u].w));
#pragma unroll
        for (int u = 0; u < kAhead; ++u) {
#pragma unroll
            for (int g = 0; g < kSumGroup; ++g) {
                if ((bits[u] >> g) & 1u) {
                    acc[g].x += h[u].x;
                    acc[g].y += h[u].y;
                    acc[g].z += h[u].z;
                    acc[g].w += h[u].w;
                }
            }
        }
    }
    float *dst = sums + (bh * nq + i0) * int64_t(kStateFloats) + cc * kSumChunk + 4 * tid;
#pragma unroll
    for (int g = 0; g < kSumGroup; ++g)
        if (g < ng) *reinterpret_cast<float4 *>(dst + int64_t(g) * kStateFloats) = acc[g];
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

size_t sla_state_bytes(const Shape &s) { return size_t(s.BH()) * size_t(s.nk()) * kStateFloats * sizeof(float); }
size_t sla_sum_bytes(const Shape &s) { return size_t(s.BH()) * size_t(s.nq()) * kStateFloats * sizeof(float); }

cudaError_t launch_sla_linear(const void *q, const void *k, const void *v, const uint8_t *classes, const Shape &s,
                              int phi, const float *proj, float *state, float *sums, float *out, cudaStream_t st)
{
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const size_t state_smem = size_t(2) * kKBlk * kD * sizeof(float);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        if ((e = cudaFuncSetAttribute(sla_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(state_smem))) != cudaSuccess ||
            (e = cudaFuncSetAttribute(sla_state_sum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(sizeof(uint32_t) * kMaskMaxKeyBlocks))) != cudaSuccess ||
            (e = cudaFuncSetAttribute(sla_apply_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(kApplySmemBytes))) != cudaSuccess)
            return e;
        attr_set[dev] = true;
    }
    const int nq = int(s.nq()), nk = int(s.nk()), N = int(s.N);
    const auto *qb = static_cast<const uint16_t *>(q);
    sla_state_kernel<<<dim3(unsigned(nk), unsigned(s.BH())), 256, state_smem, st>>>(
        static_cast<const uint16_t *>(k), static_cast<const uint16_t *>(v), N, nk, phi, state);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    sla_state_sum_kernel<<<dim3(unsigned(kSumChunks), unsigned((nq + kSumGroup - 1) / kSumGroup), unsigned(s.BH())),
                           256, sizeof(uint32_t) * size_t(nk), st>>>(state, classes, nq, nk, sums);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const dim3 ga(unsigned(nq), unsigned(s.BH()));
    sla_apply_kernel<<<ga, 256, kApplySmemBytes, st>>>(qb, sums, proj, N, nq, phi, out);
    return cudaGetLastError();
}

cudaError_t launch_sla_critical(const uint8_t *classes, int64_t n, uint8_t *keep, cudaStream_t st)
{
    const int blocks = int(n / 1024 + 1 < 4096 ? n / 1024 + 1 : 4096);
    sla_critical_kernel<<<blocks, 256, 0, st>>>(classes, n, keep);
    return cudaGetLastError();
}

}  // namespace sa
