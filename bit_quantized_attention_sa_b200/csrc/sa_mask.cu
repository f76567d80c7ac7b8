// sa_mask.cu -- the block-mask producer: the selector ahead of the block skip.
//
// Sources: NetEase article on the TurboDiffusion release, attention-acceleration section,
// SLA figure caption (attention weights fall into three classes computed at different
// costs; SLA's forward works from predicted, compressed attention weights);
// "Video-Generation-101 research log" section 5.5 table, SpargeAttention row (a block
// selector ahead of the sparse low-bit kernel).
//
// Q is mean-pooled per 128-token block and K per 64-token block (the keep mask's
// geometry); every (query block, key block) pair is scored by the fp64 dot product of the
// two means (a tiled kernel, scores kept in the workspace); a mask row keeps its
// keep_per_row best key blocks, ties going to the lower block index, and optionally the
// diagonal blocks 2i and 2i+1.  The arithmetic order is fixed so that the mask is a
// deterministic function of the inputs:
//   - a block mean is the fp64 sum of the block's tokens in ascending order (one thread per
//     channel), divided by the token count in fp64 and rounded once to fp32;
//   - a score sums the 128 exact fp64 products in ascending channel order;
//   - the kept set is the first keep_per_row blocks in the total order "larger score
//     first, then lower index" (a radix selection of the threshold score), so it is unique.
#include <cstdint>
#include <cmath>

#include "sa_internal.h"

namespace sa {
namespace {

__device__ __forceinline__ double bf16_bits_to_f64(uint16_t b)
{
    return double(__uint_as_float(uint32_t(b) << 16));
}

// grid (nq + nk, BH), kD threads: x < nq pools Q block x, else K block x - nq.
__global__ void __launch_bounds__(kD)
    pool_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k, int N, int nq,
                int nk, float *__restrict__ qbar, float *__restrict__ kbar)
{
    const int64_t bh = blockIdx.y;
    const int x = blockIdx.x, c = threadIdx.x;
    const bool isq = x < nq;
    const int b = isq ? x : x - nq, blk = isq ? kQBlk : kKBlk;
    const int t0 = b * blk, t1 = min(N, t0 + blk);
    const uint16_t *src = (isq ? q : k) + bh * int64_t(N) * kD + c;
    double s = 0.0;
    for (int t = t0; t < t1; ++t) s = __dadd_rn(s, bf16_bits_to_f64(src[int64_t(t) * kD]));
    const float mean = __double2float_rn(__ddiv_rn(s, double(t1 - t0)));
    if (isq) qbar[(bh * nq + b) * kD + c] = mean;
    else kbar[(bh * nk + b) * kD + c] = mean;
}

// grid (ceil(nk/64), ceil(nq/64), BH), 256 threads: the 64 x 64 tile of pooled scores
// scores[bh, i, j] = sum over c ascending of (double)qbar[i,c] * (double)kbar[j,c]; each
// thread owns 4 x 4 outputs and adds the products for c = 0, 1, ..., 127 in turn.  The
// product of two fp32 values is exact in fp64, so a fused multiply-add rounds exactly as
// the multiplication followed by the addition.  The means are staged as doubles,
// channel-major, 16 channels at a time.
constexpr int kScoreTile = 64, kScoreChunk = 16, kScoreThreads = 256;

__global__ void __launch_bounds__(kScoreThreads)
    block_scores_kernel(const float *__restrict__ qbar, const float *__restrict__ kbar, int nq,
                        int nk, double *__restrict__ scores)
{
    __shared__ __align__(16) double qs[kScoreChunk][kScoreTile];
    __shared__ __align__(16) double ks[kScoreChunk][kScoreTile];
    const int64_t bh = blockIdx.z;
    const int i0 = blockIdx.y * kScoreTile, j0 = blockIdx.x * kScoreTile;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const float *qb = qbar + bh * int64_t(nq) * kD, *kb = kbar + bh * int64_t(nk) * kD;
    double acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
    for (int c0 = 0; c0 < kD; c0 += kScoreChunk) {
        // 64 rows x 16 channels of each operand: 1024 values, 4 per thread
#pragma unroll
        for (int e = 0; e < kScoreTile * kScoreChunk / kScoreThreads; ++e) {
            const int f = tid + kScoreThreads * e, r = f / kScoreChunk, c = f % kScoreChunk;
            qs[c][r] = i0 + r < nq ? double(qb[int64_t(i0 + r) * kD + c0 + c]) : 0.0;
            ks[c][r] = j0 + r < nk ? double(kb[int64_t(j0 + r) * kD + c0 + c]) : 0.0;
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < kScoreChunk; ++c) {
            double qv[4], kv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) qv[a] = qs[c][ty * 4 + a];
#pragma unroll
            for (int b = 0; b < 4; ++b) kv[b] = ks[c][tx * 4 + b];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = __fma_rn(qv[a], kv[b], acc[a][b]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int i = i0 + ty * 4 + a;
        if (i >= nq) continue;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int j = j0 + tx * 4 + b;
            if (j < nk) scores[(bh * nq + i) * int64_t(nk) + j] = acc[a][b];
        }
    }
}

// Order-preserving unsigned key of a double: larger double, larger key (finite inputs;
// -0.0 and +0.0, equal as scores, get the same key).
__device__ __forceinline__ uint64_t order_key(double x)
{
    if (x == 0.0) x = 0.0;
    const uint64_t u = uint64_t(__double_as_longlong(x));
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

constexpr int kSelThreads = 256;

// grid (nq, BH), kSelThreads threads; dynamic shared memory: nk uint64 keys.  Finds the
// keep_per_row-th largest score of the row by radix selection on the order-preserving
// keys (8 passes of 8 bits, most significant first), keeps every block above it and, of
// the blocks equal to it, the lowest-indexed ones: exactly the first keep_per_row blocks
// in the order "larger score first, then lower index".
__global__ void __launch_bounds__(kSelThreads)
    block_select_kernel(const double *__restrict__ scores, int nq, int nk, int keep_per_row,
                        int keep_diagonal, uint8_t *__restrict__ mask)
{
    extern __shared__ __align__(16) uint64_t key[];
    __shared__ uint32_t hist[256];
    __shared__ uint64_t s_prefix;
    __shared__ int s_rem;
    const int64_t bh = blockIdx.y;
    const int i = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
    const double *srow = scores + (bh * nq + i) * int64_t(nk);
    uint8_t *mrow = mask + (bh * nq + i) * int64_t(nk);
    if (keep_per_row >= nk) {
        for (int j = tid; j < nk; j += kSelThreads) mrow[j] = 1;
        return;
    }
    for (int j = tid; j < nk; j += kSelThreads) key[j] = order_key(srow[j]);
    uint64_t prefix = 0, pmask = 0;
    int rem = keep_per_row;  // how many of the keys matching the prefix are still to keep
    for (int shift = 56; shift >= 0; shift -= 8) {
        hist[tid] = 0;  // kSelThreads == 256 bins
        __syncthreads();
        for (int j = tid; j < nk; j += kSelThreads) {
            const uint64_t kj = key[j];
            if ((kj & pmask) == prefix) atomicAdd(&hist[(kj >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid < 32) {
            // bins from the top: lane l holds bins 255-8l ... 248-8l
            uint32_t c[8], tot = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) tot += (c[e] = hist[255 - 8 * lane - e]);
            uint32_t incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const uint32_t excl = incl - tot;  // keys in bins above this lane's
            const bool here = excl < uint32_t(rem) && uint32_t(rem) <= incl;
            if (here) {
                uint32_t above = excl;
                int e = 0;
                while (above + c[e] < uint32_t(rem)) above += c[e++];
                s_prefix = prefix | (uint64_t(255 - 8 * lane - e) << shift);
                s_rem = rem - int(above);
            }
        }
        __syncthreads();
        prefix = s_prefix;
        rem = s_rem;
        pmask |= uint64_t(255) << shift;
        __syncthreads();
    }
    // keep every key above the threshold, then the first `rem` equal ones in index order
    for (int j = tid; j < nk; j += kSelThreads) mrow[j] = key[j] > prefix ? 1 : 0;
    __syncthreads();
    if (tid < 32) {
        int left = rem;
        for (int base = 0; base < nk && left > 0; base += 32) {
            const int j = base + lane;
            const bool eq = j < nk && key[j] == prefix;
            const uint32_t bal = __ballot_sync(0xffffffffu, eq);
            const int before_me = __popc(bal & ((1u << lane) - 1u));
            if (eq && before_me < left) mrow[j] = 1;
            left -= __popc(bal);
        }
    }
    __syncthreads();
    if (keep_diagonal && tid < 2 && 2 * i + tid < nk) mrow[2 * i + tid] = 1;
}

// grid-stride over BH * nq * nk entries.
__global__ void causal_mask_kernel(const uint8_t *__restrict__ user, int64_t nq, int64_t nk, int64_t n,
                                   uint8_t *__restrict__ out)
{
    for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < n; e += int64_t(gridDim.x) * blockDim.x) {
        const int64_t j = e % nk, i = (e / nk) % nq;
        out[e] = (j <= 2 * i + 1 && (!user || user[e])) ? 1 : 0;
    }
}

}  // namespace

cudaError_t launch_causal_mask(const uint8_t *user, const Shape &s, uint8_t *out, cudaStream_t st)
{
    const int64_t n = s.BH() * s.nq() * s.nk();
    const int64_t want = (n + 255) / 256;
    const int blocks = int(want < 4096 ? want : 4096);
    causal_mask_kernel<<<blocks, 256, 0, st>>>(user, s.nq(), s.nk(), n, out);
    return cudaGetLastError();
}

cudaError_t launch_pool_qk(const void *q, const void *k, const Shape &s, float *qbar, float *kbar,
                           cudaStream_t st)
{
    const dim3 g(unsigned(s.nq() + s.nk()), unsigned(s.BH()));
    pool_kernel<<<g, kD, 0, st>>>(static_cast<const uint16_t *>(q), static_cast<const uint16_t *>(k),
                                  int(s.N), int(s.nq()), int(s.nk()), qbar, kbar);
    return cudaGetLastError();
}

cudaError_t launch_block_select(const float *qbar, const float *kbar, double *scores, const Shape &s,
                                int keep_per_row, int keep_diagonal, uint8_t *mask, cudaStream_t st)
{
    const dim3 gs(unsigned((s.nk() + kScoreTile - 1) / kScoreTile), unsigned((s.nq() + kScoreTile - 1) / kScoreTile),
                  unsigned(s.BH()));
    block_scores_kernel<<<gs, kScoreThreads, 0, st>>>(qbar, kbar, int(s.nq()), int(s.nk()), scores);
    const int nk = int(s.nk());
    const size_t smem = sizeof(uint64_t) * size_t(nk);
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        e = cudaFuncSetAttribute(block_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(sizeof(uint64_t) * kMaskMaxKeyBlocks));
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    const dim3 g(unsigned(s.nq()), unsigned(s.BH()));
    block_select_kernel<<<g, kSelThreads, smem, st>>>(scores, int(s.nq()), nk, keep_per_row,
                                                       keep_diagonal, mask);
    return cudaGetLastError();
}

}  // namespace sa
