// sa_prologue.cu -- the quantise/smooth prologue: K channel means, INT8 Q and smoothed K
// per block, FP8 e4m3 V per channel written channel-major.  All passes are HBM-bound
// streams over [B,H,N,128] bf16 tensors; each thread moves 16-byte chunks (8 channels of
// one token) so every warp access is a fully used 256-byte row pair.
//
// Sources: "AIGC weekend special 5.10", section 1.2 Method item (1) (Q/K to INT8 for the
// tensor cores); "Video-Generation-101: inference systems" reference [3] (outlier
// smoothing, read as subtracting K's per-channel token mean); "Video-Generation-101
// research log" section 5.5 (FP8 P.V, so V in FP8).
//
// Bit-exactness: scales are IEEE fp32 divisions amax/127 and amax/448, codes use IEEE
// division followed by round-to-nearest-even (cvt.rni) or the e4m3 round-to-nearest-even
// saturating conversion.  This file must not be built with fast-math or -prec-div=false.
#include <cstdint>
#include <mutex>

#include <cuda_bf16.h>

#include "sa_internal.h"
#include "sa_ptx.cuh"

namespace sa {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ void unpack8(const uint4 &u, float (&x)[8])
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
        x[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    }
}

// ---- K channel sums: per (head, 1024-token chunk) fp64 partial sums, fixed order.
__global__ void __launch_bounds__(kThreads) k_partial_kernel(const uint16_t *__restrict__ k,
                                                             int Nmax, int nchunks,
                                                             double *__restrict__ part, SeqTable seq)
{
    __shared__ double red[16][kD];
    const int chunk = blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int N = seq_tokens(seq, bh, Nmax);
    const int tid = threadIdx.x, cg = tid & 15, rs = tid >> 4;
    const int t0 = chunk * kMeanChunk;
    if (t0 >= N) return;  // past this head's tokens (variable-length batches)
    const int t1 = min(N, t0 + kMeanChunk);
    const uint16_t *kh = k + seq_row0(seq, bh, Nmax) * kD;
    double acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0;
    for (int t = t0 + rs; t < t1; t += 16) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(kh + int64_t(t) * kD + cg * 8));
        float x[8];
        unpack8(u, x);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += double(x[e]);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[rs][cg * 8 + e] = acc[e];
    __syncthreads();
    if (tid < kD) {
        double s = 0.0;
#pragma unroll
        for (int r = 0; r < 16; ++r) s += red[r][tid];
        part[(bh * nchunks + chunk) * kD + tid] = s;
    }
}

// mean_k[c] = fp32( (sum over this head's chunks, in order) / N ) in fp64.
__global__ void __launch_bounds__(kD) k_mean_kernel(const double *__restrict__ part, int Nmax,
                                                    int nchunks, float *__restrict__ mean, SeqTable seq)
{
    const int64_t bh = blockIdx.x;
    const int c = threadIdx.x;
    const int N = seq_tokens(seq, bh, Nmax), nch = (N + kMeanChunk - 1) / kMeanChunk;
    double s = 0.0;
    for (int i = 0; i < nch; ++i) s += part[(bh * nchunks + i) * kD + c];
    mean[bh * kD + c] = float(s / double(N));
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// INT8 code of x under scale s: round-half-even of the IEEE quotient x/s, clamped to
// [-127, 127].  r = 1/s (correctly rounded).  Fast path: y = x*r differs from the IEEE
// quotient fl(x/s) by at most |x/s| * 3 * 2^-24 < 2.3e-5 (|x/s| <= 127 + tiny), so when y
// is at least 2^-14 away from every half-integer both round to the same integer; the
// rare y within 2^-14 of a half-integer takes the exact division.
__device__ __forceinline__ int int8_code(float x, float s, float r)
{
    if (s == 0.0f) return 0;
    const float y = __fmul_rn(x, r);
    float n = rintf(y);
    if (fabsf(fabsf(__fsub_rn(y, n)) - 0.5f) < 6.103515625e-05f) n = rintf(__fdiv_rn(x, s));
    return max(-127, min(127, int(n)));
}

// One quantisation block of ROWS tokens x 128 channels starting at token r0.
// mean != nullptr: smooth first (x - mean[c], one fp32 subtraction).  Rows >= N are
// excluded from the max and stored as zero codes.  scale_out may be null (padding-only
// block).  The block is held as raw bf16 (4 registers per 8 values) and unpacked twice,
// which keeps the kernel at 4 CTAs per SM.
template <int ROWS>
__device__ __forceinline__ void quant_block(const uint16_t *__restrict__ src, int N, int r0,
                                            const float *__restrict__ mean,
                                            int8_t *__restrict__ dst, float *scale_out,
                                            float *red)
{
    constexpr int PER = ROWS * 16 / kThreads;  // 16-byte chunks per thread
    const int tid = threadIdx.x, cg = tid & 15, rs = tid >> 4;
    uint4 raw[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int t = r0 + rs + 16 * i;
        raw[i] = t < N ? __ldg(reinterpret_cast<const uint4 *>(src + int64_t(t) * kD + cg * 8))
                       : make_uint4(0, 0, 0, 0);
    }
    float mc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) mc[e] = mean ? mean[cg * 8 + e] : 0.0f;
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        if (r0 + rs + 16 * i < N) {
            float x[8];
            unpack8(raw[i], x);
#pragma unroll
            for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(mean ? __fsub_rn(x[e], mc[e]) : x[e]));
        }
    }
    amax = warp_max(amax);
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, red[w]);
    const float s = __fdiv_rn(amax, 127.0f);
    const float r = s == 0.0f ? 0.0f : __frcp_rn(s);
    if (tid == 0 && scale_out) *scale_out = s;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int t = r0 + rs + 16 * i;
        uint32_t lo = 0, hi = 0;
        if (t < N) {
            float x[8];
            unpack8(raw[i], x);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const uint32_t code = uint32_t(uint8_t(int8_code(mean ? __fsub_rn(x[e], mc[e]) : x[e], s, r)));
                if (e < 4) lo |= code << (8 * e);
                else hi |= code << (8 * (e - 4));
            }
        }
        *reinterpret_cast<uint2 *>(dst + int64_t(t) * kD + cg * 8) = make_uint2(lo, hi);
    }
}

// grid (nq + Npad/64, BH): x < nq quantises Q block x; otherwise K block x - nq
// (blocks at or past nk only zero-fill the padded key rows).  With a variable-length
// table, N is the head's own length and blocks past its padded length are skipped (the
// attention kernel never reads them); nq, nk and Npad are the strides of the longest.
__global__ void __launch_bounds__(kThreads, 4)
    qk_quant_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k, int Nmax,
                    int Npad, int nq, int nk, const float *__restrict__ kmean,
                    int8_t *__restrict__ q_i8, float *__restrict__ q_scale,
                    int8_t *__restrict__ k_i8, float *__restrict__ k_scale, SeqTable seq)
{
    __shared__ float red[kThreads / 32];
    const int64_t bh = blockIdx.y;
    const int x = blockIdx.x;
    const int N = seq_tokens(seq, bh, Nmax), nqh = (N + kQBlk - 1) / kQBlk, nkh = (N + kKBlk - 1) / kKBlk;
    const int64_t row0 = seq_row0(seq, bh, Nmax);
    if (x < nq) {
        if (x >= nqh) return;
        quant_block<kQBlk>(q + row0 * kD, N, x * kQBlk, nullptr, q_i8 + bh * int64_t(Npad) * kD,
                           q_scale + bh * nq + x, red);
    } else {
        const int j = x - nq;
        if (j * kKBlk >= nqh * kQBlk) return;
        quant_block<kKBlk>(k + row0 * kD, N, j * kKBlk, kmean + bh * kD, k_i8 + bh * int64_t(Npad) * kD,
                           j < nkh ? k_scale + bh * nk + j : nullptr, red);
    }
}

// ---- V: per-channel max |v| (as bf16 magnitude bits; order-free), then codes.
__global__ void __launch_bounds__(kThreads) v_amax_kernel(const uint16_t *__restrict__ v, int Nmax,
                                                          uint32_t *__restrict__ amax_bits, SeqTable seq)
{
    __shared__ uint32_t red[16][kD];
    const int chunk = blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int N = seq_tokens(seq, bh, Nmax);
    const int tid = threadIdx.x, cg = tid & 15, rs = tid >> 4;
    const int t0 = chunk * kMeanChunk;
    if (t0 >= N) return;
    const int t1 = min(N, t0 + kMeanChunk);
    const uint16_t *vh = v + seq_row0(seq, bh, Nmax) * kD;
    uint32_t m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int t = t0 + rs; t < t1; t += 16) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(vh + int64_t(t) * kD + cg * 8));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            m[2 * i] = max(m[2 * i], w[i] & 0x7FFFu);
            m[2 * i + 1] = max(m[2 * i + 1], (w[i] >> 16) & 0x7FFFu);
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[rs][cg * 8 + e] = m[e];
    __syncthreads();
    if (tid < kD) {
        uint32_t r = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) r = max(r, red[i][tid]);
        atomicMax(amax_bits + bh * kD + tid, r);
    }
}

// grid (Npad/128, BH): a 128-token x 128-channel tile, quantised and transposed through
// shared memory so that both the bf16 reads and the channel-major FP8 writes are
// coalesced 16-byte accesses.  The tile is channel-major, 128 B per channel; byte (c, r)
// sits in 16-byte chunk (r / 16) ^ (g & 7) and 4-byte word ((r % 16) / 4) ^ (g >> 3) of
// row c, g = c / 8: the 16 threads of a half-warp, each writing one byte for its own group
// of 8 channels, then hit 16 different banks, and a thread still reads a whole chunk.
__global__ void __launch_bounds__(kThreads)
    v_quant_kernel(const uint16_t *__restrict__ v, int Nmax, int Npad,
                   const uint32_t *__restrict__ amax_bits, uint8_t *__restrict__ v_t,
                   float *__restrict__ v_scale, SeqTable seq)
{
    __shared__ __align__(16) uint8_t tile[kD][kQBlk];
    __shared__ float sv[kD];
    const int64_t bh = blockIdx.y;
    const int t0 = blockIdx.x * kQBlk;
    const int N = seq_tokens(seq, bh, Nmax);
    if (blockIdx.x > 0 && t0 >= N) return;  // past this head's padded length (tile 0 writes the scales)
    const int tid = threadIdx.x, cg = tid & 15, rs = tid >> 4;
    if (tid < kD) {
        const float s = __fdiv_rn(bf16_bits_to_f32(amax_bits[bh * kD + tid]), 448.0f);
        sv[tid] = s;
        if (blockIdx.x == 0) v_scale[bh * kD + tid] = s;
    }
    __syncthreads();
    const uint16_t *vh = v + seq_row0(seq, bh, Nmax) * kD;
    const int swz_chunk = cg & 7, swz_word = cg >> 3;
#pragma unroll
    for (int i = 0; i < kQBlk * 16 / kThreads; ++i) {
        const int r = rs + 16 * i;
        const int t = t0 + r;
        float x[8];
        if (t < N) {
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(vh + int64_t(t) * kD + cg * 8));
            unpack8(u, x);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = 0.0f;
        }
        const int pos = (((r >> 4) ^ swz_chunk) << 4) | ((((r & 15) >> 2) ^ swz_word) << 2) | (r & 3);
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const float s0 = sv[cg * 8 + e], s1 = sv[cg * 8 + e + 1];
            const float y0 = s0 == 0.0f ? 0.0f : __fdiv_rn(x[e], s0);
            const float y1 = s1 == 0.0f ? 0.0f : __fdiv_rn(x[e + 1], s1);
            const uint32_t p = pack_e4m3x2(y0, y1);
            tile[cg * 8 + e][pos] = uint8_t(p & 0xFFu);
            tile[cg * 8 + e + 1][pos] = uint8_t(p >> 8);
        }
    }
    __syncthreads();
    uint8_t *vt = v_t + bh * int64_t(kD) * Npad;
#pragma unroll
    for (int i = 0; i < kD * 8 / kThreads; ++i) {
        const int qd = tid + kThreads * i;
        const int c = qd >> 3, part = qd & 7, g = c >> 3;
        const uint4 w = *reinterpret_cast<const uint4 *>(&tile[c][(part ^ (g & 7)) << 4]);
        const uint4 u = (g >> 3) ? make_uint4(w.y, w.x, w.w, w.z) : w;  // undo the word swizzle
        *reinterpret_cast<uint4 *>(vt + int64_t(c) * Npad + t0 + part * 16) = u;
    }
}

// Head-size padding for d = 64 calls: rows of 64 bf16 channels <-> rows of 128 whose upper
// 64 channels are zero.  One thread per 16-byte group (8 channels) of the wider row.
__global__ void pad_heads_kernel(const uint4 *__restrict__ src, int64_t rows, uint4 *__restrict__ dst)
{
    const int64_t n = rows * 16;
    for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < n; e += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = e >> 4;
        const int g = int(e & 15);
        dst[e] = g < 8 ? src[r * 8 + g] : make_uint4(0, 0, 0, 0);
    }
}

__global__ void unpad_heads_kernel(const uint4 *__restrict__ src, int64_t rows, uint4 *__restrict__ dst)
{
    const int64_t n = rows * 8;
    for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < n; e += int64_t(gridDim.x) * blockDim.x)
        dst[e] = src[(e >> 3) * 16 + (e & 7)];
}

}  // namespace

static int grid_for(int64_t n)
{
    const int64_t want = (n + 255) / 256;
    return int(want < 8192 ? want : 8192);
}

cudaError_t launch_pad_heads(const void *src, int64_t rows, void *dst, cudaStream_t st)
{
    pad_heads_kernel<<<grid_for(rows * 16), 256, 0, st>>>(static_cast<const uint4 *>(src), rows,
                                                         static_cast<uint4 *>(dst));
    return cudaGetLastError();
}

cudaError_t launch_unpad_heads(const void *src, int64_t rows, void *dst, cudaStream_t st)
{
    unpad_heads_kernel<<<grid_for(rows * 8), 256, 0, st>>>(static_cast<const uint4 *>(src), rows,
                                                          static_cast<uint4 *>(dst));
    return cudaGetLastError();
}

// Scratch of sa_quantize_qk_noalloc: the fp64 per-chunk column sums of K, in a fixed
// device array instead of the library's cudaMalloc'd workspace.  It lives for the whole
// process on every device that loads the library, is shared by all calls (each call
// overwrites every element it reads, so nothing needs clearing between calls), and two
// such calls whose kernels overlap on one device race on it.
static __device__ __align__(256) double g_noalloc_kpart[kNoAllocPartialDoubles];

cudaError_t noalloc_kpart(double **out)
{
    // In host code the array's name is only a stand-in; the address the kernels must use
    // is looked up once per device, with that device current.
    static double *addr[64] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_kpart);
        if (e != cudaSuccess) return e;
        addr[dev] = static_cast<double *>(ptr);
    }
    *out = addr[dev];
    return cudaSuccess;
}

cudaError_t launch_quantize_qk(const void *q, const void *k, const Shape &s, int8_t *q_i8,
                               float *q_scale, int8_t *k_i8, float *k_scale, float *k_mean,
                               double *k_partial, cudaStream_t st, const SeqTable &seq)
{
    const int N = int(s.N), Npad = int(s.Npad()), nq = int(s.nq()), nk = int(s.nk());
    const int nch = int(s.nchunks());
    const dim3 g1(nch, unsigned(s.BH()));
    k_partial_kernel<<<g1, kThreads, 0, st>>>(static_cast<const uint16_t *>(k), N, nch, k_partial, seq);
    k_mean_kernel<<<unsigned(s.BH()), kD, 0, st>>>(k_partial, N, nch, k_mean, seq);
    const dim3 g2(nq + Npad / kKBlk, unsigned(s.BH()));
    qk_quant_kernel<<<g2, kThreads, 0, st>>>(static_cast<const uint16_t *>(q),
                                             static_cast<const uint16_t *>(k), N, Npad, nq, nk,
                                             k_mean, q_i8, q_scale, k_i8, k_scale, seq);
    return cudaGetLastError();
}

cudaError_t launch_quantize_v(const void *v, const Shape &s, uint8_t *v_t, float *v_scale,
                              uint32_t *v_amax_bits, cudaStream_t st, const SeqTable &seq)
{
    const int N = int(s.N), Npad = int(s.Npad());
    cudaError_t e = cudaMemsetAsync(v_amax_bits, 0, sizeof(uint32_t) * s.BH() * kD, st);
    if (e != cudaSuccess) return e;
    const dim3 g1(unsigned(s.nchunks()), unsigned(s.BH()));
    v_amax_kernel<<<g1, kThreads, 0, st>>>(static_cast<const uint16_t *>(v), N, v_amax_bits, seq);
    const dim3 g2(unsigned(Npad / kQBlk), unsigned(s.BH()));
    v_quant_kernel<<<g2, kThreads, 0, st>>>(static_cast<const uint16_t *>(v), N, Npad, v_amax_bits,
                                            v_t, v_scale, seq);
    return cudaGetLastError();
}

}  // namespace sa
