// sa_api.cu -- the C ABI declared in include/sa.h: argument validation, the per-device
// grow-only workspace, TMA tensor-map encoding and launch sequencing on the caller's
// stream.  No entry point synchronises except sa_get_device_status and
// sa_release_workspace.
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <numeric>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/sa.h"
#include "sa_internal.h"

namespace sa {

// ------------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool encode_tmap_2d_u8(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                       uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                       CUtensorMapSwizzle swizzle)
{
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tmap_3d_f32(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                        uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1,
                        CUtensorMapSwizzle swizzle)
{
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    const cuuint32_t box[3] = {box0, box1, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ validation

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static sa_status check_shape(int B, int H, int N, int d, Shape *s)
{
    if (B < 1 || H < 1 || N < 1) return SA_ERR_INVALID_ARG;
    if (d != kD) return SA_ERR_UNSUPPORTED;
    s->B = B;
    s->H = H;
    s->N = N;
    // TMA row coordinates and tile indices are 32-bit
    if (s->BH() > INT_MAX / 8 || s->BH() * s->Npad() > INT_MAX) return SA_ERR_INVALID_ARG;
    // the heads are a grid dimension (y) of the prologue kernels
    if (s->BH() > 65535) return SA_ERR_UNSUPPORTED;
    return SA_OK;
}

static sa_status check_ptrs(std::initializer_list<const void *> ps)
{
    for (const void *p : ps)
        if (!p) return SA_ERR_INVALID_ARG;
    for (const void *p : ps)
        if (!aligned16(p)) return SA_ERR_MISALIGNED;
    return SA_OK;
}

// sm_100 device check, cached per device.
static sa_status check_device()
{
    static int cached[64];  // 0 unknown, 1 ok, 2 unsupported
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
    if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev] == 1 ? SA_OK : SA_ERR_UNSUPPORTED;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return SA_ERR_CUDA;
    const bool ok = (major == 10 && minor == 0);
    if (dev >= 0 && dev < 64) cached[dev] = ok ? 1 : 2;
    return ok ? SA_OK : SA_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------------ workspace

struct WsLayout {
    size_t q8, k8, v8, sq, sk, sv, kmean, kpart, vamax, total;
};

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

static WsLayout ws_layout(const Shape &s)
{
    WsLayout L;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
    const size_t BH = size_t(s.BH()), Np = size_t(s.Npad());
    L.q8 = take(BH * Np * kD);
    L.k8 = take(BH * Np * kD);
    L.v8 = take(BH * Np * kD);
    L.sq = take(BH * size_t(s.nq()) * 4);
    L.sk = take(BH * size_t(s.nk()) * 4);
    L.sv = take(BH * kD * 4);
    L.kmean = take(BH * kD * 4);
    L.kpart = take(BH * size_t(s.nchunks()) * kD * 8);
    L.vamax = take(BH * kD * 4);
    L.total = off;
    return L;
}

struct DeviceWs {
    void *ptr = nullptr;
    size_t bytes = 0;
};
static DeviceWs g_ws[64];
// Held by a call from its workspace request until its launches are enqueued, so that no
// other host thread can grow (and so free) the buffer in between.  Recursive: the d = 64
// and SLA paths request the workspace again inside the same call.
static std::recursive_mutex g_ws_mutex;
typedef std::unique_lock<std::recursive_mutex> WsLock;

// Returns the current device's workspace grown to at least `bytes`, with `lock` held.
static sa_status get_workspace(WsLock &lock, size_t bytes, uint8_t **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SA_ERR_CUDA;
    if (!lock.owns_lock()) lock = WsLock(g_ws_mutex);
    DeviceWs &w = g_ws[dev];
    if (w.bytes < bytes) {
        if (w.ptr) {
            // work enqueued earlier, on any stream, may still use the old buffer
            if (cudaDeviceSynchronize() != cudaSuccess) return SA_ERR_CUDA;
            cudaFree(w.ptr);
            w.ptr = nullptr;
            w.bytes = 0;
        }
        if (cudaMalloc(&w.ptr, bytes) != cudaSuccess) {
            cudaGetLastError();
            w.ptr = nullptr;
            return SA_ERR_OOM;
        }
        w.bytes = bytes;
    }
    *out = static_cast<uint8_t *>(w.ptr);
    return SA_OK;
}

// Page-locked host staging for small tables that a call uploads (variable-length
// batches), per device, grow-only.  Used with the workspace lock held; the event marks the
// last upload, which must have left the buffer before it is overwritten.
struct HostStage {
    void *ptr = nullptr;
    size_t bytes = 0;
    cudaEvent_t ev = nullptr;
};
static HostStage g_stage[64];

static sa_status upload_table(const void *src, size_t n, void *dst, cudaStream_t st)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SA_ERR_CUDA;
    HostStage &h = g_stage[dev];
    if (!h.ev) {
        if (cudaEventCreateWithFlags(&h.ev, cudaEventDisableTiming) != cudaSuccess) return SA_ERR_CUDA;
    } else if (cudaEventSynchronize(h.ev) != cudaSuccess) {
        return SA_ERR_CUDA;
    }
    if (h.bytes < n) {
        if (h.ptr) cudaFreeHost(h.ptr);
        h.ptr = nullptr;
        h.bytes = 0;
        if (cudaMallocHost(&h.ptr, n) != cudaSuccess) {
            cudaGetLastError();
            return SA_ERR_OOM;
        }
        h.bytes = n;
    }
    std::memcpy(h.ptr, src, n);
    if (cudaMemcpyAsync(dst, h.ptr, n, cudaMemcpyHostToDevice, st) != cudaSuccess) return SA_ERR_CUDA;
    return cudaEventRecord(h.ev, st) == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

static sa_status attention_core(const int8_t *q8, const float *sq, const int8_t *k8,
                                const float *sk, const uint8_t *v8, const float *sv, void *o,
                                const Shape &s, float sm_scale, const uint8_t *mask,
                                cudaStream_t st, bool causal = false, const float *addend = nullptr,
                                const SeqTable &seq = SeqTable())
{
    AttnArgs a;
    const uint64_t rows = uint64_t(s.BH() * s.Npad());
    if (!encode_tmap_2d_u8(&a.tm_q, q8, kD, rows, kD, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tmap_2d_u8(&a.tm_k, k8, kD, rows, kD, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tmap_2d_u8(&a.tm_v, v8, uint64_t(s.Npad()), uint64_t(s.BH()) * kD,
                           uint64_t(s.Npad()), 64, 128, CU_TENSOR_MAP_SWIZZLE_64B))
        return SA_ERR_CUDA;
    a.q_scale = sq;
    a.k_scale = sk;
    a.v_scale = sv;
    a.mask = mask;
    a.o = static_cast<__nv_bfloat16 *>(o);
    a.BH = int(s.BH());
    a.N = int(s.N);
    a.Npad = int(s.Npad());
    a.nq = int(s.nq());
    a.nk = int(s.nk());
    a.sm_scale = sm_scale;
    a.causal = causal ? 1 : 0;
    a.addend = addend;
    a.seq = seq;
    return launch_attention(a, st) == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

// Prologue into the library workspace, then the fused attention kernel (validated args).
static sa_status attn_fwd_device(const void *q, const void *k, const void *v, void *o,
                                 const Shape &s, float sm_scale, const uint8_t *block_mask,
                                 cudaStream_t st, bool causal = false, const float *addend = nullptr,
                                 const SeqTable &seq = SeqTable())
{
    const WsLayout L = ws_layout(s);
    WsLock lock;
    uint8_t *ws = nullptr;
    sa_status r = get_workspace(lock, L.total, &ws);
    if (r != SA_OK) return r;
    int8_t *q8 = reinterpret_cast<int8_t *>(ws + L.q8);
    int8_t *k8 = reinterpret_cast<int8_t *>(ws + L.k8);
    uint8_t *v8 = ws + L.v8;
    float *sq = reinterpret_cast<float *>(ws + L.sq);
    float *sk = reinterpret_cast<float *>(ws + L.sk);
    float *sv = reinterpret_cast<float *>(ws + L.sv);
    if (launch_quantize_qk(q, k, s, q8, sq, k8, sk, reinterpret_cast<float *>(ws + L.kmean),
                           reinterpret_cast<double *>(ws + L.kpart), st, seq) != cudaSuccess)
        return SA_ERR_CUDA;
    if (launch_quantize_v(v, s, v8, sv, reinterpret_cast<uint32_t *>(ws + L.vamax), st, seq) !=
        cudaSuccess)
        return SA_ERR_CUDA;
    return attention_core(q8, sq, k8, sk, v8, sv, o, s, sm_scale, block_mask, st, causal, addend, seq);
}

// ------------------------------------------------------------------ host-buffer pipeline
//
// sa_attn_fwd_host: the heads (b, h) are independent, so the B*H heads are cut into chunks
// of consecutive heads; the upload of chunk c+1 and the download of chunk c-1 run on two
// library streams while chunk c is computed on the caller's stream.  Chunk c holds at most
// c + 1 heads (then the full chunk size): the first upload, which nothing overlaps, stays
// one head long, and each later upload still fits under the computation before it.  Two staging slots per
// device alternate between chunks; events order each slot's reuse:
//   upload(c)   waits compute(c-2)   (its inputs were read)
//   compute(c)  waits upload(c) and download(c-2) (its output slot was copied out)
//   download(c) waits compute(c)
// and the caller's stream finally waits for both slots' last download.

constexpr size_t kHostChunkTensorBytes = size_t(64) << 20;  // target bytes of q per chunk

struct HostPipe {
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t entry = nullptr, in[2] = {nullptr, nullptr}, comp[2] = {nullptr, nullptr},
                out[2] = {nullptr, nullptr};
    void *buf = nullptr;
    size_t bytes = 0;
};
static HostPipe g_hp[64];
static std::mutex g_hp_mutex;

static sa_status host_pipe_init(HostPipe &P)
{
    if (P.h2d) return SA_OK;
    if (cudaStreamCreateWithFlags(&P.h2d, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&P.d2h, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&P.entry, cudaEventDisableTiming) != cudaSuccess)
        return SA_ERR_CUDA;
    for (int i = 0; i < 2; ++i)
        if (cudaEventCreateWithFlags(&P.in[i], cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&P.comp[i], cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&P.out[i], cudaEventDisableTiming) != cudaSuccess)
            return SA_ERR_CUDA;
    return SA_OK;
}

static sa_status attn_fwd_host_pipeline(const void *q, const void *k, const void *v, void *o,
                                        const Shape &s, float sm_scale, const uint8_t *mask,
                                        cudaStream_t st)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_hp_mutex);
    HostPipe &P = g_hp[dev];
    sa_status r = host_pipe_init(P);
    if (r != SA_OK) return r;

    const int64_t BH = s.BH();
    const size_t head_bytes = size_t(s.N) * kD * 2;                  // one head of q (bf16)
    const size_t head_mask = size_t(s.nq()) * size_t(s.nk());        // one head of the mask
    const int64_t hc = std::max<int64_t>(1, std::min<int64_t>(BH, int64_t(kHostChunkTensorBytes / head_bytes)));
    const size_t t_bytes = align256(size_t(hc) * head_bytes);
    const size_t m_bytes = mask ? align256(size_t(hc) * head_mask) : 0;
    const size_t slot = 4 * t_bytes + m_bytes;
    if (P.bytes < 2 * slot) {
        if (P.buf) {
            // earlier calls may still use the old staging buffer
            if (cudaDeviceSynchronize() != cudaSuccess) return SA_ERR_CUDA;
            cudaFree(P.buf);
            P.buf = nullptr;
            P.bytes = 0;
        }
        if (cudaMalloc(&P.buf, 2 * slot) != cudaSuccess) {
            cudaGetLastError();
            return SA_ERR_OOM;
        }
        P.bytes = 2 * slot;
    }
    const uint8_t *hq = static_cast<const uint8_t *>(q), *hk = static_cast<const uint8_t *>(k),
                  *hv = static_cast<const uint8_t *>(v);
    uint8_t *ho = static_cast<uint8_t *>(o);
    // the inputs may be written by work already enqueued on the caller's stream
    if (cudaEventRecord(P.entry, st) != cudaSuccess || cudaStreamWaitEvent(P.h2d, P.entry, 0) != cudaSuccess)
        return SA_ERR_CUDA;
    int last[2] = {0, 0};
    for (int64_t h0 = 0, c = 0, hn = 0; h0 < BH; h0 += hn, ++c) {
        const int i = int(c & 1);
        hn = std::min<int64_t>(std::min<int64_t>(hc, c + 1), BH - h0);
        const size_t nb = size_t(hn) * head_bytes, off = size_t(h0) * head_bytes;
        uint8_t *base = static_cast<uint8_t *>(P.buf) + size_t(i) * slot;
        uint8_t *dq = base, *dk = base + t_bytes, *dv = base + 2 * t_bytes, *dout = base + 3 * t_bytes;
        uint8_t *dm = mask ? base + 4 * t_bytes : nullptr;
        bool ok = cudaStreamWaitEvent(P.h2d, P.comp[i], 0) == cudaSuccess &&
                  cudaMemcpyAsync(dq, hq + off, nb, cudaMemcpyHostToDevice, P.h2d) == cudaSuccess &&
                  cudaMemcpyAsync(dk, hk + off, nb, cudaMemcpyHostToDevice, P.h2d) == cudaSuccess &&
                  cudaMemcpyAsync(dv, hv + off, nb, cudaMemcpyHostToDevice, P.h2d) == cudaSuccess &&
                  (!mask || cudaMemcpyAsync(dm, mask + size_t(h0) * head_mask, size_t(hn) * head_mask,
                                            cudaMemcpyHostToDevice, P.h2d) == cudaSuccess) &&
                  cudaEventRecord(P.in[i], P.h2d) == cudaSuccess &&
                  cudaStreamWaitEvent(st, P.in[i], 0) == cudaSuccess &&
                  cudaStreamWaitEvent(st, P.out[i], 0) == cudaSuccess;
        if (!ok) return SA_ERR_CUDA;
        Shape sc;
        sc.B = 1;
        sc.H = int(hn);
        sc.N = s.N;
        r = attn_fwd_device(dq, dk, dv, dout, sc, sm_scale, dm, st);
        if (r != SA_OK) return r;
        ok = cudaEventRecord(P.comp[i], st) == cudaSuccess &&
             cudaStreamWaitEvent(P.d2h, P.comp[i], 0) == cudaSuccess &&
             cudaMemcpyAsync(ho + off, dout, nb, cudaMemcpyDeviceToHost, P.d2h) == cudaSuccess &&
             cudaEventRecord(P.out[i], P.d2h) == cudaSuccess;
        if (!ok) return SA_ERR_CUDA;
        last[i] = 1;
    }
    // the call is complete on the caller's stream once the outputs are in host memory
    for (int i = 0; i < 2; ++i)
        if (last[i] && cudaStreamWaitEvent(st, P.out[i], 0) != cudaSuccess) return SA_ERR_CUDA;
    return SA_OK;
}

// Variable-length groups: sequences taken longest first (ord, a stable order); a group
// runs as one prologue and one attention launch over heads padded to its longest sequence,
// and takes the next sequence while the padded size stays within twice the group's own
// (or below 2^20 padded token-heads, where the padding costs little) and its heads stay a
// valid grid dimension.
struct VarlenGroup {
    int first, count;  // positions in ord
    int64_t nmax;
};
static void varlen_groups(int nseq, const int *seqlens, int H, std::vector<int> &ord, std::vector<VarlenGroup> &groups)
{
    ord.resize(static_cast<size_t>(nseq));
    std::iota(ord.begin(), ord.end(), 0);
    std::stable_sort(ord.begin(), ord.end(), [&](int a, int b) { return seqlens[a] > seqlens[b]; });
    groups.clear();
    for (int g0 = 0; g0 < nseq;) {
        const int64_t nmax = seqlens[ord[g0]], pmax = padded_len(nmax);
        int64_t own = pmax;
        int cnt = 1;
        while (g0 + cnt < nseq) {
            const int64_t own2 = own + padded_len(seqlens[ord[g0 + cnt]]), pad2 = int64_t(cnt + 1) * pmax;
            if (pad2 > 2 * own2 && pad2 * H > (int64_t(1) << 20)) break;
            if (int64_t(cnt + 1) * H > 65535) break;
            own = own2;
            ++cnt;
        }
        groups.push_back({g0, cnt, nmax});
        g0 += cnt;
    }
}

}  // namespace sa

using namespace sa;

extern "C" {

sa_status sa_quantize_qk(const void *q, const void *k, int B, int H, int N, int d,
                         int8_t *q_i8, float *q_scale, int8_t *k_i8, float *k_scale,
                         float *k_mean, void *stream)
{
    Shape s;
    sa_status r = check_shape(B, H, N, d, &s);
    if (r != SA_OK) return r;
    if ((r = check_ptrs({q, k, q_i8, q_scale, k_i8, k_scale, k_mean})) != SA_OK) return r;
    if ((r = check_device()) != SA_OK) return r;
    const WsLayout L = ws_layout(s);
    WsLock lock;
    uint8_t *ws = nullptr;
    if ((r = get_workspace(lock, L.total, &ws)) != SA_OK) return r;
    cudaError_t e = launch_quantize_qk(q, k, s, q_i8, q_scale, k_i8, k_scale, k_mean,
                                       reinterpret_cast<double *>(ws + L.kpart),
                                       static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

sa_status sa_quantize_qk_noalloc(const void *q, const void *k, int B, int H, int N, int d,
                                 int8_t *q_i8, float *q_scale, int8_t *k_i8, float *k_scale,
                                 float *k_mean, void *stream)
{
    Shape s;
    sa_status r = check_shape(B, H, N, d, &s);
    if (r != SA_OK) return r;
    if ((r = check_ptrs({q, k, q_i8, q_scale, k_i8, k_scale, k_mean})) != SA_OK) return r;
    if (size_t(s.BH()) * size_t(s.nchunks()) * kD > kNoAllocPartialDoubles) return SA_ERR_SCRATCH_LIMIT;
    if ((r = check_device()) != SA_OK) return r;
    double *part = nullptr;
    if (noalloc_kpart(&part) != cudaSuccess) return SA_ERR_CUDA;
    cudaError_t e = launch_quantize_qk(q, k, s, q_i8, q_scale, k_i8, k_scale, k_mean, part,
                                       static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

sa_status sa_quantize_v(const void *v, int B, int H, int N, int d, uint8_t *v_fp8_t,
                        float *v_scale, void *stream)
{
    Shape s;
    sa_status r = check_shape(B, H, N, d, &s);
    if (r != SA_OK) return r;
    if ((r = check_ptrs({v, v_fp8_t, v_scale})) != SA_OK) return r;
    if ((r = check_device()) != SA_OK) return r;
    const WsLayout L = ws_layout(s);
    WsLock lock;
    uint8_t *ws = nullptr;
    if ((r = get_workspace(lock, L.total, &ws)) != SA_OK) return r;
    cudaError_t e = launch_quantize_v(v, s, v_fp8_t, v_scale,
                                      reinterpret_cast<uint32_t *>(ws + L.vamax),
                                      static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

// d = 64: the inputs are zero-padded to 128 channels in the workspace (after the d = 128
// call's own region, `inner` bytes), the d = 128 path runs on them, and O's first 64
// channels are copied out.  Zero channels add nothing to S, leave every block maximum (and
// so every scale and code) unchanged, have mean 0 and V scale 0: the result is the d = 64
// definition's.  The kernel's time is set by the softmax per score, not by d.
static sa_status attn_fwd_d64(const void *q, const void *k, const void *v, void *o, int B, int H, int N,
                              float sm_scale, const uint8_t *block_mask, bool causal, cudaStream_t st)
{
    Shape s;
    sa_status r = check_shape(B, H, N, kD, &s);
    if (r != SA_OK) return r;
    size_t inner = align256(ws_layout(s).total);
    if (causal) inner = align256(inner + size_t(s.BH()) * size_t(s.nq()) * size_t(s.nk()));
    const int64_t rows = s.BH() * s.N;
    const size_t tb = align256(size_t(rows) * kD * 2);
    WsLock lock;
    uint8_t *ws = nullptr;
    if ((r = get_workspace(lock, inner + 4 * tb, &ws)) != SA_OK) return r;
    uint8_t *pq = ws + inner, *pk = pq + tb, *pv = pk + tb, *po = pv + tb;
    if (launch_pad_heads(q, rows, pq, st) != cudaSuccess || launch_pad_heads(k, rows, pk, st) != cudaSuccess ||
        launch_pad_heads(v, rows, pv, st) != cudaSuccess)
        return SA_ERR_CUDA;
    if (causal && block_mask) {
        const size_t attn = align256(ws_layout(s).total);
        if (launch_causal_mask(block_mask, s, ws + attn, st) != cudaSuccess) return SA_ERR_CUDA;
        r = attn_fwd_device(pq, pk, pv, po, s, sm_scale, ws + attn, st, true);
    } else if (causal) {
        r = attn_fwd_device(pq, pk, pv, po, s, sm_scale, nullptr, st, true);
    } else {
        r = attn_fwd_device(pq, pk, pv, po, s, sm_scale, block_mask, st);
    }
    if (r != SA_OK) return r;
    return launch_unpad_heads(po, rows, o, st) == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

// A keep mask row of a masked attention call holds at most kMaskedAttnMaxKeyBlocks blocks.
static sa_status check_mask_len(const Shape &s, const void *mask)
{
    return mask && s.nk() > kMaskedAttnMaxKeyBlocks ? SA_ERR_UNSUPPORTED : SA_OK;
}

static sa_status check_d64_call(int B, int H, int N, float sm_scale, std::initializer_list<const void *> ptrs,
                                const void *mask)
{
    Shape s;
    sa_status r = check_shape(B, H, N, kD, &s);
    if (r != SA_OK) return r;
    if ((r = check_mask_len(s, mask)) != SA_OK) return r;
    if (!(sm_scale > 0.0f) || !std::isfinite(sm_scale)) return SA_ERR_INVALID_ARG;
    if ((r = check_ptrs(ptrs)) != SA_OK) return r;
    return check_device();
}

sa_status sa_attn_fwd(const void *q, const void *k, const void *v, void *o, int B, int H,
                      int N, int d, float sm_scale, const uint8_t *block_mask, void *stream)
{
    if (d == kD / 2) {
        const sa_status r = check_d64_call(B, H, N, sm_scale, {q, k, v, o}, block_mask);
        return r != SA_OK ? r
                          : attn_fwd_d64(q, k, v, o, B, H, N, sm_scale, block_mask, false,
                                         static_cast<cudaStream_t>(stream));
    }
    Shape s;
    sa_status r = check_shape(B, H, N, d, &s);
    if (r != SA_OK) return r;
    if (!(sm_scale > 0.0f) || !std::isfinite(sm_scale)) return SA_ERR_INVALID_ARG;
    if ((r = check_ptrs({q, k, v, o})) != SA_OK) return r;
    if ((r = check_mask_len(s, block_mask)) != SA_OK) return r;
    if ((r = check_device()) != SA_OK) return r;
    return attn_fwd_device(q, k, v, o, s, sm_scale, block_mask, static_cast<cudaStream_t>(stream));
}

sa_status sa_attn_fwd_host(const void *q, const void *k, const void *v, void *o, int B, int H,
                           int N, int d, float sm_scale, const uint8_t *block_mask, void *stream)
{
    Shape s;
    sa_status r = check_shape(B, H, N, d, &s);
    if (r != SA_OK) return r;
    if (!(sm_scale > 0.0f) || !std::isfinite(sm_scale)) return SA_ERR_INVALID_ARG;
    if ((r = check_ptrs({q, k, v, o})) != SA_OK) return r;
    if ((r = check_mask_len(s, block_mask)) != SA_OK) return r;
    if ((r = check_device()) != SA_OK) return r;
    return attn_fwd_host_pipeline(q, k, v, o, s, sm_scale, block_mask, static_cast<cudaStream_t>(stream));
}

sa_status sa_attn_fwd_quantized(const int8_t *q_i8, const float *q_scale, const int8_t *k_i8,
                                const float *k_scale, const uint8_t *v_fp8_t,
                                const float *v_scale, void *o, int B, int H, int N, int d,
                                float sm_scale, const uint8_t *block_mask, void *stream)
{
    Shape s;
    sa_status r = check_shape(B, H, N, d, &s);
    if (r != SA_OK) return r;
    if (!(sm_scale > 0.0f) || !std::isfinite(sm_scale)) return SA_ERR_INVALID_ARG;
    if ((r = check_ptrs({q_i8, k_i8, v_fp8_t, o})) != SA_OK) return r;
    if (!q_scale || !k_scale || !v_scale) return SA_ERR_INVALID_ARG;
    if ((r = check_mask_len(s, block_mask)) != SA_OK) return r;
    if ((r = check_device()) != SA_OK) return r;
    return attention_core(q_i8, q_scale, k_i8, k_scale, v_fp8_t, v_scale, o, s, sm_scale,
                          block_mask, static_cast<cudaStream_t>(stream));
}

sa_status sa_block_mask(const void *q, const void *k, int B, int H, int N, int d, int keep_per_row,
                        int keep_diagonal, uint8_t *block_mask, void *stream)
{
    Shape s;
    sa_status r = check_shape(B, H, N, d, &s);
    if (r != SA_OK) return r;
    if (keep_per_row < 1) return SA_ERR_INVALID_ARG;
    if (!q || !k || !block_mask) return SA_ERR_INVALID_ARG;
    if ((r = check_ptrs({q, k})) != SA_OK) return r;
    if (s.nk() > kMaskMaxKeyBlocks) return SA_ERR_UNSUPPORTED;
    if ((r = check_device()) != SA_OK) return r;
    const size_t qb = align256(size_t(s.BH() * s.nq()) * kD * 4), kb = align256(size_t(s.BH() * s.nk()) * kD * 4);
    const size_t sb = size_t(s.BH() * s.nq()) * size_t(s.nk()) * 8;
    WsLock lock;
    uint8_t *ws = nullptr;
    if ((r = get_workspace(lock, qb + kb + sb, &ws)) != SA_OK) return r;
    float *qbar = reinterpret_cast<float *>(ws), *kbar = reinterpret_cast<float *>(ws + qb);
    double *scores = reinterpret_cast<double *>(ws + qb + kb);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (launch_pool_qk(q, k, s, qbar, kbar, st) != cudaSuccess) return SA_ERR_CUDA;
    return launch_block_select(qbar, kbar, scores, s, keep_per_row, keep_diagonal ? 1 : 0, block_mask, st) == cudaSuccess
               ? SA_OK
               : SA_ERR_CUDA;
}

sa_status sa_debug_pool(const void *q, const void *k, int B, int H, int N, int d, float *qbar,
                        float *kbar, void *stream)
{
    Shape s;
    sa_status r = check_shape(B, H, N, d, &s);
    if (r != SA_OK) return r;
    if ((r = check_ptrs({q, k, qbar, kbar})) != SA_OK) return r;
    if ((r = check_device()) != SA_OK) return r;
    return launch_pool_qk(q, k, s, qbar, kbar, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SA_OK
                                                                                              : SA_ERR_CUDA;
}

sa_status sa_w8a8_quantize(const void *x, int rows, int cols, int8_t *codes, float *scales, void *stream)
{
    if (rows < 1 || cols < 1) return SA_ERR_INVALID_ARG;
    if (cols % 8 != 0 || cdiv(rows, 128) > 65535) return SA_ERR_UNSUPPORTED;
    sa_status r = check_ptrs({x, codes, scales});
    if (r != SA_OK) return r;
    if ((r = check_device()) != SA_OK) return r;
    return launch_w8a8_quantize(x, rows, cols, codes, scales, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SA_OK
               : SA_ERR_CUDA;
}

static sa_status w8a8_gemm_checked(const int8_t *x_codes, const float *x_scales, const int8_t *w_codes,
                                   const float *w_scales, int M, int N, int K, void *y, cudaStream_t st)
{
    const int64_t kpad = cdiv(K, 128) * 128;
    CUtensorMap tx, tw;
    if (!encode_tmap_2d_u8(&tx, x_codes, uint64_t(kpad), uint64_t(M), uint64_t(kpad), 128, kW8a8BoxRows,
                           CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tmap_2d_u8(&tw, w_codes, uint64_t(kpad), uint64_t(N), uint64_t(kpad), 128, kW8a8BoxRows,
                           CU_TENSOR_MAP_SWIZZLE_128B))
        return SA_ERR_CUDA;
    return launch_w8a8_gemm(tx, tw, x_scales, w_scales, M, N, int(kpad / 128), y, st) == cudaSuccess ? SA_OK
                                                                                                : SA_ERR_CUDA;
}

// need_k8: x is quantised here from bf16 rows, read 8 values (16 bytes) at a time
static sa_status check_w8a8_sizes(int M, int N, int K, bool need_k8)
{
    if (M < 1 || N < 1 || K < 1) return SA_ERR_INVALID_ARG;
    if (N % 8 != 0 || (need_k8 && K % 8 != 0)) return SA_ERR_UNSUPPORTED;
    // TMA row coordinates and tile counts are 32-bit; grid rows of the quantiser <= 65535
    if (cdiv(M, 128) > 65535 || cdiv(N, 128) > 65535) return SA_ERR_UNSUPPORTED;
    return SA_OK;
}

sa_status sa_w8a8_gemm(const int8_t *x_codes, const float *x_scales, const int8_t *w_codes, const float *w_scales,
                       int M, int N, int K, void *y, void *stream)
{
    sa_status r = check_w8a8_sizes(M, N, K, false);
    if (r != SA_OK) return r;
    if ((r = check_ptrs({x_codes, x_scales, w_codes, w_scales, y})) != SA_OK) return r;
    if ((r = check_device()) != SA_OK) return r;
    return w8a8_gemm_checked(x_codes, x_scales, w_codes, w_scales, M, N, K, y, static_cast<cudaStream_t>(stream));
}

sa_status sa_w8a8_linear(const void *x, const int8_t *w_codes, const float *w_scales, int M, int N, int K,
                         void *y, void *stream)
{
    sa_status r = check_w8a8_sizes(M, N, K, true);
    if (r != SA_OK) return r;
    if ((r = check_ptrs({x, w_codes, w_scales, y})) != SA_OK) return r;
    if ((r = check_device()) != SA_OK) return r;
    const size_t kpad = size_t(cdiv(K, 128)) * 128;
    const size_t cb = align256(size_t(M) * kpad), sb = size_t(cdiv(M, 128)) * size_t(kpad / 128) * 4;
    WsLock lock;
    uint8_t *ws = nullptr;
    if ((r = get_workspace(lock, cb + sb, &ws)) != SA_OK) return r;
    int8_t *xc = reinterpret_cast<int8_t *>(ws);
    float *xs = reinterpret_cast<float *>(ws + cb);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (launch_w8a8_quantize(x, M, K, xc, xs, st) != cudaSuccess) return SA_ERR_CUDA;
    return w8a8_gemm_checked(xc, xs, w_codes, w_scales, M, N, K, y, st);
}

static sa_status check_sla(const Shape &s, int phi, std::initializer_list<const void *> ptrs)
{
    if (phi != 0 && phi != 1) return SA_ERR_INVALID_ARG;
    if (s.nk() > kMaskMaxKeyBlocks) return SA_ERR_UNSUPPORTED;
    return check_ptrs(ptrs);
}

sa_status sa_sla_linear(const void *q, const void *k, const void *v, const uint8_t *classes, int B, int H, int N,
                        int d, int phi, const float *proj, float *out, void *stream)
{
    Shape s;
    sa_status r = check_shape(B, H, N, d, &s);
    if (r != SA_OK) return r;
    if (!classes) return SA_ERR_INVALID_ARG;
    if ((r = check_sla(s, phi, {q, k, v, out})) != SA_OK) return r;
    if (proj && (r = check_ptrs({proj})) != SA_OK) return r;
    if ((r = check_device()) != SA_OK) return r;
    WsLock lock;
    uint8_t *ws = nullptr;
    if ((r = get_workspace(lock, sla_workspace_bytes(s), &ws)) != SA_OK) return r;
    return launch_sla_linear(q, k, v, classes, s, phi, proj, ws, out, static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? SA_OK
               : SA_ERR_CUDA;
}

sa_status sa_sla_fwd(const void *q, const void *k, const void *v, void *o, int B, int H, int N, int d,
                     float sm_scale, const uint8_t *classes, int phi, const float *proj, void *stream)
{
    Shape s;
    sa_status r = check_shape(B, H, N, d, &s);
    if (r != SA_OK) return r;
    if (!(sm_scale > 0.0f) || !std::isfinite(sm_scale) || !classes) return SA_ERR_INVALID_ARG;
    if ((r = check_sla(s, phi, {q, k, v, o})) != SA_OK) return r;
    if (proj && (r = check_ptrs({proj})) != SA_OK) return r;
    if ((r = check_device()) != SA_OK) return r;
    // workspace: [attention prologue | keep mask | linear-branch states | linear part, fp32]
    const size_t attn = align256(ws_layout(s).total);
    const size_t nmask = size_t(s.BH()) * size_t(s.nq()) * size_t(s.nk());
    const size_t mb = align256(nmask), sb = align256(sla_workspace_bytes(s));
    const size_t lb = size_t(s.BH()) * size_t(s.N) * kD * sizeof(float);
    WsLock lock;
    uint8_t *ws = nullptr;
    if ((r = get_workspace(lock, attn + mb + sb + lb, &ws)) != SA_OK) return r;
    uint8_t *keep = ws + attn;
    float *lin = reinterpret_cast<float *>(ws + attn + mb + sb);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (launch_sla_critical(classes, int64_t(nmask), keep, st) != cudaSuccess) return SA_ERR_CUDA;
    // the linear part first, in fp32; the sparse part's epilogue adds it to O before O's
    // only rounding to bf16
    if (launch_sla_linear(q, k, v, classes, s, phi, proj, ws + attn + mb, lin, st) != cudaSuccess)
        return SA_ERR_CUDA;
    return attn_fwd_device(q, k, v, o, s, sm_scale, keep, st, false, lin);
}

sa_status sa_attn_fwd_causal(const void *q, const void *k, const void *v, void *o, int B, int H, int N, int d,
                             float sm_scale, const uint8_t *block_mask, void *stream)
{
    if (d == kD / 2) {
        const sa_status r = check_d64_call(B, H, N, sm_scale, {q, k, v, o}, block_mask);
        return r != SA_OK ? r
                          : attn_fwd_d64(q, k, v, o, B, H, N, sm_scale, block_mask, true,
                                         static_cast<cudaStream_t>(stream));
    }
    Shape s;
    sa_status r = check_shape(B, H, N, d, &s);
    if (r != SA_OK) return r;
    if (!(sm_scale > 0.0f) || !std::isfinite(sm_scale)) return SA_ERR_INVALID_ARG;
    if ((r = check_ptrs({q, k, v, o})) != SA_OK) return r;
    if ((r = check_mask_len(s, block_mask)) != SA_OK) return r;
    if ((r = check_device()) != SA_OK) return r;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // without a keep mask the pair kernel runs the causal pattern itself
    if (!block_mask) return attn_fwd_device(q, k, v, o, s, sm_scale, nullptr, st, true);
    // with one: workspace [attention prologue | keep mask intersected with the causal blocks]
    const size_t attn = align256(ws_layout(s).total);
    WsLock lock;
    uint8_t *ws = nullptr;
    if ((r = get_workspace(lock, attn + size_t(s.BH()) * size_t(s.nq()) * size_t(s.nk()), &ws)) != SA_OK) return r;
    if (launch_causal_mask(block_mask, s, ws + attn, st) != cudaSuccess) return SA_ERR_CUDA;
    return attn_fwd_device(q, k, v, o, s, sm_scale, ws + attn, st, true);
}

sa_status sa_attn_fwd_varlen(const void *q, const void *k, const void *v, void *o, int nseq, const int *seqlens,
                             int H, int d, float sm_scale, int causal, void *stream)
{
    if (nseq < 1 || !seqlens || H < 1) return SA_ERR_INVALID_ARG;
    if (d != kD) return SA_ERR_UNSUPPORTED;
    if (!(sm_scale > 0.0f) || !std::isfinite(sm_scale)) return SA_ERR_INVALID_ARG;
    sa_status r = check_ptrs({q, k, v, o});
    if (r != SA_OK) return r;
    // every sequence is valid on its own; start[i] = its first token in the packed batch
    std::vector<int64_t> start(static_cast<size_t>(nseq) + 1, 0);
    for (int i = 0; i < nseq; ++i) {
        Shape s;
        if ((r = check_shape(1, H, seqlens[i], d, &s)) != SA_OK) return r;
        start[i + 1] = start[i] + seqlens[i];
    }
    if (start[nseq] > INT_MAX / 8 || int64_t(H) * start[nseq] > INT64_MAX / kD) return SA_ERR_INVALID_ARG;
    std::vector<int> ord;
    std::vector<VarlenGroup> groups;
    varlen_groups(nseq, seqlens, H, ord, groups);
    size_t need = 0;
    for (const VarlenGroup &g : groups) {
        Shape s;
        if ((r = check_shape(g.count, H, int(g.nmax), d, &s)) != SA_OK) return r;
        need = std::max(need, align256(ws_layout(s).total));
    }
    // device table after the largest group's workspace: the lengths in group order, then
    // the first row (of d elements) of every head in q, k, v and o
    const size_t lb = align256(size_t(nseq) * sizeof(int)), tb = lb + size_t(nseq) * H * sizeof(int64_t);
    std::vector<uint8_t> table(tb, 0);
    int *lens = reinterpret_cast<int *>(table.data());
    int64_t *rows = reinterpret_cast<int64_t *>(table.data() + lb);
    for (int i = 0; i < nseq; ++i) {
        const int sq = ord[i];
        lens[i] = seqlens[sq];
        for (int h = 0; h < H; ++h) rows[size_t(i) * H + h] = int64_t(H) * start[sq] + int64_t(h) * seqlens[sq];
    }
    if ((r = check_device()) != SA_OK) return r;
    WsLock lock;
    uint8_t *ws = nullptr;
    if ((r = get_workspace(lock, need + tb, &ws)) != SA_OK) return r;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((r = upload_table(table.data(), tb, ws + need, st)) != SA_OK) return r;
    const int *dlens = reinterpret_cast<const int *>(ws + need);
    const int64_t *drows = reinterpret_cast<const int64_t *>(ws + need + lb);
    for (const VarlenGroup &g : groups) {
        Shape s;
        check_shape(g.count, H, int(g.nmax), d, &s);
        SeqTable t;
        t.len = dlens + g.first;
        t.row = drows + size_t(g.first) * H;
        t.H = H;
        if ((r = attn_fwd_device(q, k, v, o, s, sm_scale, nullptr, st, causal != 0, nullptr, t)) != SA_OK) return r;
    }
    return SA_OK;
}

int sa_debug_varlen_groups(int nseq, const int *seqlens, int H, int *group_of)
{
    if (nseq < 1 || !seqlens || !group_of || H < 1) return -1;
    for (int i = 0; i < nseq; ++i)
        if (seqlens[i] < 1) return -1;
    std::vector<int> ord;
    std::vector<VarlenGroup> groups;
    varlen_groups(nseq, seqlens, H, ord, groups);
    for (size_t g = 0; g < groups.size(); ++g)
        for (int i = 0; i < groups[g].count; ++i) group_of[ord[size_t(groups[g].first + i)]] = int(g);
    return int(groups.size());
}

sa_status sa_debug_qk_s32(const int8_t *q_i8, const int8_t *k_i8, int B, int H, int N, int d,
                          int32_t *s_out, void *stream)
{
    Shape s;
    sa_status r = check_shape(B, H, N, d, &s);
    if (r != SA_OK) return r;
    if ((r = check_ptrs({q_i8, k_i8, s_out})) != SA_OK) return r;
    if ((r = check_device()) != SA_OK) return r;
    CUtensorMap tq, tk;
    const uint64_t rows = uint64_t(s.BH() * s.Npad());
    if (!encode_tmap_2d_u8(&tq, q_i8, kD, rows, kD, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tmap_2d_u8(&tk, k_i8, kD, rows, kD, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return SA_ERR_CUDA;
    return launch_debug_qk_s32(tq, tk, int(s.BH()), int(s.Npad()), s_out,
                               static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SA_OK
               : SA_ERR_CUDA;
}

sa_status sa_debug_wait_timeout(int timeout_us, void *stream)
{
    if (timeout_us < 1 || timeout_us > 10000000) return SA_ERR_INVALID_ARG;
    sa_status r = check_device();
    if (r != SA_OK) return r;
    return launch_debug_wait_timeout(timeout_us, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SA_OK
               : SA_ERR_CUDA;
}

sa_status sa_debug_mma_peak(int kind, int reps, void *stream)
{
    if ((kind != 0 && kind != 1) || reps < 1 || reps > (1 << 20)) return SA_ERR_INVALID_ARG;
    sa_status r = check_device();
    if (r != SA_OK) return r;
    return launch_mma_peak(kind, reps, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

sa_status sa_get_device_status(void)
{
    int st = 0, st_w8a8 = 0, st_peak = 0, st_sla = 0;
    if (read_and_clear_status(&st) != cudaSuccess || read_and_clear_w8a8_status(&st_w8a8) != cudaSuccess ||
        read_and_clear_peak_status(&st_peak) != cudaSuccess || read_and_clear_sla_status(&st_sla) != cudaSuccess)
        return SA_ERR_CUDA;
    return st == 0 && st_w8a8 == 0 && st_peak == 0 && st_sla == 0 ? SA_OK : SA_ERR_DEVICE_TIMEOUT;
}

const char *sa_status_string(sa_status s)
{
    switch (s) {
    case SA_OK: return "SA_OK";
    case SA_ERR_INVALID_ARG: return "SA_ERR_INVALID_ARG";
    case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED";
    case SA_ERR_MISALIGNED: return "SA_ERR_MISALIGNED";
    case SA_ERR_CUDA: return "SA_ERR_CUDA";
    case SA_ERR_OOM: return "SA_ERR_OOM";
    case SA_ERR_DEVICE_TIMEOUT: return "SA_ERR_DEVICE_TIMEOUT";
    case SA_ERR_SCRATCH_LIMIT: return "SA_ERR_SCRATCH_LIMIT";
    }
    return "SA_ERR_UNKNOWN";
}

size_t sa_workspace_bytes(int B, int H, int N, int d)
{
    Shape s;
    if (check_shape(B, H, N, d == kD / 2 ? kD : d, &s) != SA_OK) return 0;
    if (d != kD / 2) return ws_layout(s).total;
    // d = 64: the d = 128 workspace, then the four zero-padded copies of q, k, v and o
    return align256(ws_layout(s).total) + 4 * align256(size_t(s.BH()) * size_t(s.N) * kD * 2);
}

sa_status sa_release_workspace(void)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SA_ERR_CUDA;
    WsLock lock(g_ws_mutex);
    DeviceWs &w = g_ws[dev];
    if (w.ptr) {
        if (cudaDeviceSynchronize() != cudaSuccess) return SA_ERR_CUDA;
        cudaFree(w.ptr);
        w.ptr = nullptr;
        w.bytes = 0;
    }
    HostStage &h = g_stage[dev];
    if (h.ptr) {
        if (cudaEventSynchronize(h.ev) != cudaSuccess) return SA_ERR_CUDA;
        cudaFreeHost(h.ptr);
        h.ptr = nullptr;
        h.bytes = 0;
    }
    return SA_OK;
}

int64_t sa_padded_len(int N) { return N < 1 ? 0 : sa::padded_len(N); }

}  // extern "C"
