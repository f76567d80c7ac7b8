// sa_internal.h -- launchers shared between the C-ABI layer and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace sa {

constexpr int kD = 128;      // head dimension
constexpr int kQBlk = 128;   // query tokens per quantisation block / tile / mask row
constexpr int kKBlk = 64;    // key tokens per quantisation block / mask column
constexpr int kMeanChunk = 1024;  // tokens per partial-sum block of the K mean

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t padded_len(int64_t n) { return cdiv(n, kQBlk) * kQBlk; }

struct Shape {
    int64_t B, H, N;
    int64_t BH() const { return B * H; }
    int64_t Npad() const { return padded_len(N); }
    int64_t nq() const { return cdiv(N, kQBlk); }
    int64_t nk() const { return cdiv(N, kKBlk); }
    int64_t nchunks() const { return cdiv(N, kMeanChunk); }
};

// Packed variable-length batches: head bh = b * H + h holds len[b] tokens, whose rows (d
// elements each) start at row[bh] in q, k, v and o; the quantised buffers, scales and
// partial sums keep the uniform layout of a Shape whose N is the longest sequence.  With
// len == nullptr every head has Shape::N tokens at row bh * N.
struct SeqTable {
    const int *len = nullptr;
    const int64_t *row = nullptr;
    int H = 1;
};
__device__ __forceinline__ int seq_tokens(const SeqTable &t, int64_t bh, int N)
{
    return t.len ? __ldg(t.len + bh / t.H) : N;
}
__device__ __forceinline__ int64_t seq_row0(const SeqTable &t, int64_t bh, int N)
{
    return t.len ? __ldg(t.row + bh) : bh * int64_t(N);
}

// ---- prologue (sa_prologue.cu)
cudaError_t launch_quantize_qk(const void *q, const void *k, const Shape &s, int8_t *q_i8,
                               float *q_scale, int8_t *k_i8, float *k_scale, float *k_mean,
                               double *k_partial /* [BH, nchunks, d] */, cudaStream_t st,
                               const SeqTable &seq = SeqTable());
cudaError_t launch_quantize_v(const void *v, const Shape &s, uint8_t *v_t, float *v_scale,
                              uint32_t *v_amax_bits /* [BH, d] */, cudaStream_t st,
                              const SeqTable &seq = SeqTable());
// d = 64 calls: [rows][64] bf16 -> [rows][128] with zero upper channels, and back.
cudaError_t launch_pad_heads(const void *src, int64_t rows, void *dst, cudaStream_t st);
cudaError_t launch_unpad_heads(const void *src, int64_t rows, void *dst, cudaStream_t st);
// Fixed scratch for the allocation-free Q/K quantisation: [BH, nchunks, d] fp64 must fit.
constexpr size_t kNoAllocPartialDoubles = (size_t(4) << 20) / sizeof(double);  // 4 MiB
cudaError_t noalloc_kpart(double **out);

// ---- attention (sa_attn.cu)
struct AttnArgs {
    CUtensorMap tm_q, tm_k, tm_v;
    const float *q_scale, *k_scale, *v_scale;
    const uint8_t *mask;
    __nv_bfloat16 *o;
    int BH, N, Npad, nq, nk;
    float sm_scale;
    int causal = 0;  // row r keeps only the keys t <= r (mask must then be set)
    // fp32 [B,H,N,d] added to O before its single rounding to bf16 (masked calls), or null
    const float *addend = nullptr;
    SeqTable seq;  // variable-length heads (unmasked calls only)
};
cudaError_t launch_attention(const AttnArgs &a, cudaStream_t st);
cudaError_t launch_debug_qk_s32(const CUtensorMap &tm_q, const CUtensorMap &tm_k, int BH,
                                int Npad, int32_t *s_out, cudaStream_t st);
cudaError_t launch_debug_wait_timeout(int timeout_us, cudaStream_t st);
// ---- block-mask producer (sa_mask.cu)
constexpr int kMaskMaxKeyBlocks = 4096;  // key blocks per mask row the selector sorts in shared memory
constexpr int kMaskedAttnMaxKeyBlocks = 16384;  // key blocks per mask row of a masked attention call
cudaError_t launch_pool_qk(const void *q, const void *k, const Shape &s, float *qbar, float *kbar,
                           cudaStream_t st);
// Causal block mask: out[bh][i][j] = (j <= 2i + 1) && (user == null || user[bh][i][j] != 0).
cudaError_t launch_causal_mask(const uint8_t *user, const Shape &s, uint8_t *out, cudaStream_t st);
cudaError_t launch_block_select(const float *qbar, const float *kbar, double *scores, const Shape &s,
                                int keep_per_row, int keep_diagonal, uint8_t *mask, cudaStream_t st);
// ---- W8A8 linear layer (sa_w8a8.cu)
// x bf16 [rows, cols] (cols % 8 == 0) -> codes int8 [rows, kpad = 128 * ceil(cols / 128)]
// (padding columns zero) and scales fp32 [ceil(rows / 128), ceil(cols / 128)].
cudaError_t launch_w8a8_quantize(const void *x, int64_t rows, int64_t cols, int8_t *codes, float *scales,
                                 cudaStream_t st);
// y bf16 [M, N] (N % 8 == 0) from the codes behind tm_x ([M, kpad]) and tm_w ([N, kpad]),
// both encoded with a box of 128 bytes x kW8a8BoxRows rows and 128-byte swizzle, and their
// block scales, nkb = kpad / 128.
constexpr int kW8a8BoxRows = 128;
cudaError_t launch_w8a8_gemm(const CUtensorMap &tm_x, const CUtensorMap &tm_w, const float *sx,
                             const float *sw, int M, int N, int nkb, void *y, cudaStream_t st);
cudaError_t read_and_clear_w8a8_status(int *status);
// ---- SLA linear branch (sa_sla.cu)
// Workspace of launch_sla_linear: the per-key-block and per-query-block states of one group
// of heads (fp32), at most about 1 GiB whatever the number of heads.
size_t sla_workspace_bytes(const Shape &s);
// The branch for all rows: fp32 out [B,H,N,d].  classes uint8 [B,H,nq,nk] (1 = marginal);
// proj fp32 [d][d] or null; workspace of sla_workspace_bytes(s) bytes, 256-byte aligned.
cudaError_t launch_sla_linear(const void *q, const void *k, const void *v, const uint8_t *classes, const Shape &s,
                              int phi, const float *proj, void *workspace, float *out, cudaStream_t st);
// keep[e] = classes[e] >= 2 (the sparse part's block mask), n entries.
cudaError_t launch_sla_critical(const uint8_t *classes, int64_t n, uint8_t *keep, cudaStream_t st);
cudaError_t read_and_clear_sla_status(int *status);
// Reads and clears the device status word of the current device (synchronous).
cudaError_t read_and_clear_status(int *status);
// ---- measured tensor-core peak (sa_peak.cu): one CTA per SM, reps chains of four
// M128 N256 K32 MMAs (kind 0: i8, kind 1: e4m3), 2*128*256*32 operations per MMA
cudaError_t launch_mma_peak(int kind, int reps, cudaStream_t st);
cudaError_t read_and_clear_peak_status(int *status);

// ---- tensor maps (sa_api.cu)
bool encode_tmap_2d_u8(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                       uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                       CUtensorMapSwizzle swizzle);
// fp32 [d2][d1][d0] (d0 contiguous), box {box0, box1, 1}, zero fill
bool encode_tmap_3d_f32(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                        uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1,
                        CUtensorMapSwizzle swizzle);

}  // namespace sa
