/*
 * sa.h -- C ABI of libsa.so, a B200 (sm_100a) SageAttention-style low-bit attention
 * forward with optional SLA-style block sparsity.
 *
 * The method (sources, by page and section):
 *   - "AIGC weekend special 5.10: full-stack optimisation of visual-generation
 *     inference", section 1 (TurboDiffusion), 1.2 Method, item (1): SageAttention2++
 *     quantises Q and K to low bit and runs Q.K^T on tensor cores; item (2): SLA
 *     sparse attention is orthogonal to it and runs on top of it.
 *   - "Video-Generation-101: inference systems", kernel paragraph and reference [3]:
 *     format / thread-granularity / accumulation co-design with outlier smoothing.
 *   - "Video-Generation-101 research log", section 5.5 table: INT4/INT8 Q.K^T with
 *     FP8/FP16 P.V.
 *   - NetEase article on the TurboDiffusion release, "attention acceleration" section
 *     and the SLA figure caption: only the critical blocks of the attention weights
 *     get exact (sparse) attention.
 * Numerical definition implemented (the pages give the outline; each detail they leave
 * open is stated here):
 *   per (b,h): mean_k[c] = fp32( sum_t K[t,c] (fp64) / N );
 *   Q: per 128-token block, scale_q = max|q| / 127, q_i8 = rint_even(q / scale_q);
 *   K: ks = K - mean_k (fp32), per 64-token block scale_k = max|ks| / 127,
 *      k_i8 = rint_even(ks / scale_k); codes clamp to [-127, 127]; zero block -> scale 0;
 *   V: per channel scale_v = max_t |v| / 448, v_fp8 = e4m3_rn_satfinite(v / scale_v);
 *   S = q_i8 . k_i8^T exact in int32; s = S * (scale_q * scale_k * sm_scale);
 *   online softmax in fp32 over the kept 64-key blocks, two blocks per step;
 *   p8 = e4m3(448 * exp(s - m)); l = sum of p8; acc = sum p8 * v_fp8 (fp32);
 *   O = acc * scale_v / l (bf16), 0 for a row with no kept key.
 *
 * Conventions for every entry point:
 *   - Tensors are contiguous row-major.  q, k, v, o: bf16 [B,H,N,d].  d must be 128, except
 *     that sa_attn_fwd and sa_attn_fwd_causal also take d = 64: they zero-pad q, k, v to 128
 *     channels in the workspace and copy out o's first 64, which gives exactly the d = 64
 *     definition (zero channels add nothing to S and leave every scale and code unchanged).
 *     Npad = 128 * ceil(N/128); nq = ceil(N/128); nk = ceil(N/64).  B * H <= 65535 (the
     heads are a grid dimension of the prologue kernels), else SA_ERR_UNSUPPORTED.
 *   - Device pointers are owned by the caller; the library never frees them.  All
 *     pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Every
 *     call only enqueues work on that stream and returns without synchronising, except
 *     sa_get_device_status, which synchronises the device.
 *   - Argument errors are detected on the host before any launch; outputs are then
 *     untouched.  Launch failures return SA_ERR_CUDA.  Device-side bounded waits that
 *     expire set a device status word read by sa_get_device_status.
 *   - Block mask: uint8 [B,H,nq,nk], nonzero keeps the (128-query x 64-key) block; NULL
 *     keeps every block.  Masked blocks are neither loaded nor computed.  With a mask,
 *     nk <= 16384 (N <= 1,048,576), else SA_ERR_UNSUPPORTED.
 *   - Library workspace.  The entry points marked "uses the library workspace" keep their
 *     intermediates (quantised Q/K/V, scales, partial sums, masks, SLA states) in ONE
 *     buffer per device, owned by the library and grown on demand.  Growing it
 *     synchronises the device and frees the old buffer; the library holds a lock from a
 *     call's workspace request until that call's launches are enqueued, so calls from
 *     several host threads cannot free memory another call is about to use.  The buffer
 *     is NOT per stream: two such calls in flight at once on different streams of one
 *     device overwrite each other's intermediates and give wrong results without any
 *     error.  Order such calls on one stream (or with events).  sa_attn_fwd_quantized,
 *     sa_debug_qk_s32 and sa_w8a8_gemm use no workspace; sa_quantize_qk_noalloc uses its
 *     own fixed array (see there).
 *   - The library caches per-device state (the workspace, tensor-map encoder, kernel
 *     attributes and the scratch array's address) for the life of the process: do not use
 *     it across cudaDeviceReset.
 */
#ifndef SA_H
#define SA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SA_OK = 0,
    SA_ERR_INVALID_ARG = 1,    /* null pointer, non-positive size, size overflow */
    SA_ERR_UNSUPPORTED = 2,    /* d != 128, B * H > 65535, or no sm_100 device */
    SA_ERR_MISALIGNED = 3,     /* a pointer is not 16-byte aligned */
    SA_ERR_CUDA = 4,           /* a CUDA runtime/driver call or launch failed */
    SA_ERR_OOM = 5,            /* the library workspace could not be allocated */
    SA_ERR_DEVICE_TIMEOUT = 6, /* a device-side bounded wait expired */
    SA_ERR_SCRATCH_LIMIT = 7   /* the problem needs more than a fixed scratch array holds */
} sa_status;

/* Quantise Q and smooth + quantise K (the Q/K half of the prologue).
 * Sources: TurboDiffusion digest 1.2(1) (Q/K to INT8 on tensor cores);
 * Video-Generation-101 reference [3] (outlier smoothing).
 * Outputs (device, caller-owned):
 *   q_i8 int8 [B,H,Npad,d] (rows >= N zero), q_scale fp32 [B,H,nq],
 *   k_i8 int8 [B,H,Npad,d] (rows >= N zero), k_scale fp32 [B,H,nk],
 *   k_mean fp32 [B,H,d].
 * Results are bit-identical to the definition above (the K mean whenever the fp64 sum
 * of the column is exact, which holds for bf16 inputs of ordinary range).
 * Uses the library workspace for per-block fp64 partial sums of K. */
sa_status sa_quantize_qk(const void *q, const void *k, int B, int H, int N, int d,
                         int8_t *q_i8, float *q_scale, int8_t *k_i8, float *k_scale,
                         float *k_mean, void *stream);

/* sa_quantize_qk without any device allocation.  The method's pages have no counterpart
 * for this; it exists for callers that cannot call cudaMalloc: code whose device memory is
 * owned by a host framework or memory pool that has already reserved the device (so a
 * library allocation would fail or fragment it), and latency-critical loops that cannot
 * afford cudaMalloc's implicit synchronisation.  The library workspace that sa_quantize_qk
 * grows on first use is replaced by a fixed 4 MiB device array compiled into the library
 * (each GPU that loads the library holds it until the process exits).
 * Arguments, outputs and results are exactly those of sa_quantize_qk.
 * Limit: B * H * ceil(N / 1024) <= 4096 (e.g. 40 heads of up to 104,448 tokens); larger
 * problems return SA_ERR_SCRATCH_LIMIT before any launch.
 * The first call on each device looks up the array's device address (a synchronous
 * runtime call), so make that first call before any stream capture.  All calls share the
 * array: calls whose kernels overlap on the same device (e.g. on two streams) race on it
 * and must be ordered by the caller.  No state carries over between calls. */
sa_status sa_quantize_qk_noalloc(const void *q, const void *k, int B, int H, int N, int d,
                                 int8_t *q_i8, float *q_scale, int8_t *k_i8, float *k_scale,
                                 float *k_mean, void *stream);

/* Quantise V to FP8 e4m3 per channel, stored transposed (the V half of the prologue).
 * Source: Video-Generation-101 research log 5.5 (FP8 P.V).
 * Outputs: v_fp8_t uint8 e4m3 [B,H,d,Npad] (keys contiguous, keys >= N zero),
 *          v_scale fp32 [B,H,d].  Bit-identical to the definition above.
 * Uses the library workspace for per-channel maxima. */
sa_status sa_quantize_v(const void *v, int B, int H, int N, int d, uint8_t *v_fp8_t,
                        float *v_scale, void *stream);

/* Full forward: prologue into the library workspace, then the fused attention kernel.
 * Sources: all of the above; FlashAttention tiling (digest timeline, 2022.06) for the
 * online softmax.  o: bf16 [B,H,N,d] (device, caller-owned).  sm_scale: the logit scale,
 * normally 1/sqrt(d).  block_mask: see conventions, or NULL.
 * The workspace is library-owned, per device, grow-only (cudaMalloc on first use or
 * growth, so the first call at a new size must not be inside a stream capture). */
sa_status sa_attn_fwd(const void *q, const void *k, const void *v, void *o, int B, int H,
                      int N, int d, float sm_scale, const uint8_t *block_mask, void *stream);

/* Causal forward: as sa_attn_fwd, where query row r attends to the keys t <= r only.
 * Source: "AIGC weekend special 5.10", sections 4 (HiAR: causal generation over all blocks
 * at each denoising step) and 6 (SDVG: autoregressive video diffusion).  Reading: the
 * quantisation is unchanged (scales over all N tokens); a tile of 128 queries visits its
 * kept blocks j <= 2i + 1 in pairs, as without causality, and keys after the row are left
 * out of the max and the sums.  block_mask (or NULL) is intersected with the causal
 * block pattern.  Uses the library workspace (plus nq * nk bytes per head for the mask). */
sa_status sa_attn_fwd_causal(const void *q, const void *k, const void *v, void *o, int B, int H, int N,
                             int d, float sm_scale, const uint8_t *block_mask, void *stream);

/* Variable-length batch: nseq independent sequences of lengths seqlens[i] (host array,
 * each >= 1), packed back to back: sequence i is a [1, H, N_i, d] bf16 block of q, k, v
 * and o starting H * (N_0 + ... + N_{i-1}) * d elements in.  Each sequence is computed as
 * sa_attn_fwd (causal = 0) or sa_attn_fwd_causal without a mask (causal != 0) would compute
 * it alone, with the same results.  Every block must start 16-byte aligned (H * N_i * d is a
 * multiple of 8 elements, which d = 128 guarantees).  All sizes are checked before the first
 * launch.  The sequences are taken longest first in groups: a group takes the next sequence
 * while its heads padded to its longest stay within twice their own padded size, or below
 * 2^20 padded token-heads; each group is one prologue and one attention launch (the kernels
 * read every head's own length from a table), so a batch of short sequences is a single
 * launch of each kernel.  The workspace is sized for the largest group, plus the table,
 * which is uploaded through a library-owned page-locked host buffer. */
sa_status sa_attn_fwd_varlen(const void *q, const void *k, const void *v, void *o, int nseq, const int *seqlens,
                             int H, int d, float sm_scale, int causal, void *stream);

/* Debug (host only, no CUDA call): the groups sa_attn_fwd_varlen forms for these lengths.
 * group_of[i] (host array of nseq) receives the group of sequence i; groups are numbered
 * in launch order (longest sequences first).  Returns the number of groups, or -1 on bad
 * arguments (nseq < 1, H < 1, a null pointer or a length < 1). */
int sa_debug_varlen_groups(int nseq, const int *seqlens, int H, int *group_of);

/* Full forward on HOST buffers: q, k, v, o bf16 [B,H,N,d] and block_mask (or NULL) in host
 * memory, page-locked for the copies to overlap (pageable memory works but serialises).
 * The B*H heads are independent, so they are processed in chunks of consecutive heads
 * (one head first, then growing by one head per chunk up to about 64 MB of q, so that the
 * first upload, which nothing overlaps, is short): the upload of chunk c+1 and the
 * download of chunk c-1 run on two library-owned streams while chunk c runs sa_attn_fwd's
 * prologue and kernel on `stream`.  The call returns after enqueueing; the work is
 * complete when `stream` reaches the point after the call (o is then filled), and q, k,
 * v, o and block_mask must stay valid until then.  Device staging (two chunks) is
 * library-owned, per device and grow-only, like the workspace.  Calls for the same device
 * from several host threads are serialised.  Results are identical to sa_attn_fwd on the
 * same inputs. */
sa_status sa_attn_fwd_host(const void *q, const void *k, const void *v, void *o, int B, int H,
                           int N, int d, float sm_scale, const uint8_t *block_mask, void *stream);

/* The fused attention kernel alone, on already-quantised inputs (the layouts written by
 * sa_quantize_qk and sa_quantize_v).  For callers that reuse quantised K/V across
 * queries, and for timing the kernel without the prologue.  Allocates nothing. */
sa_status sa_attn_fwd_quantized(const int8_t *q_i8, const float *q_scale, const int8_t *k_i8,
                                const float *k_scale, const uint8_t *v_fp8_t,
                                const float *v_scale, void *o, int B, int H, int N, int d,
                                float sm_scale, const uint8_t *block_mask, void *stream);

/* Block-mask producer: the keep mask block_mask uint8 [B,H,ceil(N/128),ceil(N/64)] (device,
 * caller-owned, fully written) for q, k bf16 [B,H,N,d] (device).
 * Sources: NetEase article on the TurboDiffusion release, attention-acceleration section,
 * SLA figure caption (selection from predicted, compressed attention weights);
 * "Video-Generation-101 research log" section 5.5, SpargeAttention row (a block selector
 * ahead of the sparse low-bit kernel).  Reading: Q is mean-pooled per 128-token block and
 * K per 64-token block (fp64 sums in token order, rounded to fp32); each pair is scored by
 * the fp64 dot product of the two means (channel order); row i keeps its keep_per_row
 * highest-scoring key blocks (ties: lower block index), plus blocks 2i and 2i+1 when
 * keep_diagonal is non-zero.  keep_per_row >= 1 (values >= ceil(N/64) keep every block).
 * Needs ceil(N/64) <= 4096 (else SA_ERR_UNSUPPORTED).  Uses the library workspace for the
 * block means and the scores.  The result is a deterministic function of q and k. */
sa_status sa_block_mask(const void *q, const void *k, int B, int H, int N, int d, int keep_per_row,
                        int keep_diagonal, uint8_t *block_mask, void *stream);

/* Debug: the block means of sa_block_mask, qbar fp32 [B,H,ceil(N/128),d] and kbar fp32
 * [B,H,ceil(N/64),d] (device, caller-owned).  Allocates nothing. */
sa_status sa_debug_pool(const void *q, const void *k, int B, int H, int N, int d, float *qbar,
                        float *kbar, void *stream);

/* ---- W8A8 linear layer: y = x . w^T with x [M,K] and w [N,K] both quantised to INT8 with
 * one scale per 128 x 128 block, products on the INT8 tensor cores.
 * Sources: NetEase article on the TurboDiffusion release, W8A8 linear-layer section
 * (weights and activations of the linear layers to 8 bits, 128 x 128 blocks, INT8 tensor
 * cores); "AIGC weekend special 5.10" section 1.2 Method, item (4).
 * Definition (readings where the pages are silent): a block's scale is max|x| / 127 over
 * the block (fp32), codes rint_even(x / scale) clamped to [-127, 127], a zero block has
 * scale 0 and codes 0; K is padded with zero codes to kpad = 128 * ceil(K/128);
 * y[m,n] = bf16_rn( acc ), acc = 0, then for each k-block b = 0, 1, ... in order:
 *   acc = fmaf( (float) S_b, sx[m/128][b] * sw[n/128][b], acc )   (fp32, one rounding),
 * S_b the exact int32 dot product of the 128 codes of block b. */

/* Block quantisation of x bf16 [rows, cols] (device): codes int8 [rows, 128*ceil(cols/128)]
 * (padding columns written as zero), scales fp32 [ceil(rows/128), ceil(cols/128)] (both
 * device, caller-owned).  cols % 8 == 0 and ceil(rows/128) <= 65535, else SA_ERR_UNSUPPORTED.
 * Bit-identical to the definition above.  Allocates nothing.  Used for the weights once and
 * for the activations on every call. */
sa_status sa_w8a8_quantize(const void *x, int rows, int cols, int8_t *codes, float *scales, void *stream);

/* y bf16 [M, N] (device, caller-owned) from quantised x (codes [M, kpad], scales
 * [ceil(M/128), kpad/128]) and w (codes [N, kpad], scales [ceil(N/128), kpad/128]), as laid
 * out by sa_w8a8_quantize.  N % 8 == 0, else SA_ERR_UNSUPPORTED.
 * Bit-identical to the definition above.  Allocates nothing. */
sa_status sa_w8a8_gemm(const int8_t *x_codes, const float *x_scales, const int8_t *w_codes,
                       const float *w_scales, int M, int N, int K, void *y, void *stream);

/* The linear layer: quantises x bf16 [M, K] into the library workspace, then sa_w8a8_gemm
 * with the pre-quantised weight.  K % 8 == 0 and N % 8 == 0, else SA_ERR_UNSUPPORTED.
 * Workspace rules as for sa_attn_fwd. */
sa_status sa_w8a8_linear(const void *x, const int8_t *w_codes, const float *w_scales, int M, int N,
                         int K, void *y, void *stream);

/* ---- SLA: sparse quantised attention on the critical blocks plus linear attention on the
 * marginal blocks.
 * Sources: NetEase article on the TurboDiffusion release, attention-acceleration section
 * (SLA combines sparse and linear attention; its figure caption splits the attention
 * weights into three classes handled at different costs); "AIGC weekend special 5.10"
 * section 1.2 Method item (2) (SLA runs on top of SageAttention).  The pages give no
 * formula for the linear part.  Reading: block classes come per (128-query block,
 * 64-key block) in classes uint8 [B,H,nq,nk] (device): 0 = negligible (skipped), 1 =
 * marginal (linear attention), >= 2 = critical (sparse quantised attention).  The linear
 * part is kernelised linear attention over the keys of the row's marginal blocks,
 *     O_lin[r] = sum_t w_t v_t / sum_t w_t,  w_t = phi(q_r) . phi(k_t)   (0 if no such key),
 * with phi = SA_PHI_SOFTMAX (softmax over the d features of a row) or SA_PHI_ELU1
 * (elu(x) + 1), projected by W: out[r][c] = sum_e W[c][e] O_lin[r][e], W fp32 [d][d]
 * (device; NULL = identity; in SLA a trained layer).  Evaluated in fp32 in the factorised
 * form phi(q)^T (sum_t phi(k_t) v_t^T) / (phi(q) . sum_t phi(k_t)): per 64-key block
 * the state sum_t phi(k_t) [v_t, 1]^T (128 x 129), then per 128-query block the sum of
 * its marginal blocks' states on the tensor cores (TF32 products of the 0/1 class matrix
 * with the states split into two TF32 terms, about 22 significant bits each, fp32
 * accumulation), then the division and projection.
 * Needs ceil(N/64) <= 4096 (else SA_ERR_UNSUPPORTED).  Uses the library workspace for
 * the states of one group of heads at a time: 69,632 bytes per 64-key block and per
 * 128-query block of a head, at most about 1 GiB (one head at least). */
enum { SA_PHI_SOFTMAX = 0, SA_PHI_ELU1 = 1 };

/* The linear branch alone: out fp32 [B,H,N,d] (device, caller-owned) = W O_lin. */
sa_status sa_sla_linear(const void *q, const void *k, const void *v, const uint8_t *classes, int B, int H,
                        int N, int d, int phi, const float *proj, float *out, void *stream);

/* The SLA forward: o bf16 [B,H,N,d] = the quantised attention of sa_attn_fwd restricted to
 * the critical blocks (a row without one gives 0), plus the projected linear branch,
 * added in fp32 and rounded once to bf16.  The linear branch runs first, into the library
 * workspace in fp32 (a further 4 * d bytes per query token), and the sparse part's
 * epilogue adds it to O before O's only rounding. */
sa_status sa_sla_fwd(const void *q, const void *k, const void *v, void *o, int B, int H, int N, int d,
                     float sm_scale, const uint8_t *classes, int phi, const float *proj, void *stream);

/* Debug: the int32 S = q_i8 . k_i8^T tiles computed by the same tcgen05 INT8 path the
 * attention kernel uses, stored to s_out int32 [B,H,Npad,Npad] (padded rows/keys
 * included).  For bit-exact checks on small problems only.  Allocates nothing. */
sa_status sa_debug_qk_s32(const int8_t *q_i8, const int8_t *k_i8, int B, int H, int N, int d,
                          int32_t *s_out, void *stream);

/* Debug: launches a one-CTA kernel whose mbarrier wait can never complete, bounded by
 * timeout_us microseconds; the kernel then records SA_ERR_DEVICE_TIMEOUT in the device
 * status word and returns.  Exercises the failure path without faulting the GPU. */
sa_status sa_debug_wait_timeout(int timeout_us, void *stream);


/* Synchronises the current device, returns and clears its device status word
 * (SA_OK or SA_ERR_DEVICE_TIMEOUT), or SA_ERR_CUDA if synchronisation failed. */
sa_status sa_get_device_status(void);

/* Human-readable name of a status code (static string). */
const char *sa_status_string(sa_status s);

/* Bytes of library workspace sa_attn_fwd needs for this problem size, d = 128 or 64 (0 on
 * bad sizes).  Causal calls with a keep mask add B * H * ceil(N/128) * ceil(N/64) bytes. */
size_t sa_workspace_bytes(int B, int H, int N, int d);

/* Measurement aid (no counterpart on the pages): the device's own 8-bit tensor-core rate,
 * the denominator of the attention kernel's roofline.  Launches one CTA per SM; each
 * issues `reps` chains of four tcgen05 MMAs of M = 128, N = 256, K = 32 (one K = 128
 * contraction, the way the attention kernel issues them) from shared memory into tensor
 * memory: kind 0 = kind::i8 (int8 x int8 -> int32), kind 1 = kind::f8f6f4 with e4m3
 * operands (-> fp32).  The caller times the launch (e.g. with CUDA events on `stream`);
 * it performs SMs * reps * 4 * 2*128*256*32 operations.  reps in [1, 2^20]; the final
 * bounded wait reports through sa_get_device_status. */
sa_status sa_debug_mma_peak(int kind, int reps, void *stream);

/* Frees the current device's workspace (synchronises the device first). */
sa_status sa_release_workspace(void);

/* Padded token count Npad = 128 * ceil(N/128) (0 for N < 1). */
int64_t sa_padded_len(int N);

#ifdef __cplusplus
}
#endif

#endif /* SA_H */
