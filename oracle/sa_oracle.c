/*
 * sa_oracle.c -- CPU oracle for the SageAttention-style low-bit attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and its
 * Python binding) may include, link, load or call this file.  Only the test-suite,
 * the smoke check and the CPU-baseline leg of the benchmark use it.  It shares no
 * code, header, table or constant generator with the CUDA path.
 *
 * Plain, slow, single-threaded C11.  Build with
 *     gcc -O2 -std=c11 -fno-fast-math -ffp-contract=off -fPIC -shared
 * so that every float operation is one IEEE-754 binary32 (or binary64) operation
 * rounded to nearest-even, in the order written (x86-64 SSE arithmetic, no FMA
 * contraction, no re-association).
 *
 * What the method computes (sources, by page and section):
 *   - "AIGC weekend special 5.10: full-stack optimisation of visual-generation
 *     inference", section 1 (TurboDiffusion), 1.2 Method, item (1): SageAttention2++
 *     quantises Q and K to low bit (INT4/INT8) and runs Q.K^T on tensor cores; item (2):
 *     SLA sparse attention runs on top of it.
 *   - "Video-Generation-101: inference systems", kernel paragraph: SageAttention2 is a
 *     co-design of number format, thread granularity and accumulation; reference [3]
 *     names "thorough outlier smoothing".
 *   - "Video-Generation-101 research log", section 5.5 table, SageAttention2 row:
 *     INT4/INT8 Q.K^T, FP8/FP16 P.V.
 *   - NetEase article on the TurboDiffusion release, "attention acceleration" section:
 *     SageAttention2++ variant; SLA keeps "critical" blocks of the attention weights
 *     (figure caption).
 *   - FlashAttention (IO-aware tiled attention, same digest's timeline, 2022.06):
 *     online softmax over key blocks.
 * The pages give the outline only; the numerical definition implemented here is:
 *   K smoothed by subtracting its per-channel mean over tokens; Q quantised to INT8 per
 *   128-token block and K per 64-token block with scale = max|x|/127 and round-half-even;
 *   S = q_i8 . k_i8^T exact in int32, dequantised by scale_q * scale_k * sm_scale;
 *   online softmax in fp32; P scaled by 448 and cast to FP8 e4m3; V cast to FP8 e4m3
 *   per channel with scale = max|v|/448; P.V accumulated in fp32.
 * Readings where the pages are silent are marked "reading:" below.
 *
 * Parity pins (tests/test_oracle_*.py): e4m3 codec against the OCP FP8 definition and
 * a library cast; quantiser closed forms (exact-integer case, tie cases, block
 * boundaries, shift invariance); attention closed forms (N = 1, identical keys,
 * dominant key), invariants (rows sum to one, constant V columns), brute force against
 * the fp64 exact attention below.  Block-mask producer (end of file): block means against
 * numpy, pooled scores against an fp64 einsum, the selection rule against an independent
 * stable sort (ties included), invariants (scaling Q, swapping key blocks) and a planted
 * key block (tests/test_oracle_mask.py).  W8A8 linear layer (end of file): quantiser
 * against a numpy restatement, exact-integer and single-k-block closed forms, zero blocks,
 * error against the fp64 product (tests/test_oracle_w8a8.py).  SLA linear branch (end of
 * file): the factorised form in numpy, closed forms (one key, identical keys, no marginal
 * block), invariants (constant V columns, W = identity vs W applied afterwards) and the
 * class semantics (tests/test_oracle_sla.py).
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define QBLK 128 /* query tokens per quantisation block and per mask row */
#define KBLK 64  /* key tokens per quantisation block and per mask column */

static int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }
static int64_t padded_len(int64_t n) { return cdiv64(n, QBLK) * QBLK; }

static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------------------------
 * FP8 e4m3 (OCP 8-bit floating point specification, E4M3 variant): 1 sign bit, 4
 * exponent bits with bias 7, 3 mantissa bits.  No infinities; exponent 1111 with
 * mantissa 111 is NaN, so the largest finite magnitude is 1.75 * 2^8 = 448.  Exponent
 * field 0 holds subnormals m/8 * 2^-6 = m * 2^-9.
 * ---------------------------------------------------------------------------------- */

/* Magnitude of the non-negative code c (0..126), exactly, as a double. */
static double e4m3_magnitude(int c)
{
    int e = (c >> 3) & 15;
    int m = c & 7;
    if (e == 0) return ldexp((double)m, -9);
    return ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
}

float sa_oracle_e4m3_to_f32(uint8_t b)
{
    int mag = b & 0x7F;
    if (mag == 0x7F) return NAN;
    double v = e4m3_magnitude(mag);
    return (float)((b & 0x80) ? -v : v);
}

/* Round to nearest, ties to the even code, saturating to +-448 ("satfinite").
 * reading: values at or beyond the largest finite magnitude clamp to it; NaN maps
 * to the NaN code (never reached from finite inputs). */
uint8_t sa_oracle_e4m3_from_f32(float x)
{
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    /* largest code lo in [0,126] whose magnitude is <= a (codes increase with value) */
    int lo = 0, hi = 126;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (e4m3_magnitude(mid) <= a) lo = mid; else hi = mid - 1;
    }
    if (e4m3_magnitude(lo) == a) return (uint8_t)(sign | lo);
    int up = lo + 1; /* magnitude(up) > a and up <= 126 because a < 448 */
    double dlo = a - e4m3_magnitude(lo);
    double dup = e4m3_magnitude(up) - a;
    int c;
    if (dlo < dup) c = lo;
    else if (dup < dlo) c = up;
    else c = (lo % 2 == 0) ? lo : up; /* tie: the code whose mantissa LSB is 0 */
    return (uint8_t)(sign | c);
}

/* ------------------------------------------------------------------------------------
 * INT8 code of x under scale s: round-half-even of the IEEE quotient x/s, clamped to
 * [-127, 127].  reading: the quotient is an IEEE fp32 division (not x * (1/s)); a zero
 * scale (all-zero block) gives code 0.
 * ---------------------------------------------------------------------------------- */
static int8_t int8_code(float x, float s)
{
    if (s == 0.0f) return 0;
    float r = nearbyintf(x / s); /* FE_TONEAREST: ties to even */
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

/* Per-channel mean of one head's K over its N tokens.
 * reading: the sum runs in fp64 over t = 0..N-1 in order, is divided by N in fp64 and
 * rounded once to fp32.  *all_exact is cleared when some channel's fp64 running sum was
 * not exact (checked with Knuth's TwoSum error term), i.e. when another summation order
 * could give a different fp64 sum. */
static void k_mean_head(const uint16_t *k, int64_t N, int d, float *mean, int *all_exact)
{
    for (int c = 0; c < d; ++c) {
        double s = 0.0;
        int exact = 1;
        for (int64_t t = 0; t < N; ++t) {
            double x = (double)bf16_to_f32(k[t * d + c]);
            double sum = s + x;
            /* TwoSum: err is the exact rounding error of s + x */
            double bp = sum - s;
            double ap = sum - bp;
            double err = (s - ap) + (x - bp);
            if (err != 0.0) exact = 0;
            s = sum;
        }
        mean[c] = (float)(s / (double)N);
        if (!exact) *all_exact = 0;
    }
}

/* Q: per (b,h) and 128-token block i, scale_q = max|q|/127 over the block's valid
 * tokens and all channels; q_i8 = code(q, scale_q).  K: smoothed ks = k - mean_k[c]
 * (one fp32 subtraction), then per 64-token block scale_k = max|ks|/127 and
 * k_i8 = code(ks, scale_k).  Rows from N up to the padded length are zero.
 * Layouts: q,k bf16 [B,H,N,d]; q_i8,k_i8 [B,H,Npad,d]; q_scale [B,H,nq];
 * k_scale [B,H,nk]; k_mean [B,H,d].  Returns 1 when every K mean came from an exact
 * fp64 sum, else 0. */
int sa_oracle_quantize_qk(const uint16_t *q, const uint16_t *k, int B, int H, int N, int d,
                          int8_t *q_i8, float *q_scale, int8_t *k_i8, float *k_scale,
                          float *k_mean)
{
    fesetround(FE_TONEAREST);
    const int64_t Npad = padded_len(N);
    const int64_t nq = cdiv64(N, QBLK), nk = cdiv64(N, KBLK);
    int all_exact = 1;
    float *ks = (float *)malloc(sizeof(float) * (size_t)N * (size_t)d);
    for (int64_t bh = 0; bh < (int64_t)B * H; ++bh) {
        const uint16_t *qh = q + bh * N * d;
        const uint16_t *kh = k + bh * N * d;
        int8_t *q8 = q_i8 + bh * Npad * d;
        int8_t *k8 = k_i8 + bh * Npad * d;
        memset(q8, 0, (size_t)(Npad * d));
        memset(k8, 0, (size_t)(Npad * d));

        for (int64_t i = 0; i < nq; ++i) {
            int64_t t0 = i * QBLK, t1 = t0 + QBLK < N ? t0 + QBLK : N;
            float amax = 0.0f;
            for (int64_t t = t0; t < t1; ++t)
                for (int c = 0; c < d; ++c) {
                    float a = fabsf(bf16_to_f32(qh[t * d + c]));
                    if (a > amax) amax = a;
                }
            float s = amax / 127.0f;
            q_scale[bh * nq + i] = s;
            for (int64_t t = t0; t < t1; ++t)
                for (int c = 0; c < d; ++c)
                    q8[t * d + c] = int8_code(bf16_to_f32(qh[t * d + c]), s);
        }

        float *mean = k_mean + bh * d;
        k_mean_head(kh, N, d, mean, &all_exact);
        for (int64_t t = 0; t < N; ++t)
            for (int c = 0; c < d; ++c)
                ks[t * d + c] = bf16_to_f32(kh[t * d + c]) - mean[c];

        for (int64_t j = 0; j < nk; ++j) {
            int64_t t0 = j * KBLK, t1 = t0 + KBLK < N ? t0 + KBLK : N;
            float amax = 0.0f;
            for (int64_t t = t0; t < t1; ++t)
                for (int c = 0; c < d; ++c) {
                    float a = fabsf(ks[t * d + c]);
                    if (a > amax) amax = a;
                }
            float s = amax / 127.0f;
            k_scale[bh * nk + j] = s;
            for (int64_t t = t0; t < t1; ++t)
                for (int c = 0; c < d; ++c)
                    k8[t * d + c] = int8_code(ks[t * d + c], s);
        }
    }
    free(ks);
    return all_exact;
}

/* V: per (b,h) and channel c, scale_v = max_t |v|/448 over all N tokens;
 * v_fp8 = e4m3(v / scale_v), stored transposed as [B,H,d,Npad] (channel-major, keys
 * contiguous), padded keys zero.  reading: per-channel scale over the whole sequence;
 * the quotient is an IEEE fp32 division; a zero scale gives code 0. */
void sa_oracle_quantize_v(const uint16_t *v, int B, int H, int N, int d, uint8_t *v_fp8_t,
                          float *v_scale)
{
    fesetround(FE_TONEAREST);
    const int64_t Npad = padded_len(N);
    for (int64_t bh = 0; bh < (int64_t)B * H; ++bh) {
        const uint16_t *vh = v + bh * N * d;
        uint8_t *vt = v_fp8_t + bh * d * Npad;
        memset(vt, 0, (size_t)(d * Npad));
        for (int c = 0; c < d; ++c) {
            float amax = 0.0f;
            for (int64_t t = 0; t < N; ++t) {
                float a = fabsf(bf16_to_f32(vh[t * d + c]));
                if (a > amax) amax = a;
            }
            float s = amax / 448.0f;
            v_scale[bh * d + c] = s;
            for (int64_t t = 0; t < N; ++t)
                vt[c * Npad + t] = (s == 0.0f) ? 0 : sa_oracle_e4m3_from_f32(bf16_to_f32(vh[t * d + c]) / s);
        }
    }
}

/* Kept 64-key blocks of query block i, ascending.  mask is [B,H,nq,nk] uint8 with
 * nonzero = keep, or NULL (every block kept).  Returns the count. */
static int64_t kept_blocks(const uint8_t *mask, int64_t bh, int64_t i, int64_t nq, int64_t nk,
                           int64_t *out)
{
    int64_t n = 0;
    for (int64_t j = 0; j < nk; ++j)
        if (!mask || mask[(bh * nq + i) * nk + j]) out[n++] = j;
    return n;
}

/* Quantised attention for selected query rows.
 * rows: nrows pairs (bh, r) flattened as int64 [2*nrows]; out: fp32 [nrows, d].
 * group: how many kept 64-key blocks form one online-softmax step (1 or 2).
 *   reading: the pages fix the online softmax but not its step; steps are runs of
 *   `group` consecutive kept blocks in ascending order (the last run may be shorter).
 * Per step, for the step's keys t (t < N):
 *   S_t = sum_c q_i8[r,c] * k_i8[t,c]                 (int32, exact)
 *   s_t = (float)S_t * (scale_q[i] * scale_k[j(t)] * sm_scale)   (fp32, left to right)
 *   m'  = max(m, max_t s_t);  alpha = exp(m - m') (0 while m = -inf)
 *   p8_t = e4m3(448 * exp(s_t - m'))                  (decoded to fp32)
 *   l   = alpha * l + sum_t p8_t
 *   acc = alpha * acc + sum_t p8_t * v_fp8[t,c]       (fp32, keys ascending)
 * then O[r,c] = acc[c] * scale_v[c] / l, or 0 when l = 0 (no kept key).
 * reading: l sums the FP8-rounded P, the same weights that multiply V, so a constant V
 * column is reproduced and the normalised weights sum to one up to fp32 rounding.
 * reading: alpha is applied whenever the running max grows (no lazy rescaling, which
 * would push 448*P past the e4m3 range). */
static void attn_rows_impl(const int8_t *q_i8, const float *q_scale, const int8_t *k_i8,
                           const float *k_scale, const uint8_t *v_fp8_t, const float *v_scale,
                           int B, int H, int N, int d, float sm_scale, const uint8_t *mask,
                           int group, int causal, const int64_t *rows, int64_t nrows, float *out)
{
    fesetround(FE_TONEAREST);
    (void)B; (void)H;
    const int64_t Npad = padded_len(N);
    const int64_t nq = cdiv64(N, QBLK), nk = cdiv64(N, KBLK);
    int64_t *blocks = (int64_t *)malloc(sizeof(int64_t) * (size_t)nk);
    float *s = (float *)malloc(sizeof(float) * (size_t)(KBLK * (group > 0 ? group : 1)));
    int64_t *tk = (int64_t *)malloc(sizeof(int64_t) * (size_t)(KBLK * (group > 0 ? group : 1)));
    float *acc = (float *)malloc(sizeof(float) * (size_t)d);
    float *blk = (float *)malloc(sizeof(float) * (size_t)d);
    if (group < 1) group = 1;

    for (int64_t n = 0; n < nrows; ++n) {
        const int64_t bh = rows[2 * n], r = rows[2 * n + 1];
        const int64_t i = r / QBLK;
        const int8_t *qrow = q_i8 + (bh * Npad + r) * d;
        const int8_t *kh = k_i8 + bh * Npad * d;
        const uint8_t *vt = v_fp8_t + bh * d * Npad;
        const float sq = q_scale[bh * nq + i];
        int64_t nkept = kept_blocks(mask, bh, i, nq, nk, blocks);
        if (causal) {
            /* reading: causal rows keep the blocks up to their tile's diagonal pair,
             * j <= 2i + 1, so the steps are the same pairs as without causality */
            int64_t n2 = 0;
            for (int64_t g = 0; g < nkept; ++g)
                if (blocks[g] <= 2 * i + 1) blocks[n2++] = blocks[g];
            nkept = n2;
        }

        float m = -INFINITY, l = 0.0f;
        for (int c = 0; c < d; ++c) acc[c] = 0.0f;

        for (int64_t g0 = 0; g0 < nkept; g0 += group) {
            int64_t g1 = g0 + group < nkept ? g0 + group : nkept;
            int64_t nt = 0;
            float bmax = -INFINITY;
            for (int64_t g = g0; g < g1; ++g) {
                const int64_t j = blocks[g];
                const float sk = k_scale[bh * nk + j];
                for (int64_t t = j * KBLK; t < (j + 1) * KBLK && t < N && (!causal || t <= r); ++t) {
                    int32_t S = 0;
                    for (int c = 0; c < d; ++c) S += (int32_t)qrow[c] * (int32_t)kh[t * d + c];
                    float sc = sq * sk;
                    sc = sc * sm_scale;
                    s[nt] = (float)S * sc;
                    tk[nt] = t;
                    if (s[nt] > bmax) bmax = s[nt];
                    ++nt;
                }
            }
            if (nt == 0) continue;
            const float mnew = m > bmax ? m : bmax;
            const float alpha = (m == -INFINITY) ? 0.0f : expf(m - mnew);
            float psum = 0.0f;
            for (int c = 0; c < d; ++c) blk[c] = 0.0f;
            for (int64_t u = 0; u < nt; ++u) {
                float p = expf(s[u] - mnew);
                float p8 = sa_oracle_e4m3_to_f32(sa_oracle_e4m3_from_f32(448.0f * p));
                psum += p8;
                for (int c = 0; c < d; ++c)
                    blk[c] += p8 * sa_oracle_e4m3_to_f32(vt[(int64_t)c * Npad + tk[u]]);
            }
            l = alpha * l + psum;
            for (int c = 0; c < d; ++c) acc[c] = alpha * acc[c] + blk[c];
            m = mnew;
        }
        float *o = out + n * d;
        for (int c = 0; c < d; ++c) {
            const float sv = v_scale[bh * d + c];
            o[c] = (l > 0.0f) ? (acc[c] * sv) / l : 0.0f;
        }
    }
    free(blocks); free(s); free(tk); free(acc); free(blk);
}

void sa_oracle_attn_rows(const int8_t *q_i8, const float *q_scale, const int8_t *k_i8,
                         const float *k_scale, const uint8_t *v_fp8_t, const float *v_scale,
                         int B, int H, int N, int d, float sm_scale, const uint8_t *mask,
                         int group, const int64_t *rows, int64_t nrows, float *out)
{
    attn_rows_impl(q_i8, q_scale, k_i8, k_scale, v_fp8_t, v_scale, B, H, N, d, sm_scale, mask, group, 0,
                   rows, nrows, out);
}

/* Causal quantised attention: as sa_oracle_attn_rows, where row r takes only the keys
 * t <= r.  Source: "AIGC weekend special 5.10", section 4 (HiAR: every denoising step runs
 * causal generation over all blocks) and section 6 (SDVG: autoregressive video diffusion):
 * a query attends to itself and earlier tokens only.
 * reading: the quantisation is unchanged (scales over all N tokens); the online-softmax
 * steps are the pairs of kept blocks up to the tile's diagonal pair (2i, 2i+1), and keys
 * after the row are left out of the step's max and sums. */
void sa_oracle_attn_rows_causal(const int8_t *q_i8, const float *q_scale, const int8_t *k_i8,
                                const float *k_scale, const uint8_t *v_fp8_t, const float *v_scale,
                                int B, int H, int N, int d, float sm_scale, const uint8_t *mask,
                                int group, const int64_t *rows, int64_t nrows, float *out)
{
    attn_rows_impl(q_i8, q_scale, k_i8, k_scale, v_fp8_t, v_scale, B, H, N, d, sm_scale, mask, group, 1,
                   rows, nrows, out);
}

/* Exact attention in fp64 for selected rows, from the bf16 inputs, with no smoothing
 * and no quantisation: O = softmax(q.K^T * sm_scale) . V over the kept keys (mask
 * semantics as above; NULL = all keys).  out: fp64 [nrows, d]; a row with no kept key
 * gives 0. */
static void exact_rows_impl(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B,
                            int H, int N, int d, double sm_scale, const uint8_t *mask, int causal,
                            const int64_t *rows, int64_t nrows, double *out)
{
    (void)B; (void)H;
    const int64_t nq = cdiv64(N, QBLK), nk = cdiv64(N, KBLK);
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    for (int64_t n = 0; n < nrows; ++n) {
        const int64_t bh = rows[2 * n], r = rows[2 * n + 1];
        const int64_t i = r / QBLK;
        const uint16_t *qr = q + (bh * N + r) * d;
        const uint16_t *kh = k + bh * N * d;
        const uint16_t *vh = v + bh * N * d;
        double mx = -INFINITY;
        for (int64_t t = 0; t < N; ++t) {
            int keep = (!mask || mask[(bh * nq + i) * nk + t / KBLK]) && (!causal || t <= r);
            if (!keep) { s[t] = -INFINITY; continue; }
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += (double)bf16_to_f32(qr[c]) * (double)bf16_to_f32(kh[t * d + c]);
            s[t] = acc * sm_scale;
            if (s[t] > mx) mx = s[t];
        }
        double *o = out + n * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        if (mx == -INFINITY) continue;
        double den = 0.0;
        for (int64_t t = 0; t < N; ++t) {
            if (s[t] == -INFINITY) continue;
            double p = exp(s[t] - mx);
            den += p;
            for (int c = 0; c < d; ++c) o[c] += p * (double)bf16_to_f32(vh[t * d + c]);
        }
        for (int c = 0; c < d; ++c) o[c] /= den;
    }
    free(s);
}

void sa_oracle_exact_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B,
                          int H, int N, int d, double sm_scale, const uint8_t *mask,
                          const int64_t *rows, int64_t nrows, double *out)
{
    exact_rows_impl(q, k, v, B, H, N, d, sm_scale, mask, 0, rows, nrows, out);
}

/* Exact causal attention in fp64: row r over the keys t <= r (and the mask, if any). */
void sa_oracle_exact_rows_causal(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B,
                                 int H, int N, int d, double sm_scale, const uint8_t *mask,
                                 const int64_t *rows, int64_t nrows, double *out)
{
    exact_rows_impl(q, k, v, B, H, N, d, sm_scale, mask, 1, rows, nrows, out);
}

/* int32 S = q_i8 . k_i8^T for selected query rows against all Npad key rows (padded
 * keys included, which are zero codes).  rows as above; out: int32 [nrows, Npad]. */
void sa_oracle_qk_s32_rows(const int8_t *q_i8, const int8_t *k_i8, int B, int H, int N, int d,
                           const int64_t *rows, int64_t nrows, int32_t *out)
{
    (void)B; (void)H;
    const int64_t Npad = padded_len(N);
    for (int64_t n = 0; n < nrows; ++n) {
        const int64_t bh = rows[2 * n], r = rows[2 * n + 1];
        const int8_t *qr = q_i8 + (bh * Npad + r) * d;
        const int8_t *kh = k_i8 + bh * Npad * d;
        for (int64_t t = 0; t < Npad; ++t) {
            int32_t S = 0;
            for (int c = 0; c < d; ++c) S += (int32_t)qr[c] * (int32_t)kh[t * d + c];
            out[n * Npad + t] = S;
        }
    }
}

/* ------------------------------------------------------------------------------------
 * Block-mask producer: the selector ahead of the block skip.
 *
 * Sources: NetEase article on the TurboDiffusion release, attention-acceleration section,
 * SLA figure caption (the attention weights fall into three classes that are computed at
 * different costs; SLA's forward works from predicted, compressed attention weights);
 * "Video-Generation-101 research log" section 5.5 table, SpargeAttention row (a two-level
 * online filter selects blocks ahead of a sparse, low-bit kernel); "Video-Generation-101:
 * inference systems", kernel paragraph (selector, sparse layout and low-bit kernel are
 * designed together).
 * reading: the compressed weights are those of Q mean-pooled per 128-token block against
 * K mean-pooled per 64-token block (the geometry of the keep mask); a mask row keeps its
 * keep_per_row highest-scoring key blocks, ties going to the lower block index; the row
 * softmax and sm_scale are increasing in the score and leave the choice unchanged, so
 * the raw pooled dot product ranks; optionally the diagonal blocks 2i and 2i+1 (the key
 * blocks covering the query block's own tokens) are kept as well.
 * ------------------------------------------------------------------------------------ */

/*
 * Block means of x (bf16 bits [B,H,N,d]) over blocks of `blk` tokens: out fp32
 * [B,H,ceil(N/blk),d] = (float)((sum over the block's tokens t < N, t ascending, of
 * (double)x[t,c]) / (double)count).  Returns 1 if every fp64 sum was exact (TwoSum error
 * zero), else 0: the sums are then order-independent.
 */
int sa_oracle_pool(const uint16_t *x, int B, int H, int N, int d, int blk, float *out)
{
    const int64_t BH = (int64_t)B * H, nb = cdiv64(N, blk);
    int exact = 1;
    for (int64_t bh = 0; bh < BH; ++bh) {
        const uint16_t *xh = x + bh * (int64_t)N * d;
        for (int64_t b = 0; b < nb; ++b) {
            const int64_t t0 = b * blk, t1 = (t0 + blk < N) ? t0 + blk : N;
            for (int c = 0; c < d; ++c) {
                double s = 0.0, err = 0.0;
                for (int64_t t = t0; t < t1; ++t) {
                    const double v = (double)bf16_to_f32(xh[t * d + c]);
                    const double ns = s + v;
                    /* TwoSum: err is the exact rounding error of s + v */
                    const double bv = ns - s, av = ns - bv;
                    err += (s - av) + (v - bv);
                    s = ns;
                }
                if (err != 0.0) exact = 0;
                out[(bh * nb + b) * d + c] = (float)(s / (double)(t1 - t0));
            }
        }
    }
    return exact;
}

/*
 * Pooled scores: scores fp64 [BH, nq, nk] = sum over c ascending of
 * (double)qbar[i,c] * (double)kbar[j,c] (each product exact, one rounding per addition).
 */
void sa_oracle_block_scores(const float *qbar, const float *kbar, int64_t BH, int nq, int nk,
                            int d, double *scores)
{
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int i = 0; i < nq; ++i)
            for (int j = 0; j < nk; ++j) {
                const float *a = qbar + (bh * nq + i) * d, *b = kbar + (bh * nk + j) * d;
                double s = 0.0;
                for (int c = 0; c < d; ++c) {
                    const double p = (double)a[c] * (double)b[c];
                    s = s + p;
                }
                scores[(bh * nq + i) * nk + j] = s;
            }
}

/*
 * Keep mask uint8 [BH, nq, nk] from the scores: block j of row i is kept when fewer than
 * keep_per_row blocks rank before it, where j' ranks before j if its score is larger, or
 * equal with j' < j; with keep_diagonal the blocks 2i and 2i+1 (when they exist) are kept
 * too.
 */
void sa_oracle_block_mask(const double *scores, int64_t BH, int nq, int nk, int keep_per_row,
                          int keep_diagonal, uint8_t *mask)
{
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int i = 0; i < nq; ++i) {
            const double *s = scores + (bh * nq + i) * nk;
            uint8_t *m = mask + (bh * nq + i) * nk;
            for (int j = 0; j < nk; ++j) {
                int rank = 0;
                for (int jj = 0; jj < nk; ++jj)
                    if (s[jj] > s[j] || (s[jj] == s[j] && jj < j)) ++rank;
                m[j] = rank < keep_per_row ? 1 : 0;
            }
            if (keep_diagonal) {
                if (2 * i < nk) m[2 * i] = 1;
                if (2 * i + 1 < nk) m[2 * i + 1] = 1;
            }
        }
}

/* ------------------------------------------------------------------------------------
 * W8A8 linear layer: INT8 weights and activations with per-128x128-block scales.
 *
 * Sources: NetEase article on the TurboDiffusion release, "W8A8 linear-layer
 * quantisation" section (the weights and activations of the linear layers are quantised to
 * 8 bits in blocks of 128 x 128 and the products run on INT8 tensor cores); "AIGC weekend
 * special 5.10" section 1.2 Method item (4) (W8A8: weights and activations of the
 * non-attention linear layers to INT8).
 * reading: a block's scale is max|x|/127 over its (valid) elements and its codes are
 * round-half-even(x/scale) clamped to [-127, 127], as for Q and K above; y = x . w^T for
 * x [M,K] and w [N,K] (the out x in layout of a linear layer's weight); the int32 product
 * of one 128-wide k-block is exact and is added to an fp32 accumulator as
 * acc = fmaf((float)S, sx[m-block, k-block] * sw[n-block, k-block], acc), k-blocks in
 * ascending order; y is acc rounded to bf16 (nearest-even).  K is padded to a multiple of
 * 128 with zero codes.
 * ------------------------------------------------------------------------------------ */

/*
 * Codes int8 [rows, Kpad] (Kpad = 128 * ceil(cols/128), padding zero) and scales fp32
 * [ceil(rows/128), ceil(cols/128)] of x (bf16 bits [rows, cols]), per 128 x 128 block.
 */
void sa_oracle_w8a8_quantize(const uint16_t *x, int64_t rows, int64_t cols, int8_t *codes,
                             float *scales)
{
    const int64_t rb = cdiv64(rows, 128), cb = cdiv64(cols, 128), kpad = cb * 128;
    fesetround(FE_TONEAREST);
    for (int64_t i = 0; i < rows * kpad; ++i) codes[i] = 0;
    for (int64_t a = 0; a < rb; ++a)
        for (int64_t b = 0; b < cb; ++b) {
            const int64_t r0 = a * 128, r1 = r0 + 128 < rows ? r0 + 128 : rows;
            const int64_t c0 = b * 128, c1 = c0 + 128 < cols ? c0 + 128 : cols;
            float amax = 0.0f;
            for (int64_t r = r0; r < r1; ++r)
                for (int64_t c = c0; c < c1; ++c) {
                    const float v = fabsf(bf16_to_f32(x[r * cols + c]));
                    if (v > amax) amax = v;
                }
            const float s = amax / 127.0f;
            scales[a * cb + b] = s;
            for (int64_t r = r0; r < r1; ++r)
                for (int64_t c = c0; c < c1; ++c)
                    codes[r * kpad + c] = int8_code(bf16_to_f32(x[r * cols + c]), s);
        }
}

/*
 * y fp32 [nrows, N] for the given rows of x: y[r, n] = the fp32 accumulator above (before
 * the bf16 rounding), from codes x8 [M, Kpad], w8 [N, Kpad] and scales sx, sw.
 */
void sa_oracle_w8a8_gemm_rows(const int8_t *x8, const float *sx, const int8_t *w8,
                              const float *sw, int64_t M, int64_t N, int64_t K,
                              const int64_t *rows, int64_t nrows, float *y)
{
    const int64_t cb = cdiv64(K, 128), kpad = cb * 128;
    (void)M;
    for (int64_t ri = 0; ri < nrows; ++ri) {
        const int64_t m = rows[ri];
        for (int64_t n = 0; n < N; ++n) {
            float acc = 0.0f;
            for (int64_t b = 0; b < cb; ++b) {
                int32_t S = 0;
                for (int64_t k = b * 128; k < b * 128 + 128; ++k)
                    S += (int32_t)x8[m * kpad + k] * (int32_t)w8[n * kpad + k];
                const float s = sx[(m / 128) * cb + b] * sw[(n / 128) * cb + b];
                acc = fmaf((float)S, s, acc);
            }
            y[ri * N + n] = acc;
        }
    }
}

/* ------------------------------------------------------------------------------------
 * SLA linear-attention branch (the "marginal" blocks of Sparse-Linear Attention).
 *
 * Sources: NetEase article on the TurboDiffusion release, attention-acceleration section:
 * SLA combines sparse attention with linear attention, and its figure caption splits the
 * attention weights into three classes computed at different costs; "AIGC weekend
 * special 5.10" section 1.2 Method item (2): SLA is a trainable sparse *linear* attention
 * used on top of SageAttention.  The pages give no formula for the linear part.
 *
 * Reading: the classes come per (128-query block i, 64-key block j) in a uint8 map:
 * 0 = negligible (skipped), 1 = marginal (linear attention), >= 2 = critical (the sparse
 * quantised attention above).  The marginal part is kernelised linear attention with a
 * feature map phi applied to each row's d features:
 *     w_t = phi(q_r) . phi(k_t) over the keys t < N of the row's marginal blocks,
 *     O_lin[r] = sum_t w_t v_t / sum_t w_t          (0 when the row has no marginal key),
 * and the branch's output is O_lin projected by a d x d matrix W (a trained layer in
 * SLA; here any given matrix, the identity when NULL): out[r][c] = sum_e W[c][e] O_lin[r][e].
 * phi = 0: softmax over the features, phi(x)_a = exp(x_a - max x) / sum_b exp(x_b - max x);
 * phi = 1: elu(x) + 1, i.e. x + 1 for x > 0 and exp(x) otherwise.  Both are positive, so
 * sum_t w_t > 0 whenever the row has a marginal key.
 * This is the weighted-average form written out in fp64 per row; it equals the
 * factorised form phi(q)^T (sum_t phi(k_t) v_t^T) / (phi(q) . sum_t phi(k_t)) by
 * associativity, which is how a fast implementation evaluates it.
 * ------------------------------------------------------------------------------------ */

static void phi_row(const uint16_t *x, int d, int phi, double *out)
{
    if (phi == 0) {
        double mx = -INFINITY;
        for (int a = 0; a < d; ++a) {
            const double v = (double)bf16_to_f32(x[a]);
            if (v > mx) mx = v;
        }
        double sum = 0.0;
        for (int a = 0; a < d; ++a) {
            out[a] = exp((double)bf16_to_f32(x[a]) - mx);
            sum += out[a];
        }
        for (int a = 0; a < d; ++a) out[a] /= sum;
    } else {
        for (int a = 0; a < d; ++a) {
            const double v = (double)bf16_to_f32(x[a]);
            out[a] = v > 0.0 ? v + 1.0 : exp(v);
        }
    }
}

/* classes: uint8 [B,H,nq,nk]; proj: fp32 [d][d] (row = output feature) or NULL;
 * rows: (bh, r) pairs; out: fp64 [nrows, d]. */
void sa_oracle_sla_linear_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int H,
                               int N, int d, const uint8_t *classes, int phi, const float *proj,
                               const int64_t *rows, int64_t nrows, double *out)
{
    (void)B; (void)H;
    const int64_t nq = cdiv64(N, QBLK), nk = cdiv64(N, KBLK);
    double *pq = (double *)malloc(sizeof(double) * (size_t)d);
    double *pk = (double *)malloc(sizeof(double) * (size_t)d);
    double *ol = (double *)malloc(sizeof(double) * (size_t)d);
    for (int64_t n = 0; n < nrows; ++n) {
        const int64_t bh = rows[2 * n], r = rows[2 * n + 1];
        const int64_t i = r / QBLK;
        const uint8_t *crow = classes + (bh * nq + i) * nk;
        phi_row(q + (bh * N + r) * d, d, phi, pq);
        double den = 0.0;
        for (int c = 0; c < d; ++c) ol[c] = 0.0;
        for (int64_t t = 0; t < N; ++t) {
            if (crow[t / KBLK] != 1) continue;
            phi_row(k + (bh * N + t) * d, d, phi, pk);
            double w = 0.0;
            for (int a = 0; a < d; ++a) w += pq[a] * pk[a];
            den += w;
            const uint16_t *vt = v + (bh * N + t) * d;
            for (int c = 0; c < d; ++c) ol[c] += w * (double)bf16_to_f32(vt[c]);
        }
        double *o = out + n * d;
        for (int c = 0; c < d; ++c) ol[c] = den > 0.0 ? ol[c] / den : 0.0;
        for (int c = 0; c < d; ++c) {
            if (!proj) {
                o[c] = ol[c];
                continue;
            }
            double acc = 0.0;
            for (int e = 0; e < d; ++e) acc += (double)proj[c * d + e] * ol[e];
            o[c] = acc;
        }
    }
    free(pq);
    free(pk);
    free(ol);
}
