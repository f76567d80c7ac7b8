// sa_attn_pairs.cuh -- the dense attention kernel: two query tiles per CTA.
// Included by sa_attn.cu inside its anonymous namespace (shares its constants, the device
// status word and the helpers above the include).
//
// The attention forward without a keep mask (every 64-key block kept, steps
// of two consecutive blocks; "AIGC weekend special 5.10" section 1.2 Method item (1),
// FlashAttention's tiled online softmax), organised for latency hiding:
//   * A CTA takes a pair of 128-query tiles (A, B) of one head.  Both read the same K/V
//     stream, so each K/V stage serves two tiles.
//   * Warpgroup 0 (warps 0-3) runs the softmax, O rescaling and epilogue of tile A,
//     warpgroup 1 (warps 4-7) those of tile B.  A thread owns one query row and all 128
//     keys of a step, so the two warps on a scheduler work on independent rows: the
//     exponentials of one overlap the tensor-memory loads, maxima and waits of the other,
//     and no row maximum is exchanged between warps.
//   * One S buffer in tensor memory serves both tiles in turn (QK_A(j), QK_B(j),
//     QK_A(j+1), ...), which also staggers the two warpgroups by half a step; each tile
//     has its own O accumulator (N = 144: 128 channels + the row-sum column fed by the
//     constant e4m3 1.0 row of every V^T stage) and its own P tile in shared memory.
//   * warp 8 producer (Q pair, K/V ring), warp 9 QK issuer, warp 10 PV issuer, warp 11
//     idle (completes the third warpgroup).  Registers: 168 per thread at launch, the
//     softmax warpgroups raise theirs to 232 (a whole 128-key row of S in registers) and
//     the third lowers its to 40 (setmaxnreg): 2*232 + 40 <= 3*168.
// Tensor memory: S [0,128), O_A [128,272), O_B [272,416).
// Every mbarrier wait is bounded (sa_ptx.cuh); on expiry the kernel records the device
// timeout status and exits.

namespace pairs {

constexpr int kStages = 4;
constexpr int kThreads = 384;
constexpr int kWarpProducer = 8;
constexpr int kWarpMmaQK = 9;
constexpr int kWarpMmaPV = 10;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;
__host__ __device__ constexpr uint32_t col_o(int t) { return 128u + 144u * uint32_t(t); }

constexpr int kLaunchRegs = (65536 / kThreads) / 8 * 8;  // what __launch_bounds__(kThreads, 1) allows
constexpr int kRegsSoftmax = 232, kRegsCtrl = 40;
static_assert(128 * (2 * kRegsSoftmax + kRegsCtrl) <= kLaunchRegs * kThreads,
              "the register split must fit the registers the block is launched with");

constexpr uint32_t kOffQ = 0;                                    // Q_A, Q_B
constexpr uint32_t kOffK = kOffQ + 2 * kQTileBytes;
constexpr uint32_t kOffV = kOffK + kStages * kKTileBytes;
constexpr uint32_t kOffP = kOffV + kStages * 2 * kVHalfBytes;    // P_A, P_B
constexpr uint32_t kOffBar = kOffP + 2 * kPTileBytes;
constexpr int kBarQFull = 0, kBarQEmpty = 1, kBarKvFull = 2, kBarKvEmpty = kBarKvFull + kStages,
              kBarSFull = kBarKvEmpty + kStages,  // [2]: per tile
              kBarSEmpty = kBarSFull + 2, kBarPFull = kBarSEmpty + 1, kBarPvDone = kBarPFull + 2,
              kBarOFull = kBarPvDone + 2, kBarOEmpty = kBarOFull + 2, kNumBars = kBarOEmpty + 2;
constexpr uint32_t kOffMisc = kOffBar + 8 * kNumBars;            // tmem base, abort flag
constexpr uint32_t kSmemBytes = kOffMisc + 16;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;               // 1024-B alignment slack

static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffP % 1024 == 0, "tile alignment");
static_assert(kSmemAlloc <= 227 * 1024, "shared memory per CTA");

template <uint32_t NR>
__device__ __forceinline__ void setmaxnreg_inc()
{
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(NR));
}

template <uint32_t NR>
__device__ __forceinline__ void setmaxnreg_dec()
{
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(NR));
}

// 32 consecutive 32-bit TMEM columns of this thread's lane, without waiting: the
// registers are valid only after tmem_wait_ld on the same array.
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// Orders later uses of r after a tcgen05.wait::ld (the array passes through the statement).
__device__ __forceinline__ void tmem_regs_ready(uint32_t (&r)[32])
{
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                   "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                   "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                   "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

// Four 32-column loads in flight, one wait: 128 columns [taddr, taddr + 128).
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r0)[32], uint32_t (&r1)[32],
                                           uint32_t (&r2)[32], uint32_t (&r3)[32])
{
    tmem_ld32_nowait(taddr, r0);
    tmem_ld32_nowait(taddr + 32, r1);
    tmem_ld32_nowait(taddr + 64, r2);
    tmem_ld32_nowait(taddr + 96, r3);
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    tmem_regs_ready(r0);
    tmem_regs_ready(r1);
    tmem_regs_ready(r2);
    tmem_regs_ready(r3);
}

// Max of the 64 int32 values in two arrays of 32.
__device__ __forceinline__ int max64x2(const uint32_t (&a)[32], const uint32_t (&b)[32])
{
    int acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = max(int(a[k]), int(b[k]));
#pragma unroll
    for (int i = 8; i < 32; i += 8)
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = max(acc[k], max(int(a[i + k]), int(b[i + k])));
    return max(max(max(acc[0], acc[1]), max(acc[2], acc[3])), max(max(acc[4], acc[5]), max(acc[6], acc[7])));
}

// S of one row (128 keys: s0..s3, keys 32a..32a+31 in sa) -> 32 words of e4m3
// P = 448 * 2^(S*k + nbias), k = k0 for keys 0-63 and k1 for keys 64-127; with MASK, the
// bytes of keys at or past nv0 (first block) or nv1 (second block) are zero.  The words are
// computed as a software pipeline -- exponent arguments of word w+1, ex2 of word w, packing
// of word w-1 -- so that the four ex2 of a word are spread among other instructions: a warp
// that has the multi-function unit to itself then keeps it busier (10.0 instead of 13.4
// cycles per 32 keys; the same 8.4 with two warps per scheduler).
template <bool MASK>
__device__ __forceinline__ void p_row_impl(const uint32_t (&s0)[32], const uint32_t (&s1)[32],
                                           const uint32_t (&s2)[32], const uint32_t (&s3)[32],
                                           float k0, float k1, float nbias, int nv0, int nv1,
                                           uint32_t (&pw)[32])
{
#define SA_SV(key) ((key) < 32 ? s0[(key)] : (key) < 64 ? s1[(key) - 32] : (key) < 96 ? s2[(key) - 64] : s3[(key) - 96])
    float y[2][4], e[2][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) y[0][i] = fma_ord(cvt_s32_f32_ord(SA_SV(i)), k0, nbias);
#pragma unroll
    for (int w = 0; w < 33; ++w) {
        const int cur = w & 1, nxt = cur ^ 1;
        if (w + 1 < 32) {
            const float k = (w + 1) < 16 ? k0 : k1;
#pragma unroll
            for (int i = 0; i < 4; ++i) y[nxt][i] = fma_ord(cvt_s32_f32_ord(SA_SV(4 * (w + 1) + i)), k, nbias);
        }
        if (w < 32) {
#pragma unroll
            for (int i = 0; i < 4; ++i) e[cur][i] = ex2_ord(y[cur][i]);
        }
        if (w >= 1) {
            uint32_t x = pack_e4m3x2_ord(e[nxt][0], e[nxt][1]) | (pack_e4m3x2_ord(e[nxt][2], e[nxt][3]) << 16);
            if (MASK) {
                const int kb = ((w - 1) < 16 ? nv0 : nv1) - 4 * ((w - 1) & 15);  // bytes to keep
                x = kb >= 4 ? x : (kb <= 0 ? 0u : (x & ((1u << (8 * kb)) - 1u)));
            }
            pw[w - 1] = x;
        }
    }
#undef SA_SV
}

// The masked form only where some row of the warp has a partial block (ragged tail, causal).
__device__ __forceinline__ void p_row(const uint32_t (&s0)[32], const uint32_t (&s1)[32],
                                      const uint32_t (&s2)[32], const uint32_t (&s3)[32],
                                      float k0, float k1, float nbias, int nv0, int nv1,
                                      uint32_t (&pw)[32])
{
    if (__any_sync(0xffffffffu, nv0 < 64 || nv1 < 64))
        p_row_impl<true>(s0, s1, s2, s3, k0, k1, nbias, nv0, nv1, pw);
    else
        p_row_impl<false>(s0, s1, s2, s3, k0, k1, nbias, nv0, nv1, pw);
}

}  // namespace pairs

// VARLEN: head bh has seq_tokens(seq, bh, N) tokens and its output rows start at
// seq_row0(seq, bh, N); N, Npad, nq and nk are those of the longest head (the strides of the
// quantised buffers and scales), and the pairs past a head's own tiles are skipped by every
// role alike.
template <bool VARLEN>
__global__ void __launch_bounds__(pairs::kThreads, 1)
    attn_pairs_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ q_scale,
                      const float *__restrict__ k_scale, const float *__restrict__ v_scale,
                      __nv_bfloat16 *__restrict__ out, int BH, int N, int Npad, int nq, int nk,
                      float sm_scale, int causal, SeqTable seq)
{
    using pairs::kStages;
    using pairs::kThreads;
    using pairs::kWarpProducer;
    using pairs::kWarpMmaQK;
    using pairs::kWarpMmaPV;
    using pairs::kTmemCols;
    using pairs::kColS;
    using pairs::col_o;
    using pairs::kRegsSoftmax;
    using pairs::kRegsCtrl;
    using pairs::kOffQ;
    using pairs::kOffK;
    using pairs::kOffV;
    using pairs::kOffP;
    using pairs::kOffBar;
    using pairs::kBarQFull;
    using pairs::kBarQEmpty;
    using pairs::kBarKvFull;
    using pairs::kBarKvEmpty;
    using pairs::kBarSFull;
    using pairs::kBarSEmpty;
    using pairs::kBarPFull;
    using pairs::kBarPvDone;
    using pairs::kBarOFull;
    using pairs::kBarOEmpty;
    using pairs::kOffMisc;
    using pairs::setmaxnreg_inc;
    using pairs::setmaxnreg_dec;
    using pairs::tmem_ld128;
    using pairs::max64x2;
    using pairs::p_row;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile uint32_t *tmem_base_slot = reinterpret_cast<volatile uint32_t *>(smem + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
    auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * uint32_t(i); };

    // ---- set-up: barriers, constant V rows, tensor memory
    if (threadIdx.x == 0) {
        mbar_init(bar(kBarQFull), 1);
        mbar_init(bar(kBarQEmpty), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar(kBarKvFull + s), 1);
            mbar_init(bar(kBarKvEmpty + s), 1);
        }
        mbar_init(bar(kBarSEmpty), 4);
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(kBarSFull + t), 1);
            mbar_init(bar(kBarPFull + t), 4);
            mbar_init(bar(kBarPvDone + t), 1);
            mbar_init(bar(kBarOFull + t), 1);
            mbar_init(bar(kBarOEmpty + t), 4);
        }
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

    const int npairs_h = (nq + 1) / 2, npairs = BH * npairs_h;
    // the tokens, query tiles and key steps of head bh (every block kept: blocks 2j and
    // 2j+1 form step j; with an odd block count the last step has one block)
    struct Geo {
        int n, nq, nk, nsteps;
        bool odd;
    };
    auto geo = [&](int bh) -> Geo {
        if (!VARLEN) return Geo{N, nq, nk, (nk + 1) / 2, (nk & 1) != 0};
        const int n = seq_tokens(seq, bh, N), q = (n + 127) / 128, k = (n + 63) / 64;
        return Geo{n, q, k, (k + 1) / 2, (k & 1) != 0};
    };
    // causal: the pair (qa, qa + 1) needs the steps up to tile qa + 1's diagonal, qa + 2 of
    // them (qa + 1 for a lone last tile); tile qa's last step is then fully masked
    auto pair_steps = [&](int qa, const Geo &g) -> int {
        return causal ? min(g.nsteps, qa + (qa + 1 < g.nq ? 2 : 1)) : g.nsteps;
    };
    // The work items of this CTA, the same sequence for every role: item r*G + b of round r
    // (G CTAs, b = this CTA).  Without causality every pair costs the same, and pairs go in
    // head-major order, so the CTAs in flight share a head's K/V in L2.  With it a pair
    // costs qa + 2 steps: pairs go longest first (heads fastest within one pair position)
    // and every other round is dealt in reverse CTA order, which evens out the CTAs' totals
    // (the largest CTA total is 1.49x the mean in head-major order at 40 x 75600, 1.00x so).
    // An index past the last pair ends the sequence: every later round's is larger.
    auto item = [&](int r) -> int {
        const int b = (causal && (r & 1)) ? int(gridDim.x) - 1 - int(blockIdx.x) : int(blockIdx.x);
        return r * int(gridDim.x) + b;
    };
    auto pair_head = [&](int i) -> int { return causal ? i % BH : i / npairs_h; };
    auto pair_qa = [&](int i) -> int { return 2 * (causal ? npairs_h - 1 - i / BH : i % npairs_h); };

    if (warp >= kWarpProducer) {
        setmaxnreg_dec<kRegsCtrl>();
        if (warp == kWarpProducer && lane == 0) {
            // ------------------------------------------------------------ producer
            bool ok = true;
            uint32_t g = 0, pl = 0;
            // K/V tiles are read by every CTA working on the head: keep them in L2 in
            // preference to the Q tiles, which one CTA reads once (DRAM traffic per launch at
            // 40 x 75600: 2.43 GB with the hints, 2.49 GB without; 1.94 GB algorithmic)
            const uint64_t pol_kv = l2_policy_evict_last(), pol_q = l2_policy_evict_first();
            for (int r = 0, p = item(0); p < npairs; p = item(++r)) {
                const int bh = pair_head(p), qa = pair_qa(p);
                const Geo ge = geo(bh);
                if (VARLEN && qa >= ge.nq) continue;
                const bool hasb = qa + 1 < ge.nq;
                if (pl >= 1 && ok) ok = mbar_wait(bar(kBarQEmpty), (pl - 1) & 1, abort_flag);
                if (ok) {
                    mbar_arrive_expect_tx(bar(kBarQFull), (hasb ? 2u : 1u) * kQTileBytes);
                    tma_load_2d_hint(sbase + kOffQ, &tm_q, bar(kBarQFull), 0, bh * Npad + qa * 128, pol_q);
                    if (hasb)
                        tma_load_2d_hint(sbase + kOffQ + kQTileBytes, &tm_q, bar(kBarQFull), 0,
                                         bh * Npad + qa * 128 + 128, pol_q);
                }
                const int ns = pair_steps(qa, ge);
                for (int j = 0; j < ns && ok; ++j, ++g) {
                    const uint32_t st = g % kStages;
                    const bool two = !(ge.odd && j == ge.nsteps - 1);
                    if (g >= kStages) ok = mbar_wait(bar(kBarKvEmpty + st), ((g / kStages) - 1) & 1, abort_flag);
                    if (!ok) break;
                    const uint32_t kb = sbase + kOffK + st * kKTileBytes;
                    const uint32_t vb = sbase + kOffV + st * 2 * kVHalfBytes;
                    mbar_arrive_expect_tx(bar(kBarKvFull + st), (two ? 2u : 1u) * (kKHalfBytes + kVHalfData));
                    tma_load_2d_hint(kb, &tm_k, bar(kBarKvFull + st), 0, bh * Npad + 128 * j, pol_kv);
                    tma_load_2d_hint(vb, &tm_v, bar(kBarKvFull + st), 128 * j, bh * 128, pol_kv);
                    if (two) {
                        tma_load_2d_hint(kb + kKHalfBytes, &tm_k, bar(kBarKvFull + st), 0, bh * Npad + 128 * j + 64,
                                         pol_kv);
                        tma_load_2d_hint(vb + kVHalfBytes, &tm_v, bar(kBarKvFull + st), 128 * j + 64, bh * 128,
                                         pol_kv);
                    }
                }
                ++pl;
            }
            if (!ok) { *abort_flag = 1; record_timeout(); }
        } else if (warp == kWarpMmaQK && lane == 0) {
            // ------------------------------------------------------------ QK issuer
            // S_A(j), S_B(j), S_A(j+1), ... through the one S buffer
            bool ok = true;
            uint32_t g = 0, u = 0, pl = 0;
            for (int r = 0, p = item(0); p < npairs && ok; p = item(++r)) {
                const int qa = pair_qa(p);
                const Geo ge = geo(pair_head(p));
                if (VARLEN && qa >= ge.nq) continue;
                const int ntile = qa + 1 < ge.nq ? 2 : 1;
                ok = mbar_wait(bar(kBarQFull), pl & 1, abort_flag);
                tc_fence_after();
                const int ns = pair_steps(qa, ge);
                for (int j = 0; j < ns && ok; ++j, ++g) {
                    const uint32_t st = g % kStages;
                    ok = mbar_wait(bar(kBarKvFull + st), (g / kStages) & 1, abort_flag);
                    const uint32_t kb = sbase + kOffK + st * kKTileBytes;
                    for (int t = 0; t < ntile && ok; ++t, ++u) {
                        if (u >= 1) ok = mbar_wait(bar(kBarSEmpty), (u - 1) & 1, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t qaddr = sbase + kOffQ + uint32_t(t) * kQTileBytes;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_i8(tmem + kColS, sdesc(qaddr + 32 * kk, 1024, SWZ_128B),
                                   sdesc(kb + 32 * kk, 1024, SWZ_128B), kIdescQK, kk > 0);
                        tc_commit(bar(kBarSFull + t));
                    }
                }
                if (ok) tc_commit(bar(kBarQEmpty));
                ++pl;
            }
            if (!ok) { *abort_flag = 1; record_timeout(); }
        } else if (warp == kWarpMmaPV && lane == 0) {
            // ------------------------------------------------------------ PV issuer
            bool ok = true;
            uint32_t g = 0, c[2] = {0, 0}, o[2] = {0, 0};
            for (int r = 0, p = item(0); p < npairs && ok; p = item(++r)) {
                const int qa = pair_qa(p);
                const Geo ge = geo(pair_head(p));
                if (VARLEN && qa >= ge.nq) continue;
                const int ntile = qa + 1 < ge.nq ? 2 : 1;
                const int ns = pair_steps(qa, ge);
                for (int j = 0; j < ns && ok; ++j, ++g) {
                    const uint32_t st = g % kStages;
                    const int nkk = (ge.odd && j == ge.nsteps - 1) ? 2 : 4;  // K = 64 or 128 keys
                    ok = mbar_wait(bar(kBarKvFull + st), (g / kStages) & 1, abort_flag);
                    const uint32_t vb = sbase + kOffV + st * 2 * kVHalfBytes;
                    for (int t = 0; t < ntile && ok; ++t) {
                        ok = mbar_wait(bar(kBarPFull + t), c[t] & 1, abort_flag);
                        if (ok && j == 0 && o[t] >= 1) ok = mbar_wait(bar(kBarOEmpty + t), (o[t] - 1) & 1, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t pa = sbase + kOffP + uint32_t(t) * kPTileBytes;
                        for (int kk = 0; kk < nkk; ++kk)
                            mma_f8(tmem + col_o(t), sdesc(pa + 32 * kk, 1024, SWZ_128B),
                                   sdesc(vb + (kk >> 1) * kVHalfBytes + 32 * (kk & 1), 512, SWZ_64B),
                                   kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
                        tc_commit(bar(kBarPvDone + t));
                        ++c[t];
                    }
                    // QK of this step completed before its P existed, so the stage is free
                    // once the PVs of this step complete
                    if (ok) tc_commit(bar(kBarKvEmpty + st));
                }
                for (int t = 0; t < ntile && ok; ++t) {
                    tc_commit(bar(kBarOFull + t));
                    ++o[t];
                }
            }
            if (!ok) { *abort_flag = 1; record_timeout(); }
        }
    } else {
        // ---------------------------------------------------------------- softmax, tile t
        setmaxnreg_inc<kRegsSoftmax>();
        const int t = warp >> 2;                 // 0: tile A, 1: tile B
        const int wq = warp & 3;                 // TMEM lane quarter
        const int row = wq * 32 + lane;          // query row within the tile
        const uint32_t lane_addr = uint32_t(wq * 32) << 16;
        const uint32_t sa = tmem + lane_addr + kColS;
        const uint32_t oa = tmem + lane_addr + col_o(t);
        uint8_t *prow = smem + kOffP + uint32_t(t) * kPTileBytes + row * 128;
        bool ok = true;
        uint32_t c = 0, o = 0;  // steps and tiles this warpgroup has processed
        for (int r = 0, p = item(0); p < npairs; p = item(++r)) {
            const int bh = pair_head(p), qt = pair_qa(p) + t;
            const Geo ge = geo(bh);
            if (qt >= ge.nq) continue;  // tile B of the last pair of an odd tile count (or past the head)
            const int qrow = qt * 128 + row;
            const float sq = q_scale[int64_t(bh) * nq + qt];
            const float *ksrow = k_scale + int64_t(bh) * nk;
            float m = -INFINITY;
            const int ns = pair_steps(qt - t, ge);
            for (int j = 0; j < ns; ++j, ++c) {
                const bool two = !(ge.odd && j == ge.nsteps - 1);
                const float ks0 = ksrow[2 * j], ks1 = two ? ksrow[2 * j + 1] : 0.0f;
                int nv0 = min(64, ge.n - 128 * j), nv1 = two ? min(64, ge.n - 128 * j - 64) : 0;
                if (causal) {
                    // this row keeps the keys up to itself
                    nv0 = max(0, min(nv0, qrow - 128 * j + 1));
                    nv1 = max(0, min(nv1, qrow - 128 * j - 63));
                }
                if (ok) ok = mbar_wait(bar(kBarSFull + t), c & 1, abort_flag);
                ok = __all_sync(0xffffffffu, ok);

                // S of this step, all 128 keys of the row, read once
                uint32_t s0[32], s1[32], s2[32], s3[32];
                if (ok) {
                    tc_fence_after();
                    tmem_ld128(sa, s0, s1, s2, s3);
                }

                // keys past the end of the sequence or after the row (causal) drop out of
                // the max (their P bytes are cleared below); a block with no key left
                // contributes no maximum at all, whatever its scale
                if (nv0 < 64) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        if (i >= nv0) s0[i] = uint32_t(INT_MIN);
                        if (i + 32 >= nv0) s1[i] = uint32_t(INT_MIN);
                    }
                }
                if (two && nv1 < 64) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        if (i >= nv1) s2[i] = uint32_t(INT_MIN);
                        if (i + 32 >= nv1) s3[i] = uint32_t(INT_MIN);
                    }
                }
                // row max on int32 S per block (each scale is non-negative, so max commutes)
                const float c0 = (sq * ks0) * sm_scale, c1 = (sq * ks1) * sm_scale;
                float pmax = nv0 > 0 ? i2f(uint32_t(max64x2(s0, s1))) * c0 : -INFINITY;
                if (nv1 > 0) pmax = fmaxf(pmax, i2f(uint32_t(max64x2(s2, s3))) * c1);
                const float mnew = fmaxf(m, pmax);
                // the S buffer goes to the other tile's QK only now, after the maximum: this
                // delays the other warpgroup by about that long, so that its exponentials
                // tend to run while this one loads, stores and waits (measured at 720p:
                // 97.2 ms, against 103.4 ms for a release right after the load and 114 ms
                // for one after the first exponentials)
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarSEmpty));

                // P = e4m3(448 * 2^(S*c*log2e - mnew*log2e)), 8 words per 32 keys
                const float nbias = kLog2_448 - mnew * kLog2e;
                uint32_t pw[32];
                p_row(s0, s1, s2, s3, c0 * kLog2e, c1 * kLog2e, nbias, nv0, two ? nv1 : 0, pw);

                // the P tile and O are free once the PV of the previous step completed
                if (c >= 1 && ok) ok = mbar_wait(bar(kBarPvDone + t), (c - 1) & 1, abort_flag);
                ok = __all_sync(0xffffffffu, ok);
                // 128B-swizzled P tile: 16-byte chunk k of row r at position k ^ (r & 7)
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    *reinterpret_cast<uint4 *>(prow + ((k ^ (row & 7)) << 4)) =
                        make_uint4(pw[4 * k], pw[4 * k + 1], pw[4 * k + 2], pw[4 * k + 3]);

                // rescale O (and its row-sum column) when the running max grew
                if (j > 0) {
                    const bool need = mnew > m;
                    if (__any_sync(0xffffffffu, need) && ok) {
                        tc_fence_after();
                        const float alpha = need ? ex2_approx((m - mnew) * kLog2e) : 1.0f;
#pragma unroll 1
                        for (int h = 0; h < 2; ++h) {
                            uint32_t r0[32], r1[32];
                            tmem_ld64_wait(oa + 64 * h, r0, r1);
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
                            tmem_st32(oa + 64 * h, r0);
                            tmem_st32(oa + 64 * h + 32, r1);
                        }
                        uint32_t r8[8];
                        tmem_ld8_wait(oa + 128, r8);
#pragma unroll
                        for (int i = 0; i < 8; ++i) r8[i] = __float_as_uint(__uint_as_float(r8[i]) * alpha);
                        tmem_st8(oa + 128, r8);
                        tmem_st_wait();
                    }
                }
                m = mnew;
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarPFull + t));
            }
            // ---- epilogue: O = acc * scale_v / l, bf16, 32 channels at a time
            if (ok) ok = mbar_wait(bar(kBarOFull + t), o & 1, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                tc_fence_after();
                uint32_t lbits;
                tmem_ld1_wait(oa + 128, lbits);
                const float l = __uint_as_float(lbits);
                const float inv_l = l > 0.0f ? __frcp_rn(l) : 0.0f;
                const float *svp = v_scale + int64_t(bh) * kD;
                __nv_bfloat16 *orow = out + ((VARLEN ? seq_row0(seq, bh, N) : int64_t(bh) * N) + qrow) * kD;
#pragma unroll 1
                for (int h = 0; h < 4; ++h) {
                    uint32_t ov[32];
                    tmem_ld32_wait(oa + 32 * h, ov);
                    if (qrow < ge.n) {
#pragma unroll
                        for (int cidx = 0; cidx < 4; ++cidx) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int i = 8 * cidx + 2 * e;
                                const float y0 = (__uint_as_float(ov[i]) * svp[32 * h + i]) * inv_l;
                                const float y1 = (__uint_as_float(ov[i + 1]) * svp[32 * h + i + 1]) * inv_l;
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
            if (lane == 0) mbar_arrive(bar(kBarOEmpty + t));
            ++o;
        }
        if (lane == 0 && !ok) { *abort_flag = 1; record_timeout(); }
    }

    // ---- teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMmaQK) tmem_dealloc(tmem, kTmemCols);
}
