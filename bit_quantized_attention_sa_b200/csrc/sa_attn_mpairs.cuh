// sa_attn_mpairs.cuh -- the attention kernel for calls with a keep mask: two query tiles
// per CTA, each with its own stream of kept key blocks.
// Included by sa_attn.cu inside its anonymous namespace, after sa_attn_pairs.cuh: it uses
// the pair kernel's shared-memory layout, register split, tensor-memory columns and P row.
//
// The attention forward with a keep mask (the kept 64-key blocks of a tile,
// taken in ascending order two per step; "AIGC weekend special 5.10" section 1.2 Method
// items (1)-(2), FlashAttention's tiled online softmax), organised as the pair kernel:
//   * A CTA takes a pair of 128-query tiles (A, B) of one head; softmax warpgroup 0 runs
//     tile A, warpgroup 1 tile B, a thread owning one row and all 128 keys of a step.
//   * The tiles keep different blocks, so each has its own steps.  The steps of the two
//     tiles take turns in one K/V ring, A0, B0, A1, B1, ..., then the rest of the longer
//     list; each stage holds one tile's step (its two blocks, or one at the end of an odd
//     count) and is freed by that step's PV.  The one S buffer serves the steps in the
//     same order.
//   * Warp 11 scans the mask rows of each pair once, up to two pairs ahead, into one of two
//     entries in shared memory: the two tiles' step counts and their kept blocks as
//     bitmasks.  Every role reads the counts from the entry and derives the same slot order
//     from them; the producer takes the blocks from the bitmasks and records each stage's
//     block indices, which the softmax reads for the K scales and the valid keys.
//   * A tile with no kept block writes zero rows (or the addend) and takes no part in the
//     barrier sequence; a pair with none at all is skipped by every role but the softmax
//     warpgroups, which write its rows.
// Every mbarrier wait is bounded, as in the other attention kernels.

namespace mpairs {

constexpr int kMaxBlocks = kMaskedAttnMaxKeyBlocks;  // key blocks per mask row (N <= 1,048,576)
constexpr int kWords = kMaxBlocks / 32;               // bitmask words per tile
constexpr uint32_t kOffInfo = pairs::kOffMisc + 16;  // int2 [kStages]: the blocks of each stage
constexpr uint32_t kOffEntBar = kOffInfo + 8 * pairs::kStages;  // entry full [2], empty [2]
constexpr uint32_t kOffEnt = (kOffEntBar + 32 + 15) / 16 * 16;
constexpr uint32_t kEntBytes = 16 + 2 * kWords * 4;   // nA, nB; kept bits of tiles A and B
constexpr uint32_t kSmemAlloc = kOffEnt + 2 * kEntBytes + 1024;
constexpr int kEntReaders = 11;                       // producer, QK, PV and the 8 softmax warps
constexpr int kWinBlocks = 256;                       // mask bytes read per window by the scanner
static_assert(kSmemAlloc <= 227 * 1024, "shared memory per CTA");

// Slot k of a pair whose tiles have nA and nB steps: its tile t and that tile's step j.
__device__ __forceinline__ void slot_of(int k, int nA, int nB, int &t, int &j)
{
    const int m = min(nA, nB);
    if (k < 2 * m) {
        t = k & 1;
        j = k >> 1;
    } else {
        t = nA > nB ? 0 : 1;
        j = m + (k - 2 * m);
    }
}

// The scanner warp's pass over one mask row: the kept bits into words[0 .. ceil(nk/32)),
// returning the kept count.  Each lane loads its 8 bytes of a 256-block window before any is
// used, so a window costs one memory latency.
__device__ __forceinline__ int scan_row(const uint8_t *row, int nk, int lane, uint32_t *words)
{
    int cnt = 0;
    for (int base = 0; base < nk; base += kWinBlocks) {
        uint32_t v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int j = base + 32 * i + lane;
            v[i] = j < nk ? row[j] : 0u;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t w = __ballot_sync(0xffffffffu, v[i] != 0);
            cnt += __popc(w);
            if (lane == i && base + 32 * i < nk) words[base / 32 + i] = w;
        }
    }
    return cnt;
}

// The kept blocks of one tile in ascending order, from its bitmask in shared memory.
struct KeptCursor {
    const uint32_t *words;
    int nw, w;
    uint32_t bits;
    __device__ __forceinline__ void init(const uint32_t *ws, int n)
    {
        words = ws;
        nw = n;
        w = -1;
        bits = 0;
    }
    __device__ __forceinline__ int next()  // -1 once the row is exhausted
    {
        while (bits == 0) {
            if (++w >= nw) return -1;
            bits = words[w];
        }
        const int j = 32 * w + __ffs(int(bits)) - 1;
        bits &= bits - 1;
        return j;
    }
};

}  // namespace mpairs

__global__ void __launch_bounds__(pairs::kThreads, 1)
    attn_mpairs_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ q_scale,
                       const float *__restrict__ k_scale, const float *__restrict__ v_scale,
                       const uint8_t *__restrict__ mask, __nv_bfloat16 *__restrict__ out, int BH, int N,
                       int Npad, int nq, int nk, float sm_scale, int causal, const float *__restrict__ addend)
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
    using mpairs::kOffInfo;
    using mpairs::kOffEnt;
    using mpairs::kEntBytes;
    using mpairs::kWords;
    using mpairs::slot_of;
    using mpairs::KeptCursor;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int2 *info = reinterpret_cast<int2 *>(smem + kOffInfo);
    volatile uint32_t *tmem_base_slot = reinterpret_cast<volatile uint32_t *>(smem + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
    auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * uint32_t(i); };
    // entry barriers: full[e] at ebar(e), empty[e] at ebar(2 + e)
    auto ebar = [&](int i) -> uint32_t { return sbase + mpairs::kOffEntBar + 8u * uint32_t(i); };
    // entry e: int nA, nB at +0, +4; kept bits of tile t at +16 + 4 * kWords * t
    auto ent_counts = [&](int e) -> volatile int * { return reinterpret_cast<volatile int *>(smem + kOffEnt + e * kEntBytes); };
    auto ent_words = [&](int e, int t) -> uint32_t * {
        return reinterpret_cast<uint32_t *>(smem + kOffEnt + e * kEntBytes + 16 + 4 * kWords * t);
    };

    // ---- set-up: barriers, constant V rows, tensor memory (as the pair kernel)
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
        for (int e = 0; e < 2; ++e) {
            mbar_init(ebar(e), 1);
            mbar_init(ebar(2 + e), mpairs::kEntReaders);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    // rows 128..143 of every V half tile: row 128 all e4m3 1.0 (0x38), the rest zero
    for (int i = threadIdx.x; i < kStages * 2 * 16 * 16; i += kThreads) {
        const int half = i / (16 * 16), w = i % (16 * 16);
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

    // work items and their order: as the pair kernel (head-major; with causality longest
    // first and every other round dealt in reverse CTA order)
    const int npairs_h = (nq + 1) / 2, npairs = BH * npairs_h;
    auto item = [&](int r) -> int {
        const int b = (causal && (r & 1)) ? int(gridDim.x) - 1 - int(blockIdx.x) : int(blockIdx.x);
        return r * int(gridDim.x) + b;
    };
    auto pair_head = [&](int i) -> int { return causal ? i % BH : i / npairs_h; };
    auto pair_qa = [&](int i) -> int { return 2 * (causal ? npairs_h - 1 - i / BH : i % npairs_h); };
    auto mrow = [&](int bh, int qt) -> const uint8_t * { return mask + (int64_t(bh) * nq + qt) * nk; };
    const int nw = (nk + 31) / 32;  // bitmask words of a row
    // the entry of the pi-th item: wait until the scanner filled it, read the counts, and
    // release it (readers other than the producer release at once)
    auto read_entry = [&](uint32_t pi, bool release, bool &ok, int &nA, int &nB) {
        const int e = int(pi & 1);
        if (ok) ok = mbar_wait(ebar(e), (pi >> 1) & 1, abort_flag);
        nA = ok ? ent_counts(e)[0] : 0;
        nB = ok ? ent_counts(e)[1] : 0;
        if (release) mbar_arrive(ebar(2 + e));
    };

    if (warp >= kWarpProducer) {
        setmaxnreg_dec<kRegsCtrl>();
        if (warp == kWarpProducer + 3) {
            // ------------------------------------------------------------ scanner (warp 11)
            bool ok = true;
            uint32_t pi = 0;
            for (int r = 0, p = item(0); p < npairs; p = item(++r), ++pi) {
                const int bh = pair_head(p), qa = pair_qa(p), e = int(pi & 1);
                if (pi >= 2 && ok) ok = mbar_wait(ebar(2 + e), ((pi >> 1) - 1) & 1, abort_flag);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                const int kA = mpairs::scan_row(mrow(bh, qa), nk, lane, ent_words(e, 0));
                const int kB = qa + 1 < nq ? mpairs::scan_row(mrow(bh, qa + 1), nk, lane, ent_words(e, 1)) : 0;
                if (lane == 0) {
                    ent_counts(e)[0] = (kA + 1) / 2;
                    ent_counts(e)[1] = (kB + 1) / 2;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(ebar(e));
            }
            if (lane == 0 && !ok) { *abort_flag = 1; record_timeout(); }
        } else if (warp == kWarpProducer && lane == 0) {
            // ------------------------------------------------------------ producer
            bool ok = true;
            uint32_t g = 0, pl = 0, pi = 0;
            const uint64_t pol_kv = l2_policy_evict_last(), pol_q = l2_policy_evict_first();
            for (int r = 0, p = item(0); p < npairs; p = item(++r), ++pi) {
                const int bh = pair_head(p), qa = pair_qa(p), e = int(pi & 1);
                int nA, nB;
                read_entry(pi, false, ok, nA, nB);
                if (nA + nB > 0) {
                    if (pl >= 1 && ok) ok = mbar_wait(bar(kBarQEmpty), (pl - 1) & 1, abort_flag);
                    if (ok) {
                        mbar_arrive_expect_tx(bar(kBarQFull), uint32_t((nA > 0) + (nB > 0)) * kQTileBytes);
                        if (nA > 0)
                            tma_load_2d_hint(sbase + kOffQ, &tm_q, bar(kBarQFull), 0, bh * Npad + qa * 128, pol_q);
                        if (nB > 0)
                            tma_load_2d_hint(sbase + kOffQ + kQTileBytes, &tm_q, bar(kBarQFull), 0,
                                             bh * Npad + qa * 128 + 128, pol_q);
                    }
                    KeptCursor ca, cb;
                    ca.init(ent_words(e, 0), nw);
                    cb.init(ent_words(e, 1), nB > 0 ? nw : 0);
                    for (int k = 0; k < nA + nB; ++k, ++g) {
                        int t, j;
                        slot_of(k, nA, nB, t, j);
                        const int b0 = t ? cb.next() : ca.next();
                        const int b1 = t ? cb.next() : ca.next();
                        const uint32_t st = g % kStages;
                        if (g >= kStages && ok)
                            ok = mbar_wait(bar(kBarKvEmpty + st), ((g / kStages) - 1) & 1, abort_flag);
                        if (!ok) continue;
                        info[st] = make_int2(b0, b1);
                        const uint32_t kb = sbase + kOffK + st * kKTileBytes;
                        const uint32_t vb = sbase + kOffV + st * 2 * kVHalfBytes;
                        mbar_arrive_expect_tx(bar(kBarKvFull + st), (b1 >= 0 ? 2u : 1u) * (kKHalfBytes + kVHalfData));
                        tma_load_2d_hint(kb, &tm_k, bar(kBarKvFull + st), 0, bh * Npad + 64 * b0, pol_kv);
                        tma_load_2d_hint(vb, &tm_v, bar(kBarKvFull + st), 64 * b0, bh * 128, pol_kv);
                        if (b1 >= 0) {
                            tma_load_2d_hint(kb + kKHalfBytes, &tm_k, bar(kBarKvFull + st), 0, bh * Npad + 64 * b1,
                                             pol_kv);
                            tma_load_2d_hint(vb + kVHalfBytes, &tm_v, bar(kBarKvFull + st), 64 * b1, bh * 128,
                                             pol_kv);
                        }
                    }
                    ++pl;
                }
                mbar_arrive(ebar(2 + e));  // the entry's bitmasks are no longer needed
            }
            if (!ok) { *abort_flag = 1; record_timeout(); }
        } else if (warp == kWarpMmaQK && lane == 0) {
            // ------------------------------------------------------------ QK issuer
            bool ok = true;
            uint32_t g = 0, u = 0, pl = 0, pi = 0;
            for (int r = 0, p = item(0); p < npairs; p = item(++r), ++pi) {
                int nA, nB;
                read_entry(pi, true, ok, nA, nB);
                if (nA + nB == 0) continue;
                if (ok) ok = mbar_wait(bar(kBarQFull), pl & 1, abort_flag);
                tc_fence_after();
                for (int k = 0; k < nA + nB && ok; ++k) {
                    int t, j;
                    slot_of(k, nA, nB, t, j);
                    const uint32_t gg = g + uint32_t(k), st = gg % kStages;
                    ok = mbar_wait(bar(kBarKvFull + st), (gg / kStages) & 1, abort_flag);
                    if (ok && u >= 1) ok = mbar_wait(bar(kBarSEmpty), (u - 1) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t qaddr = sbase + kOffQ + uint32_t(t) * kQTileBytes;
                    const uint32_t kb = sbase + kOffK + st * kKTileBytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_i8(tmem + kColS, sdesc(qaddr + 32 * kk, 1024, SWZ_128B),
                               sdesc(kb + 32 * kk, 1024, SWZ_128B), kIdescQK, kk > 0);
                    tc_commit(bar(kBarSFull + t));
                    ++u;
                }
                if (ok) tc_commit(bar(kBarQEmpty));
                g += uint32_t(nA + nB);
                ++pl;
            }
            if (!ok) { *abort_flag = 1; record_timeout(); }
        } else if (warp == kWarpMmaPV && lane == 0) {
            // ------------------------------------------------------------ PV issuer
            bool ok = true;
            uint32_t g = 0, c[2] = {0, 0}, o[2] = {0, 0}, pi = 0;
            for (int r = 0, p = item(0); p < npairs; p = item(++r), ++pi) {
                int nA, nB;
                read_entry(pi, true, ok, nA, nB);
                if (nA + nB == 0) continue;
                for (int k = 0; k < nA + nB && ok; ++k) {
                    int t, j;
                    slot_of(k, nA, nB, t, j);
                    const uint32_t gg = g + uint32_t(k), st = gg % kStages;
                    ok = mbar_wait(bar(kBarKvFull + st), (gg / kStages) & 1, abort_flag);
                    if (ok) ok = mbar_wait(bar(kBarPFull + t), c[t] & 1, abort_flag);
                    if (ok && j == 0 && o[t] >= 1) ok = mbar_wait(bar(kBarOEmpty + t), (o[t] - 1) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const int nkk = info[st].y >= 0 ? 4 : 2;  // K = 128 or 64 keys
                    const uint32_t pa = sbase + kOffP + uint32_t(t) * kPTileBytes;
                    const uint32_t vb = sbase + kOffV + st * 2 * kVHalfBytes;
                    for (int kk = 0; kk < nkk; ++kk)
                        mma_f8(tmem + col_o(t), sdesc(pa + 32 * kk, 1024, SWZ_128B),
                               sdesc(vb + (kk >> 1) * kVHalfBytes + 32 * (kk & 1), 512, SWZ_64B), kIdescPV,
                               (j > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(bar(kBarPvDone + t));
                    // the QK of this slot completed before its P existed, so the stage is
                    // free once this PV completes
                    tc_commit(bar(kBarKvEmpty + st));
                    ++c[t];
                }
                for (int t = 0; t < 2 && ok; ++t) {
                    if ((t ? nB : nA) == 0) continue;
                    tc_commit(bar(kBarOFull + t));
                    ++o[t];
                }
                g += uint32_t(nA + nB);
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
        uint32_t g = 0, c = 0, o = 0, pi = 0;  // slots of earlier pairs; steps and tiles of this warpgroup
        for (int r = 0, p = item(0); p < npairs; p = item(++r), ++pi) {
            const int bh = pair_head(p), qa = pair_qa(p);
            int nA, nB;
            read_entry(pi, false, ok, nA, nB);
            ok = __all_sync(0xffffffffu, ok);
            nA = __shfl_sync(0xffffffffu, nA, 0);
            nB = __shfl_sync(0xffffffffu, nB, 0);
            __syncwarp();
            if (lane == 0) mbar_arrive(ebar(2 + int(pi & 1)));
            // a pair with no kept block at all still writes its rows (below, n == 0)
            const int qt = qa + t, n = t ? nB : nA, mn = min(nA, nB), total = nA + nB;
            const int qrow = qt * 128 + row;
            if (n == 0) {
                __nv_bfloat16 *orow = out + (int64_t(bh) * N + qrow) * kD;
                const float *arow = addend ? addend + (int64_t(bh) * N + qrow) * kD : nullptr;
                // no kept block (or no tile B): zero rows, or the addend rounded once
                if (qt < nq && qrow < N) {
#pragma unroll 1
                    for (int cidx = 0; cidx < 16; ++cidx) {
                        uint32_t w[4] = {0u, 0u, 0u, 0u};
                        if (arow) {
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const __nv_bfloat162 h2 =
                                    __floats2bfloat162_rn(arow[8 * cidx + 2 * e], arow[8 * cidx + 2 * e + 1]);
                                w[e] = *reinterpret_cast<const uint32_t *>(&h2);
                            }
                        }
                        reinterpret_cast<uint4 *>(orow)[cidx] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
                g += uint32_t(total);
                continue;
            }
            const float sq = q_scale[int64_t(bh) * nq + qt];
            const float *ksrow = k_scale + int64_t(bh) * nk;
            float m = -INFINITY;
            for (int j = 0; j < n; ++j, ++c) {
                const uint32_t gg = g + uint32_t(j < mn ? 2 * j + t : mn + j), st = gg % kStages;
                if (ok) ok = mbar_wait(bar(kBarKvFull + st), (gg / kStages) & 1, abort_flag);
                if (ok) ok = mbar_wait(bar(kBarSFull + t), c & 1, abort_flag);
                ok = __all_sync(0xffffffffu, ok);
                const int2 jp = ok ? info[st] : make_int2(0, -1);  // the stage's blocks once loaded
                const bool two = jp.y >= 0;
                const float ks0 = ksrow[jp.x], ks1 = two ? ksrow[jp.y] : 0.0f;
                int nv0 = min(64, N - 64 * jp.x), nv1 = two ? min(64, N - 64 * jp.y) : 0;
                if (causal) {
                    // this row keeps the keys up to itself
                    nv0 = max(0, min(nv0, qrow - 64 * jp.x + 1));
                    if (two) nv1 = max(0, min(nv1, qrow - 64 * jp.y + 1));
                }

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
                const float c0 = (sq * ks0) * sm_scale, c1 = (sq * ks1) * sm_scale;
                float pmax = nv0 > 0 ? i2f(uint32_t(max64x2(s0, s1))) * c0 : -INFINITY;
                if (nv1 > 0) pmax = fmaxf(pmax, i2f(uint32_t(max64x2(s2, s3))) * c1);
                const float mnew = fmaxf(m, pmax);
                // the S buffer goes to the next slot's QK only after the maximum
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarSEmpty));

                const float nbias = kLog2_448 - mnew * kLog2e;
                uint32_t pw[32];
                p_row(s0, s1, s2, s3, c0 * kLog2e, c1 * kLog2e, nbias, nv0, nv1, pw);

                // the P tile and O are free once the PV of this tile's previous step completed
                if (c >= 1 && ok) ok = mbar_wait(bar(kBarPvDone + t), (c - 1) & 1, abort_flag);
                ok = __all_sync(0xffffffffu, ok);
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
            g += uint32_t(total);
            // ---- epilogue: O = acc * scale_v / l (+ addend), bf16, 32 channels at a time
            if (ok) ok = mbar_wait(bar(kBarOFull + t), o & 1, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                tc_fence_after();
                uint32_t lbits;
                tmem_ld1_wait(oa + 128, lbits);
                const float l = __uint_as_float(lbits);
                const float inv_l = l > 0.0f ? __frcp_rn(l) : 0.0f;  // a row with no kept key gives 0
                const float *svp = v_scale + int64_t(bh) * kD;
                __nv_bfloat16 *orow = out + (int64_t(bh) * N + qrow) * kD;
                const float *arow = addend ? addend + (int64_t(bh) * N + qrow) * kD : nullptr;
#pragma unroll 1
                for (int h = 0; h < 4; ++h) {
                    uint32_t ov[32];
                    tmem_ld32_wait(oa + 32 * h, ov);
                    if (qrow < N) {
#pragma unroll
                        for (int cidx = 0; cidx < 4; ++cidx) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int i = 8 * cidx + 2 * e;
                                float y0 = (__uint_as_float(ov[i]) * svp[32 * h + i]) * inv_l;
                                float y1 = (__uint_as_float(ov[i + 1]) * svp[32 * h + i + 1]) * inv_l;
                                if (arow) {
                                    y0 += arow[32 * h + i];
                                    y1 += arow[32 * h + i + 1];
                                }
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
