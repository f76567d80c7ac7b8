"""Benchmark of the low-bit attention forward (prologue + fused attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one sa_attn_fwd call over the whole workload (K mean, Q/K INT8 quantisation,
V FP8 quantisation, fused INT8/FP8 attention), inputs resident in HBM.  Metric: tensor
ops 4*B*H*N^2*d per second (the two contractions of dense attention).  Rank 0 prints one
JSON line.  Under torchrun every rank runs its own replica of the workload (heads and
batches are independent: no collective on the data path) and the reported time is the
maximum over ranks.  ``--impl reference`` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_quantized_attention_sa_b200.workloads import (LINEAR_WORKLOADS, WORKLOADS, make_linear_workload,  # noqa: E402
                                                       make_sla_classes, make_workload)

METRIC = "quantized attention TOPS (4·H·N²·d/s) and % of B200 dense INT8/FP8 peak"
DEFAULT_WORKLOAD = "wan14b-720p-h40-n75600"
DEFAULT_LINEAR = "wan14b-720p-ffn-up-m75600-n13824-k5120"
DATASHEET_TOPS = 4500.0  # B200 dense INT8 / FP8 tensor peak (NVIDIA datasheet)
KERNELS_PER_STEP = 6      # k_partial, k_mean, qk_quant, v_amax, v_quant, attn_fwd


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def measured_peak():
    """8-bit tensor peak in TOPS from the measured bf16 cuBLAS burst figure times the
    nominal 8-bit/bf16 ratio (4.5 / 2.25 PFLOP/s dense)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            m = json.load(f)
        return 2.0 * float(m["bf16_tflops"]), "measured bf16 burst x 2 (nominal 8-bit/bf16 ratio)"
    except Exception:
        return 2.0 * 1590.0, "fallback 1.59 PFLOP/s bf16 x 2 (nominal 8-bit/bf16 ratio)"


KERNEL_SOURCES = ("sa_attn.cu", "sa_attn_pairs.cuh")


def kernel_source_sha256():
    """sha256 over the attention kernels' source files, in order."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "bit_quantized_attention_sa_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(kernel, workload):
    """DRAM bytes per attention launch from the committed ncu summary, if it was taken on
    the current kernel sources, for this kernel and this workload (else None)."""
    p = os.path.join(ROOT, "profiles", "attn_fwd_traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)
        if (rec.get("kernel_sources_sha256") != kernel_source_sha256() or rec.get("kernel") != kernel
                or rec.get("workload") != workload):
            return None
        return rec
    except Exception:
        return None


# ------------------------------------------------------------------------ ranks


def rank_workload(w, rank: int):
    """The workload a rank runs: rank 0 the named one, every other rank the same shapes
    with its own seed (replicas of independent heads, no data exchanged)."""
    if rank == 0:
        return w
    return type(w)(w.name, w.B, w.H, w.N, w.d, w.outliers, w.mask_density, w.seed + 7919 * rank)


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest of the ranks' values (the job takes as long as its slowest rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tops(ops_per_rank: float, world: int, t_max: float) -> float:
    """Throughput of the whole job: every rank's work over the slowest rank's time."""
    return ops_per_rank * world / t_max / 1e12


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------ CPU oracle arm


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(w, q, k, v, m, threads: int, heads: int, rows_per_block=None):
    """Times the CPU oracle, as it stands, on a bounded sample of the workload: for each of
    the first `heads` heads its prologue (K mean, Q/K and V quantisation) and the query rows
    of its first and its ragged last 128-query block (the first `rows_per_block` rows of
    each, if given).  `threads` host threads run disjoint (head, block) units; each calls the
    single-threaded C oracle, which releases the interpreter lock.  The prologue of a head
    serves all N of its rows, so the sampled rows are charged their share of its time.
    Returns (ops_equivalent, seconds, description, threads)."""
    import concurrent.futures as cf
    import oracle
    oracle.build()
    nq = -(-w.N // 128)
    blocks = [0] if nq == 1 else [0, nq - 1]
    heads = max(1, min(heads, w.B * w.H))
    hsel = [(b, h) for b in range(w.B) for h in range(w.H)][:heads]

    def prologue(bh):
        b, h = bh
        sl = (slice(b, b + 1), slice(h, h + 1))
        qh, kh, vh = (np.ascontiguousarray(x[sl]) for x in (q, k, v))
        mh = np.ascontiguousarray(m[sl]) if m is not None else None
        return oracle.quantize_qk(qh, kh), oracle.quantize_v(vh), mh

    def rows_of(blk):
        lo, hi = 128 * blk, min(128 * blk + 128, w.N)
        if rows_per_block is not None:
            hi = min(hi, lo + rows_per_block)
        return [(0, r) for r in range(lo, hi)]

    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        t0 = time.perf_counter()
        pro = list(ex.map(prologue, hsel))
        t_pro = time.perf_counter() - t0
        units = [(i, blk) for i in range(len(hsel)) for blk in blocks]
        t0 = time.perf_counter()
        list(ex.map(lambda u: oracle.attn_rows(pro[u[0]][0], pro[u[0]][1], w.N, w.sm_scale, rows_of(u[1]),
                                               pro[u[0]][2], 2), units))
        t_rows = time.perf_counter() - t0
    nrows = sum(len(rows_of(blk)) for blk in blocks)  # per head
    secs = t_rows + t_pro * nrows / w.N
    ops = 4.0 * nrows * len(hsel) * w.N * w.d
    what = "all rows" if rows_per_block is None else f"the first {rows_per_block} rows"
    desc = (f"{len(hsel)} head(s) of {w.name}: {what} of the first and ragged last query blocks "
            f"({nrows} rows per head, {t_rows:.2f} s) + their prologues ({t_pro:.2f} s, charged {nrows}/{w.N}); "
            f"C oracle, {threads} host thread(s) over {len(units)} (head, block) units; rate extrapolated to "
            f"the whole workload")
    return ops, secs, desc, threads


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    q, k, v, m = make_workload(w)
    cores = host_cores()
    heads = max(1, cores // 2)
    vals = []
    desc = ""
    for i in range(args.warmup + args.steps):
        ops, secs, desc, _ = oracle_sample(w, q, k, v, m, cores, heads, args.oracle_rows)
        if i >= args.warmup:
            vals.append(ops / secs / 1e12)
    value = float(np.median(vals)) if vals else 0.0
    dense_step_s = w.dense_ops / (value * 1e12) if value > 0 else None
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dense_step_s * 1e3 if dense_step_s else None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8+fp8e4m3 (emulated in fp32 on the CPU)", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                   "mask_density": w.mask_density, "sample": desc},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": desc, "extrapolated": True},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------ GPU arm


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--oracle-rows", type=int, default=16,
                    help="rows per query block in each step of the reference arm's oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sla", action="store_true", help="skip the SLA forward timing")
    ap.add_argument("--no-causal", action="store_true", help="skip the causal forward timing")
    ap.add_argument("--linear-workload", default=DEFAULT_LINEAR, choices=list(LINEAR_WORKLOADS) + ["none"],
                    help="W8A8 linear layer timed beside the attention step ('none' skips it)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=300))

    from bit_quantized_attention_sa_b200 import binding as sa

    # each rank owns one replica of the workload (its own seed)
    q, k, v, m = make_workload(rank_workload(w, rank))
    shape = (w.B, w.H, w.N, w.d)

    def pinned_bf16(a):
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
        return t.pin_memory()

    hq, hk, hv = pinned_bf16(q), pinned_bf16(k), pinned_bf16(v)
    dq, dk, dv = (t.to(dev) for t in (hq, hk, hv))
    dm = torch.from_numpy(m).to(dev) if m is not None else None
    do = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    ho = torch.empty(shape, dtype=torch.bfloat16).pin_memory()
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def slowest(x: float) -> float:
        return max_over_ranks(x, world, dev)

    def step():
        sa.sa_attn_fwd(dq, dk, dv, w.sm_scale, block_mask=dm, out=do)

    # ---- device-resident timing of the whole step
    for _ in range(args.warmup):
        step()
    assert sa.sa_get_device_status() == 0
    sampler = ClockSampler(local_rank)
    barrier()
    sampler.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    barrier()
    clocks = sampler.stop()
    t_step = slowest(e0.elapsed_time(e1) / 1e3 / args.steps)
    assert sa.sa_get_device_status() == 0

    # ---- the attention kernel alone (dominant kernel): per-launch duration
    q8, sq, k8, sk, _ = sa.sa_quantize_qk(dq, dk)
    vt, sv = sa.sa_quantize_v(dv)
    for _ in range(args.warmup):
        sa.sa_attn_fwd_quantized(q8, sq, k8, sk, vt, sv, w.N, w.sm_scale, dm, out=do)
    barrier()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(args.steps):
        sa.sa_attn_fwd_quantized(q8, sq, k8, sk, vt, sv, w.N, w.sm_scale, dm, out=do)
    a1.record(stream)
    barrier()
    t_attn = slowest(a0.elapsed_time(a1) / 1e3 / args.steps)

    # ---- the prologue alone (K mean, Q/K INT8, V FP8 into caller buffers): reported on its
    # own, as the selector/pack/dequant cost of a low-bit attention step
    for _ in range(args.warmup):
        sa.sa_quantize_qk(dq, dk)
        sa.sa_quantize_v(dv)
    barrier()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(args.steps):
        sa.sa_quantize_qk(dq, dk)
        sa.sa_quantize_v(dv)
    g1.record(stream)
    barrier()
    t_pro = slowest(g0.elapsed_time(g1) / 1e3 / args.steps)
    # bytes per (token, channel): read K (mean), Q and K (codes), V twice (maximum, codes) in bf16;
    # write q8, k8, v8: 2 + 4 + 4 + 3 = 13
    pro_bytes = 13 * w.B * w.H * w.N * w.d
    prologue = {"ms": t_pro * 1e3, "share_of_step": t_pro / t_step,
                "steps": "sa_quantize_qk (K mean, Q INT8, smoothed K INT8) + sa_quantize_v (V FP8, transposed)",
                "algorithmic_bytes": pro_bytes, "gbs": pro_bytes / t_pro / 1e9}
    del q8, k8, vt

    # ---- this device's own 8-bit tensor-core rate: chains of four M128 N256 K32 tcgen05
    # MMAs from every SM, kind::i8 and kind::f8f6f4 (e4m3), timed on the stream
    def mma_rate(kind):
        sa.sa_debug_mma_peak(kind, 256)
        best = 0.0
        for _ in range(5):
            r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            r0.record(stream)
            ops_p = sa.sa_debug_mma_peak(kind, 65536)
            r1.record(stream)
            torch.cuda.synchronize(dev)
            best = max(best, ops_p / (r0.elapsed_time(r1) * 1e-3) / 1e12)
        return best
    peak_sampler = ClockSampler(local_rank)
    peak_sampler.start()
    time.sleep(0.2)
    peak_i8, peak_f8 = mma_rate(0), mma_rate(1)
    peak_clocks = peak_sampler.stop()
    assert sa.sa_get_device_status() == 0
    # the attention kernel's operations are half kind::i8 (Q.K^T) and half e4m3 (P.V)
    peak_8bit = 2.0 / (1.0 / peak_i8 + 1.0 / peak_f8)

    # ---- end to end through the public API with host buffers: sa_attn_fwd_host uploads
    # q, k, v (and the mask) from page-locked memory and downloads O, in chunks of heads
    # whose copies overlap the computation
    h2d = 3 * hq.numel() * 2 + (dm.numel() if dm is not None else 0)
    d2h = ho.numel() * 2
    hm = dm.cpu().pin_memory() if dm is not None else None
    for _ in range(1):
        sa.sa_attn_fwd_host(hq, hk, hv, out=ho, sm_scale=w.sm_scale, block_mask=hm, stream=stream)
    barrier()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(1, min(args.steps, 5))
    b0.record(stream)
    for _ in range(e2e_steps):
        sa.sa_attn_fwd_host(hq, hk, hv, out=ho, sm_scale=w.sm_scale, block_mask=hm, stream=stream)
    b1.record(stream)
    barrier()
    t_e2e = slowest(b0.elapsed_time(b1) / 1e3 / e2e_steps)

    # ---- the block-mask producer (selector), timed on its own for masked workloads: it
    # would run ahead of a masked forward; keep_per_row matches the workload's density
    selector = None
    if dm is not None:
        nk = -(-w.N // 64)
        keep = max(1, round(w.mask_density * nk))
        sel = torch.empty_like(dm)
        for _ in range(args.warmup):
            sa.sa_block_mask(dq, dk, keep, True, out=sel)
        barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(args.steps):
            sa.sa_block_mask(dq, dk, keep, True, out=sel)
        s1.record(stream)
        barrier()
        selector = {"ms": slowest(s0.elapsed_time(s1) / args.steps), "keep_per_row": keep,
                    "keep_diagonal": True, "kept_fraction": float(sel.float().mean().item())}
        del sel

    peak, peak_src = measured_peak()

    # ---- the causal forward on the same inputs: each 128-query tile visits the 64-key
    # blocks up to its diagonal pair; ops counted over the blocks executed
    causal = None
    if not args.no_causal and w.mask_density is None:
        nq, nk = -(-w.N // 128), -(-w.N // 64)
        blocks = sum(min(2 * i + 2, nk) for i in range(nq)) * w.B * w.H
        ops_causal = 4.0 * 128 * 64 * w.d * blocks
        for _ in range(args.warmup):
            sa.sa_attn_fwd_causal(dq, dk, dv, w.sm_scale, out=do)
        barrier()
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(args.steps):
            sa.sa_attn_fwd_causal(dq, dk, dv, w.sm_scale, out=do)
        c1.record(stream)
        barrier()
        t_causal = slowest(c0.elapsed_time(c1) / 1e3 / args.steps)
        assert sa.sa_get_device_status() == 0
        causal = {"step": "sa_attn_fwd_causal: prologue + the two-tile kernel over the blocks up to each "
                          "tile pair's diagonal, keys after each row dropped",
                  "ms": t_causal * 1e3, "executed_block_fraction": blocks / (w.B * w.H * nq * nk),
                  "executed_tops": whole_job_tops(ops_causal, world, t_causal)}

    # ---- the SLA forward on the same inputs: sparse quantised attention over the critical
    # blocks plus linear attention over the marginal blocks, projected
    sla = None
    if not args.no_sla:
        p_crit, p_marg = 0.0965, 0.4
        cls = torch.from_numpy(make_sla_classes(w.B, w.H, w.N, p_crit, p_marg, seed=w.seed + 1)).to(dev)
        proj = torch.from_numpy((np.random.default_rng(w.seed).standard_normal((w.d, w.d)) / math.sqrt(w.d))
                                .astype(np.float32)).to(dev)
        lin_out = torch.empty(shape, dtype=torch.float32, device=dev)

        def timed_sla(fn):
            for _ in range(args.warmup):
                fn()
            barrier()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for _ in range(args.steps):
                fn()
            t1.record(stream)
            barrier()
            return slowest(t0.elapsed_time(t1) / 1e3 / args.steps)

        t_sla = timed_sla(lambda: sa.sa_sla_fwd(dq, dk, dv, cls, w.sm_scale, proj=proj, out=do))
        t_lin = timed_sla(lambda: sa.sa_sla_linear(dq, dk, dv, cls, proj=proj, out=lin_out))
        assert sa.sa_get_device_status() == 0
        sla = {"step": "sa_sla_fwd: quantised attention on critical blocks + projected linear attention on "
                       "marginal blocks (phi = softmax over features)",
               "classes": {"critical": float((cls >= 2).float().mean().item()),
                           "marginal": float((cls == 1).float().mean().item()),
                           "recipe": f"critical p={p_crit} (+ diagonal), marginal p={p_marg}, else skipped"},
               "ms": t_sla * 1e3, "linear_branch_ms": t_lin * 1e3,
               "dense_equivalent_tops": whole_job_tops(w.dense_ops, world, t_sla)}
        del cls, proj, lin_out

    # ---- the W8A8 linear layer (INT8 GEMM with 128x128 block scales) on a Wan2.1-14B
    # feed-forward shape: the quantiser + GEMM call, and the GEMM kernel alone
    w8a8 = None
    if args.linear_workload != "none":
        del dq, dk, dv
        lw = LINEAR_WORKLOADS[args.linear_workload]
        x_bits, w_bits = make_linear_workload(lw)
        dx = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).to(dev)
        dw = torch.from_numpy(w_bits.view(np.int16)).view(torch.bfloat16).to(dev)
        del x_bits, w_bits
        wq = sa.sa_w8a8_quantize(dw)
        xq = sa.sa_w8a8_quantize(dx)
        dy = torch.empty((lw.M, lw.N), dtype=torch.bfloat16, device=dev)

        def timed(fn):
            for _ in range(args.warmup):
                fn()
            barrier()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for _ in range(args.steps):
                fn()
            t1.record(stream)
            barrier()
            return slowest(t0.elapsed_time(t1) / 1e3 / args.steps)

        t_lin = timed(lambda: sa.sa_w8a8_linear(dx, wq, out=dy))
        t_gemm = timed(lambda: sa.sa_w8a8_gemm(xq, wq, lw.K, out=dy))
        assert sa.sa_get_device_status() == 0
        gemm_tops = lw.ops / t_gemm / 1e12
        w8a8 = {"workload": lw.name, "M": lw.M, "N": lw.N, "K": lw.K, "ops": lw.ops,
                "step": "sa_w8a8_linear: x block quantisation + block-scaled INT8 GEMM, bf16 out",
                "value": whole_job_tops(lw.ops, world, t_lin), "unit": "TOPS", "ms": t_lin * 1e3,
                "roofline": {"bound": "tensor", "kernel": "w8a8_gemm_kernel", "achieved": gemm_tops,
                             "peak": peak, "unit": "TOPS", "frac": gemm_tops / peak, "peak_source": peak_src,
                             "ms_per_launch": t_gemm * 1e3}}
        del dx, dw, xq, wq, dy

    ops_rank = w.dense_ops
    value = whole_job_tops(ops_rank, world, t_step)
    # the kernel's roofline counts the operations it executes: with a keep mask, those of
    # the kept blocks (4 * d * 128 * 64 per block); the headline value stays dense-equivalent
    ops_kernel = 4.0 * w.d * 128 * 64 * float(m.sum()) if (w.mask_density is not None and m is not None) else ops_rank
    achieved = ops_kernel / t_attn / 1e12
    kernel = "attn_mpairs_kernel" if w.mask_density is not None else "attn_pairs_kernel"
    traffic = recorded_traffic(kernel, w.name)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # two legs of the oracle as it stands, on the host cores of this run: one thread on one
        # head, and one thread per host core over heads x (first, last) query blocks
        cores = host_cores()
        ops1, secs1, desc1, _ = oracle_sample(w, q, k, v, m, 1, 1)
        opsn, secsn, descn, _ = oracle_sample(w, q, k, v, m, cores, max(1, cores // 2))
        cpu = {"value": opsn / secsn / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": descn, "extrapolated": True,
               "single_threaded": {"value": ops1 / secs1 / 1e12, "unit": "TFLOP/s", "cores": 1,
                                   "sample": desc1, "extrapolated": True}}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int8+fp8e4m3", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                       "mask_density": w.mask_density, "sm_scale": w.sm_scale,
                       "step": "sa_attn_fwd: K mean + Q/K INT8 + V FP8 prologue + fused attention",
                       "l2": "inputs larger than L2 (each bf16 tensor %.0f MB)" % (h2d / 3 / 1e6),
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "tensor", "kernel": kernel,
                         "ops": "kept blocks, 4*d*128*64 each" if ops_kernel != ops_rank else "dense, 4*B*H*N^2*d",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "peak_source": peak_src,
                         "frac_of_datasheet_4500": achieved / DATASHEET_TOPS,
                         "measured_8bit_mma": {"i8_tops": peak_i8, "e4m3_tops": peak_f8, "combined_tops": peak_8bit,
                                               "frac": achieved / peak_8bit, "clocks": peak_clocks,
                                               "how": "sa_debug_mma_peak: every SM issues chains of four "
                                                      "M128 N256 K32 tcgen05 MMAs from shared memory, CUDA "
                                                      "events, best of 5; combined = harmonic mean (the "
                                                      "kernel's ops are half of each kind)"},
                         "ms_per_launch": t_attn * 1e3,
                         "traffic": traffic["dram_bytes_per_launch"] if traffic else None},
            "cpu_baseline": cpu,
            "e2e": {"value": whole_job_tops(ops_rank, world, t_e2e), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": t_e2e * 1e3},
            "gpu_launches": KERNELS_PER_STEP * args.steps,
            "clocks": clocks,
            "prologue": prologue,
        }
        if causal is not None:
            line["causal"] = causal
        if sla is not None:
            line["sla"] = sla
        if w8a8 is not None:
            line["w8a8"] = w8a8
        if w.mask_density is not None and m is not None:
            kept = int(m.sum())
            exe = 4.0 * w.d * 128 * 64 * kept
            line["config"]["mask_kept_fraction"] = kept / m.size
            line["executed_tflops"] = exe / t_step / 1e12 * world
            line["selector"] = selector
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
