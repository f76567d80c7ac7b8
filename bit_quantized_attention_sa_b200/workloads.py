"""Seeded synthetic inputs for the low-bit attention forward.

Shared by the tests, the benchmark and the oracle checks.  This module holds input
generation only (random draws, bf16 rounding of the draws, mask sampling); none of the
method's arithmetic lives here.

Recipe (video-DiT attention shapes; the pages measure on no public dataset, so seeded
synthetic tensors of the Wan2.1 latent shapes stand in for real activations):
  * one numpy ``Generator(PCG64(seed))`` stream, drawn in the order Q, K, V, K offsets,
    outlier-channel picks, mask;
  * Q, K, V ~ N(0, 1) in fp32, per head in token-major order;
  * K += off[b,h,c], off ~ N(0, 2^2), one offset per (head, channel) shared over tokens;
  * with ``outliers``: per (b,h), independently for Q and K, round(1% of d) channel(s)
    picked by the stream are multiplied by 8 (for K after the offset is added);
  * every tensor is rounded once from fp32 to bf16 (round to nearest, ties to even);
  * with ``mask_density``: a uint8 keep-mask over (128-query x 64-key) blocks
    [B,H,nq,nk], each off-diagonal block kept with probability ``mask_density``; the
    diagonal blocks j in {2i, 2i+1} (the key blocks overlapping query block i) are
    always kept.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

QBLK = 128
KBLK = 64


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int = 128
    outliers: bool = False
    mask_density: float | None = None
    seed: int = 0

    @property
    def sm_scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))

    @property
    def dense_ops(self) -> float:
        """4*B*H*N^2*d: the two contractions (Q.K^T and P.V) of dense attention."""
        return 4.0 * self.B * self.H * float(self.N) ** 2 * self.d


# The five workloads: a small parity case and four Wan2.1-latent-shaped ones
# (21x30x52 = 32760 tokens at 480p, 21x45x80 = 75600 tokens at 720p).
WORKLOADS = {
    "small-h2-n1024": Workload("small-h2-n1024", 1, 2, 1024, seed=1000),
    "wan1.3b-480p-h12-n32760": Workload("wan1.3b-480p-h12-n32760", 1, 12, 32760, seed=1001),
    "wan14b-480p-h40-n32760": Workload("wan14b-480p-h40-n32760", 1, 40, 32760, outliers=True,
                                       seed=1002),
    "wan14b-720p-h40-n75600": Workload("wan14b-720p-h40-n75600", 1, 40, 75600, outliers=True,
                                       seed=1003),
    "wan14b-480p-h40-n32760-sparse10": Workload("wan14b-480p-h40-n32760-sparse10", 1, 40,
                                                32760, outliers=True, mask_density=0.0965,
                                                seed=1004),
}
WORKLOAD_ORDER = list(WORKLOADS)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_heads(rng: np.random.Generator, B: int, H: int, N: int, d: int) -> np.ndarray:
    """N(0,1) fp32 [B,H,N,d], drawn head by head (same stream as one large draw)."""
    out = np.empty((B, H, N, d), np.float32)
    for b in range(B):
        for h in range(H):
            out[b, h] = rng.standard_normal((N, d), dtype=np.float32)
    return out


def make_inputs(B: int, H: int, N: int, d: int = 128, seed: int = 0, outliers: bool = False,
                mask_density: float | None = None, k_offset_std: float = 2.0):
    """Return (q, k, v, mask) with q/k/v uint16 bf16 bits [B,H,N,d] and mask uint8
    [B,H,nq,nk] or None, following the module recipe."""
    rng = np.random.Generator(np.random.PCG64(seed))
    qf = _normal_heads(rng, B, H, N, d)
    kf = _normal_heads(rng, B, H, N, d)
    vf = _normal_heads(rng, B, H, N, d)
    off = (rng.standard_normal((B, H, 1, d), dtype=np.float32) * np.float32(k_offset_std))
    kf += off
    if outliers:
        n_out = max(1, int(round(0.01 * d)))
        for b in range(B):
            for h in range(H):
                cq = rng.choice(d, size=n_out, replace=False)
                ck = rng.choice(d, size=n_out, replace=False)
                qf[b, h][:, cq] *= np.float32(8.0)
                kf[b, h][:, ck] *= np.float32(8.0)
    q = f32_to_bf16_bits(qf)
    del qf
    k = f32_to_bf16_bits(kf)
    del kf
    v = f32_to_bf16_bits(vf)
    del vf
    mask = None
    if mask_density is not None:
        nq, nk = -(-N // QBLK), -(-N // KBLK)
        mask = (rng.random((B, H, nq, nk), dtype=np.float32) < np.float32(mask_density))
        mask = mask.astype(np.uint8)
        for i in range(nq):
            for j in (2 * i, 2 * i + 1):
                if j < nk:
                    mask[:, :, i, j] = 1
    return q, k, v, mask


def make_workload(w: Workload):
    return make_inputs(w.B, w.H, w.N, w.d, seed=w.seed, outliers=w.outliers,
                       mask_density=w.mask_density)


def sample_rows(B: int, H: int, N: int, per_head: int, seed: int = 7):
    """Query rows for sampled checks: per head, rows from the first query block, the last
    (possibly ragged) block and random blocks, as [(bh, r), ...]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    rows = []
    last0 = ((N - 1) // QBLK) * QBLK
    for bh in range(B * H):
        cand = {0, min(N - 1, QBLK - 1), last0, N - 1}
        while len(cand) < min(per_head, N):
            cand.add(int(rng.integers(0, N)))
        rows.extend((bh, r) for r in sorted(cand)[:per_head] if r < N)
    return rows


# ---- linear layers (the W8A8 GEMM): activations x [M, K] and weights w [N, K] of the
# Wan2.1-14B transformer block (hidden 5120, feed-forward 13824) over the latent tokens.
@dataclass(frozen=True)
class LinearWorkload:
    name: str
    M: int
    N: int
    K: int
    seed: int = 0

    @property
    def ops(self) -> float:
        """2*M*N*K: one multiply and one add per term of the product."""
        return 2.0 * self.M * self.N * self.K


LINEAR_WORKLOADS = {
    "small-m300-n264-k1000": LinearWorkload("small-m300-n264-k1000", 300, 264, 1000, seed=2000),
    "wan14b-720p-ffn-up-m75600-n13824-k5120": LinearWorkload(
        "wan14b-720p-ffn-up-m75600-n13824-k5120", 75600, 13824, 5120, seed=2001),
    # a 16384-token slice of the same layer (codes of x and w together exceed L2), for
    # profiler captures that must stay small
    "wan14b-ffn-up-m16384-n13824-k5120": LinearWorkload(
        "wan14b-ffn-up-m16384-n13824-k5120", 16384, 13824, 5120, seed=2002),
}


def make_linear_inputs(M: int, N: int, K: int, seed: int = 0, outliers: bool = True):
    """Return (x, w), uint16 bf16 bits [M, K] and [N, K].

    Recipe: one ``Generator(PCG64(seed))`` stream drawn in the order x, w, outlier picks;
    x ~ N(0, 1) drawn in chunks of 4096 rows (same stream as one draw), w ~ N(0, 1) *
    K^-1/2; with ``outliers`` round(1% of K) activation channels (at least one), picked by
    the stream, are multiplied by 8 (the channel outliers of transformer activations);
    both rounded once from fp32 to bf16."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = np.empty((M, K), np.uint16)
    chunks = []
    for r0 in range(0, M, 4096):
        chunks.append((r0, rng.standard_normal((min(M, r0 + 4096) - r0, K), dtype=np.float32)))
    w = f32_to_bf16_bits(rng.standard_normal((N, K), dtype=np.float32) * np.float32(1.0 / np.sqrt(K)))
    cols = rng.choice(K, size=max(1, int(round(0.01 * K))), replace=False) if outliers else []
    for r0, xf in chunks:
        if len(cols):
            xf[:, cols] *= np.float32(8.0)
        x[r0:r0 + xf.shape[0]] = f32_to_bf16_bits(xf)
    return x, w


def make_linear_workload(w: LinearWorkload):
    return make_linear_inputs(w.M, w.N, w.K, seed=w.seed)


def make_sla_classes(B: int, H: int, N: int, p_critical: float, p_marginal: float, seed: int = 0):
    """uint8 [B,H,nq,nk] SLA block classes: each (128-query x 64-key) block is critical (2)
    with probability p_critical, marginal (1) with probability p_marginal, else negligible
    (0), from one ``Generator(PCG64(seed))`` draw of uniforms; the diagonal blocks
    j in {2i, 2i+1} are always critical."""
    nq, nk = -(-N // QBLK), -(-N // KBLK)
    rng = np.random.Generator(np.random.PCG64(seed))
    u = rng.random((B, H, nq, nk), dtype=np.float32)
    cls = np.where(u < np.float32(p_critical), 2, np.where(u < np.float32(p_critical + p_marginal), 1, 0))
    cls = cls.astype(np.uint8)
    for i in range(nq):
        for j in (2 * i, 2 * i + 1):
            if j < nk:
                cls[:, :, i, j] = 2
    return cls
