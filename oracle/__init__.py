"""CPU oracle for the SageAttention-style low-bit attention forward.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()`` and by
the CPU-baseline leg of ``bench.py``.  The product path (``bit_quantized_attention_sa_b200``
and its CUDA library) never imports, links or calls anything here.

This module is argument marshalling around ``sa_oracle.c`` (plain C11, built with gcc,
no fast-math, no FMA contraction); every step of the computation is in that file, with
its citations.  Arrays are numpy; bf16 tensors are passed as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sa_oracle.c")
_LIB = os.path.join(_HERE, "libsa_oracle.so")

QBLK = 128
KBLK = 64

_lib = None


def build(force: bool = False) -> str:
    """Compile sa_oracle.c into libsa_oracle.so next to it (gcc, IEEE semantics)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fPIC",
               "-shared", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        I64 = ctypes.c_int64
        lib.sa_oracle_e4m3_from_f32.argtypes = [ctypes.c_float]
        lib.sa_oracle_e4m3_from_f32.restype = ctypes.c_uint8
        lib.sa_oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        lib.sa_oracle_e4m3_to_f32.restype = ctypes.c_float
        lib.sa_oracle_quantize_qk.argtypes = [P, P, I, I, I, I, P, P, P, P, P]
        lib.sa_oracle_quantize_qk.restype = I
        lib.sa_oracle_quantize_v.argtypes = [P, I, I, I, I, P, P]
        lib.sa_oracle_quantize_v.restype = None
        lib.sa_oracle_attn_rows.argtypes = [P, P, P, P, P, P, I, I, I, I, ctypes.c_float, P,
                                            I, P, I64, P]
        lib.sa_oracle_attn_rows.restype = None
        lib.sa_oracle_exact_rows.argtypes = [P, P, P, I, I, I, I, ctypes.c_double, P, P, I64, P]
        lib.sa_oracle_exact_rows.restype = None
        lib.sa_oracle_qk_s32_rows.argtypes = [P, P, I, I, I, I, P, I64, P]
        lib.sa_oracle_qk_s32_rows.restype = None
        lib.sa_oracle_pool.argtypes = [P, I, I, I, I, I, P]
        lib.sa_oracle_pool.restype = I
        lib.sa_oracle_block_scores.argtypes = [P, P, I64, I, I, I, P]
        lib.sa_oracle_block_scores.restype = None
        lib.sa_oracle_block_mask.argtypes = [P, I64, I, I, I, I, P]
        lib.sa_oracle_block_mask.restype = None
        lib.sa_oracle_w8a8_quantize.argtypes = [P, I64, I64, P, P]
        lib.sa_oracle_w8a8_quantize.restype = None
        lib.sa_oracle_w8a8_gemm_rows.argtypes = [P, P, P, P, I64, I64, I64, P, I64, P]
        lib.sa_oracle_attn_rows_causal.argtypes = lib.sa_oracle_attn_rows.argtypes
        lib.sa_oracle_attn_rows_causal.restype = None
        lib.sa_oracle_exact_rows_causal.argtypes = lib.sa_oracle_exact_rows.argtypes
        lib.sa_oracle_exact_rows_causal.restype = None
        lib.sa_oracle_sla_linear_rows.argtypes = [P, P, P, I, I, I, I, P, I, P, P, I64, P]
        lib.sa_oracle_sla_linear_rows.restype = None
        lib.sa_oracle_w8a8_gemm_rows.restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def padded_len(n: int) -> int:
    return -(-n // QBLK) * QBLK


def e4m3_from_f32(x: float) -> int:
    return int(_load().sa_oracle_e4m3_from_f32(float(x)))


def e4m3_to_f32(b: int) -> float:
    return float(_load().sa_oracle_e4m3_to_f32(int(b)))


def quantize_qk(q: np.ndarray, k: np.ndarray):
    """q, k: uint16 bf16 bits [B,H,N,d].  Returns (q_i8, q_scale, k_i8, k_scale, k_mean,
    mean_exact) with the layouts of sa_oracle.c."""
    assert q.dtype == np.uint16 and k.dtype == np.uint16 and q.shape == k.shape
    B, H, N, d = q.shape
    Np, nq, nk = padded_len(N), -(-N // QBLK), -(-N // KBLK)
    q_i8 = np.empty((B, H, Np, d), np.int8)
    k_i8 = np.empty((B, H, Np, d), np.int8)
    q_scale = np.empty((B, H, nq), np.float32)
    k_scale = np.empty((B, H, nk), np.float32)
    k_mean = np.empty((B, H, d), np.float32)
    exact = _load().sa_oracle_quantize_qk(_ptr(q), _ptr(k), B, H, N, d, _ptr(q_i8),
                                          _ptr(q_scale), _ptr(k_i8), _ptr(k_scale),
                                          _ptr(k_mean))
    return q_i8, q_scale, k_i8, k_scale, k_mean, bool(exact)


def quantize_v(v: np.ndarray):
    """v: uint16 bf16 bits [B,H,N,d].  Returns (v_fp8_t [B,H,d,Npad] uint8, v_scale [B,H,d])."""
    assert v.dtype == np.uint16
    B, H, N, d = v.shape
    Np = padded_len(N)
    v_t = np.empty((B, H, d, Np), np.uint8)
    v_scale = np.empty((B, H, d), np.float32)
    _load().sa_oracle_quantize_v(_ptr(v), B, H, N, d, _ptr(v_t), _ptr(v_scale))
    return v_t, v_scale


def _rows_array(rows, B, H, N):
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
    assert rows.size == 0 or (rows[:, 0].min() >= 0 and rows[:, 0].max() < B * H
                              and rows[:, 1].min() >= 0 and rows[:, 1].max() < N)
    return rows


def attn_rows(qk, vq, N: int, sm_scale: float, rows, mask: np.ndarray | None = None,
              group: int = 2, causal: bool = False) -> np.ndarray:
    """Quantised attention for rows [(bh, r), ...] from quantize_qk / quantize_v outputs
    (causal: row r takes the keys t <= r only).  Returns fp32 [len(rows), d]."""
    q_i8, q_scale, k_i8, k_scale = qk[0], qk[1], qk[2], qk[3]
    v_t, v_scale = vq
    B, H, _, d = q_i8.shape
    rows = _rows_array(rows, B, H, N)
    if mask is not None:
        mask = np.ascontiguousarray(mask, dtype=np.uint8)
        assert mask.shape == (B, H, -(-N // QBLK), -(-N // KBLK))
    out = np.zeros((rows.shape[0], d), np.float32)
    fn = _load().sa_oracle_attn_rows_causal if causal else _load().sa_oracle_attn_rows
    fn(_ptr(q_i8), _ptr(q_scale), _ptr(k_i8), _ptr(k_scale),
                                _ptr(v_t), _ptr(v_scale), B, H, N, d, float(sm_scale),
                                _ptr(mask), int(group), _ptr(rows), rows.shape[0], _ptr(out))
    return out


def exact_rows(q, k, v, sm_scale: float, rows, mask: np.ndarray | None = None,
               causal: bool = False) -> np.ndarray:
    """fp64 softmax(q K^T sm_scale) V from the bf16 inputs for rows [(bh, r), ...]
    (causal: row r over the keys t <= r)."""
    B, H, N, d = q.shape
    rows = _rows_array(rows, B, H, N)
    if mask is not None:
        mask = np.ascontiguousarray(mask, dtype=np.uint8)
    out = np.zeros((rows.shape[0], d), np.float64)
    fn = _load().sa_oracle_exact_rows_causal if causal else _load().sa_oracle_exact_rows
    fn(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, float(sm_scale),
                                 _ptr(mask), _ptr(rows), rows.shape[0], _ptr(out))
    return out


def qk_s32_rows(q_i8: np.ndarray, k_i8: np.ndarray, N: int, rows) -> np.ndarray:
    """int32 S of the selected query rows against all padded key rows: [len(rows), Npad]."""
    B, H, Np, d = q_i8.shape
    rows = _rows_array(rows, B, H, N)
    out = np.zeros((rows.shape[0], Np), np.int32)
    _load().sa_oracle_qk_s32_rows(_ptr(q_i8), _ptr(k_i8), B, H, N, d, _ptr(rows),
                                  rows.shape[0], _ptr(out))
    return out


def pool(x: np.ndarray, blk: int):
    """Block means of bf16 bits x [B,H,N,d] over `blk`-token blocks: (fp32
    [B,H,ceil(N/blk),d], all_sums_exact)."""
    assert x.dtype == np.uint16
    B, H, N, d = x.shape
    out = np.empty((B, H, -(-N // blk), d), np.float32)
    exact = _load().sa_oracle_pool(_ptr(np.ascontiguousarray(x)), B, H, N, d, int(blk), _ptr(out))
    return out, bool(exact)


def block_scores(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """fp64 pooled scores [B,H,nq,nk] from block means qbar [B,H,nq,d], kbar [B,H,nk,d]."""
    B, H, nq, d = qbar.shape
    nk = kbar.shape[2]
    out = np.empty((B, H, nq, nk), np.float64)
    _load().sa_oracle_block_scores(_ptr(np.ascontiguousarray(qbar, np.float32)),
                                   _ptr(np.ascontiguousarray(kbar, np.float32)), B * H, nq, nk,
                                   d, _ptr(out))
    return out


def mask_from_scores(scores: np.ndarray, keep_per_row: int, keep_diagonal: bool = False) -> np.ndarray:
    """uint8 keep mask [B,H,nq,nk] from pooled scores (top keep_per_row per row)."""
    B, H, nq, nk = scores.shape
    out = np.empty((B, H, nq, nk), np.uint8)
    _load().sa_oracle_block_mask(_ptr(np.ascontiguousarray(scores, np.float64)), B * H, nq, nk,
                                 int(keep_per_row), int(bool(keep_diagonal)), _ptr(out))
    return out


def block_mask(q: np.ndarray, k: np.ndarray, keep_per_row: int, keep_diagonal: bool = False):
    """The whole selector: (mask uint8 [B,H,nq,nk], qbar, kbar, scores, pools_exact)."""
    qbar, ex_q = pool(q, QBLK)
    kbar, ex_k = pool(k, KBLK)
    scores = block_scores(qbar, kbar)
    return mask_from_scores(scores, keep_per_row, keep_diagonal), qbar, kbar, scores, ex_q and ex_k


def w8a8_quantize(x: np.ndarray):
    """x: bf16 bits [rows, cols].  Returns (codes int8 [rows, Kpad], scales fp32
    [ceil(rows/128), ceil(cols/128)]), Kpad = 128 * ceil(cols/128)."""
    assert x.dtype == np.uint16 and x.ndim == 2
    rows, cols = x.shape
    cb = -(-cols // 128)
    codes = np.empty((rows, cb * 128), np.int8)
    scales = np.empty((-(-rows // 128), cb), np.float32)
    _load().sa_oracle_w8a8_quantize(_ptr(np.ascontiguousarray(x)), rows, cols, _ptr(codes), _ptr(scales))
    return codes, scales


def w8a8_gemm_rows(xq, wq, K: int, rows) -> np.ndarray:
    """fp32 accumulator y [len(rows), N] of the W8A8 linear layer for the given rows of x,
    from w8a8_quantize(x) and w8a8_quantize(w)."""
    x8, sx = xq
    w8, sw = wq
    M, N = x8.shape[0], w8.shape[0]
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    assert rows.size == 0 or (rows.min() >= 0 and rows.max() < M)
    y = np.empty((rows.size, N), np.float32)
    _load().sa_oracle_w8a8_gemm_rows(_ptr(x8), _ptr(sx), _ptr(w8), _ptr(sw), M, N, K, _ptr(rows),
                                     rows.size, _ptr(y))
    return y


def sla_linear_rows(q, k, v, classes: np.ndarray, phi: int, proj: np.ndarray | None, rows) -> np.ndarray:
    """SLA linear branch for rows [(bh, r), ...]: kernelised linear attention over the
    marginal blocks (classes == 1) with feature map phi (0 softmax, 1 elu+1), projected by
    proj (fp32 [d, d], None = identity).  Returns fp64 [len(rows), d]."""
    B, H, N, d = q.shape
    rows = _rows_array(rows, B, H, N)
    classes = np.ascontiguousarray(classes, dtype=np.uint8)
    assert classes.shape == (B, H, -(-N // QBLK), -(-N // KBLK))
    if proj is not None:
        proj = np.ascontiguousarray(proj, dtype=np.float32)
        assert proj.shape == (d, d)
    out = np.zeros((rows.shape[0], d), np.float64)
    _load().sa_oracle_sla_linear_rows(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, _ptr(classes), int(phi),
                                      _ptr(proj), _ptr(rows), rows.shape[0], _ptr(out))
    return out
