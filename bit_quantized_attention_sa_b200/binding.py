"""Python binding of libsa.so: the C-ABI entry points of include/sa.h under the same
names, taking torch tensors.  This module only marshals arguments (checks dtypes and
shapes, allocates outputs with torch, passes raw pointers and the current CUDA stream);
every step of the computation runs in the library's CUDA kernels.  There is no CPU
fallback: importing this module raises if the library has not been built.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libsa.so")

if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build it with `python -m bit_quantized_attention_sa_b200.build`"
        " (there is no CPU fallback)")

_lib = ctypes.CDLL(_LIB_PATH)
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float

_lib.sa_quantize_qk.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]
_lib.sa_quantize_qk_noalloc.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]
_lib.sa_quantize_v.argtypes = [_P, _I, _I, _I, _I, _P, _P, _P]
_lib.sa_attn_fwd.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _F, _P, _P]
_lib.sa_attn_fwd_host.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _F, _P, _P]
_lib.sa_attn_fwd_causal.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _F, _P, _P]
_lib.sa_attn_fwd_varlen.argtypes = [_P, _P, _P, _P, _I, _P, _I, _I, _F, _I, _P]
_lib.sa_debug_varlen_groups.argtypes = [_I, _P, _I, _P]
_lib.sa_debug_varlen_groups.restype = _I
_lib.sa_attn_fwd_quantized.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _P, _P]
_lib.sa_debug_qk_s32.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P]
_lib.sa_block_mask.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P]
_lib.sa_debug_pool.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P, _P]
_lib.sa_w8a8_quantize.argtypes = [_P, _I, _I, _P, _P, _P]
_lib.sa_w8a8_gemm.argtypes = [_P, _P, _P, _P, _I, _I, _I, _P, _P]
_lib.sa_w8a8_linear.argtypes = [_P, _P, _P, _I, _I, _I, _P, _P]
_lib.sa_sla_linear.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P]
_lib.sa_sla_fwd.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _F, _P, _I, _P, _P]
_lib.sa_debug_wait_timeout.argtypes = [_I, _P]
_lib.sa_debug_mma_peak.argtypes = [_I, _I, _P]
_lib.sa_get_device_status.argtypes = []
_lib.sa_status_string.argtypes = [_I]
_lib.sa_status_string.restype = ctypes.c_char_p
_lib.sa_workspace_bytes.argtypes = [_I, _I, _I, _I]
_lib.sa_workspace_bytes.restype = ctypes.c_size_t
_lib.sa_release_workspace.argtypes = []
_lib.sa_padded_len.argtypes = [_I]
_lib.sa_padded_len.restype = ctypes.c_int64
for _name in ("sa_quantize_qk", "sa_quantize_qk_noalloc", "sa_quantize_v", "sa_attn_fwd", "sa_attn_fwd_host",
              "sa_attn_fwd_causal", "sa_attn_fwd_varlen",
              "sa_attn_fwd_quantized",
              "sa_debug_qk_s32", "sa_block_mask", "sa_debug_pool", "sa_w8a8_quantize", "sa_w8a8_gemm", "sa_w8a8_linear", "sa_sla_linear", "sa_sla_fwd", "sa_debug_wait_timeout", "sa_debug_mma_peak", "sa_get_device_status",
              "sa_release_workspace"):
    getattr(_lib, _name).restype = _I

SA_OK = 0
STATUS_NAMES = {0: "SA_OK", 1: "SA_ERR_INVALID_ARG", 2: "SA_ERR_UNSUPPORTED",
                3: "SA_ERR_MISALIGNED", 4: "SA_ERR_CUDA", 5: "SA_ERR_OOM",
                6: "SA_ERR_DEVICE_TIMEOUT", 7: "SA_ERR_SCRATCH_LIMIT"}


class SAError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what} failed: {sa_status_string(status)} ({status})")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def raw_library() -> ctypes.CDLL:
    """The ctypes handle itself (for tests of the C ABI)."""
    return _lib


def sa_status_string(status: int) -> str:
    return _lib.sa_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != SA_OK:
        raise SAError(status, what)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dims(q: torch.Tensor):
    if q.dim() != 4:
        raise ValueError("expected a [B, H, N, d] tensor")
    B, H, N, d = q.shape
    return int(B), int(H), int(N), int(d)


def _need(t: torch.Tensor, dtype: torch.dtype, name: str):
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")


def padded_len(N: int) -> int:
    return int(_lib.sa_padded_len(int(N)))


def sa_quantize_qk(q: torch.Tensor, k: torch.Tensor):
    """Returns (q_i8 [B,H,Npad,d], q_scale [B,H,nq], k_i8 [B,H,Npad,d], k_scale [B,H,nk],
    k_mean [B,H,d])."""
    _need(q, torch.bfloat16, "q")
    _need(k, torch.bfloat16, "k")
    B, H, N, d = _dims(q)
    if tuple(k.shape) != (B, H, N, d):
        raise ValueError("q and k shapes differ")
    Np, nq, nk = padded_len(N), -(-N // 128), -(-N // 64)
    dev = q.device
    q_i8 = torch.empty((B, H, Np, d), dtype=torch.int8, device=dev)
    k_i8 = torch.empty((B, H, Np, d), dtype=torch.int8, device=dev)
    q_scale = torch.empty((B, H, nq), dtype=torch.float32, device=dev)
    k_scale = torch.empty((B, H, nk), dtype=torch.float32, device=dev)
    k_mean = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    _check(_lib.sa_quantize_qk(_ptr(q), _ptr(k), B, H, N, d, _ptr(q_i8), _ptr(q_scale),
                               _ptr(k_i8), _ptr(k_scale), _ptr(k_mean), _stream(dev)),
           "sa_quantize_qk")
    return q_i8, q_scale, k_i8, k_scale, k_mean


def sa_quantize_v(v: torch.Tensor):
    """Returns (v_fp8_t uint8 e4m3 [B,H,d,Npad], v_scale [B,H,d])."""
    _need(v, torch.bfloat16, "v")
    B, H, N, d = _dims(v)
    Np = padded_len(N)
    v_t = torch.empty((B, H, d, Np), dtype=torch.uint8, device=v.device)
    v_scale = torch.empty((B, H, d), dtype=torch.float32, device=v.device)
    _check(_lib.sa_quantize_v(_ptr(v), B, H, N, d, _ptr(v_t), _ptr(v_scale), _stream(v.device)),
           "sa_quantize_v")
    return v_t, v_scale


def _mask_arg(block_mask, B, H, N, device):
    if block_mask is None:
        return None
    _need(block_mask, torch.uint8, "block_mask")
    if tuple(block_mask.shape) != (B, H, -(-N // 128), -(-N // 64)) or block_mask.device != device:
        raise ValueError("block_mask must be uint8 [B, H, ceil(N/128), ceil(N/64)] on q's device")
    return block_mask


def sa_attn_fwd(q, k, v, sm_scale: float | None = None, block_mask=None, out=None):
    """bf16 [B,H,N,d] q, k, v -> bf16 O.  sm_scale defaults to 1/sqrt(d)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    B, H, N, d = _dims(q)
    if tuple(k.shape) != (B, H, N, d) or tuple(v.shape) != (B, H, N, d):
        raise ValueError("q, k, v shapes differ")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    m = _mask_arg(block_mask, B, H, N, q.device)
    o = torch.empty_like(q) if out is None else out
    _need(o, torch.bfloat16, "out")
    _check(_lib.sa_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, d, float(sm_scale),
                            _ptr(m), _stream(q.device)), "sa_attn_fwd")
    return o


def sa_attn_fwd_causal(q, k, v, sm_scale: float | None = None, block_mask=None, out=None):
    """Causal forward: query row r attends to the keys t <= r (and the kept blocks of
    block_mask, if given)."""
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, name)
    B, H, N, d = _dims(q)
    if tuple(k.shape) != (B, H, N, d) or tuple(v.shape) != (B, H, N, d):
        raise ValueError("q, k and v shapes differ")
    scale = 1.0 / math.sqrt(d) if sm_scale is None else float(sm_scale)
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q.device) if out is None else out
    _need(o, torch.bfloat16, "out")
    m = _mask_arg(block_mask, B, H, N, q.device)
    _check(_lib.sa_attn_fwd_causal(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, d, scale, _ptr(m),
                                   _stream(q.device)), "sa_attn_fwd_causal")
    return o


def sa_debug_varlen_groups(seqlens, H: int):
    """The launch groups sa_attn_fwd_varlen forms for these lengths (host only): a list with
    the group of each sequence, groups numbered in launch order."""
    lens = [int(n) for n in seqlens]
    arr = (ctypes.c_int * len(lens))(*lens)
    out = (ctypes.c_int * len(lens))()
    n = _lib.sa_debug_varlen_groups(len(lens), arr, int(H), out)
    if n < 0:
        raise ValueError("sa_debug_varlen_groups: bad arguments")
    return list(out)


def sa_attn_fwd_varlen(q, k, v, seqlens, H: int, sm_scale: float | None = None, causal: bool = False, out=None,
                       d: int = 128):
    """Packed variable-length batch: q, k, v contiguous bf16 CUDA tensors of H * sum(seqlens)
    * d elements (any shape; sequence i is its [1, H, N_i, d] block after the earlier
    sequences').  Returns o of the same shape."""
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, name)
    lens = [int(n) for n in seqlens]
    d = int(d)
    if q.numel() != H * sum(lens) * d or k.numel() != q.numel() or v.numel() != q.numel():
        raise ValueError("q, k and v must hold H * sum(seqlens) * d elements")
    scale = 1.0 / math.sqrt(d) if sm_scale is None else float(sm_scale)
    o = torch.empty_like(q) if out is None else out
    _need(o, torch.bfloat16, "out")
    arr = (ctypes.c_int * len(lens))(*lens)
    _check(_lib.sa_attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), len(lens), arr, int(H), d, scale,
                                   int(bool(causal)), _stream(q.device)), "sa_attn_fwd_varlen")
    return o


def sa_attn_fwd_host(q, k, v, out=None, sm_scale: float | None = None, block_mask=None,
                     stream: torch.cuda.Stream | None = None):
    """bf16 [B,H,N,d] CPU tensors (pin_memory() for overlapped copies) -> bf16 CPU O.  The
    copies and the computation are enqueued on `stream` (default: the current CUDA stream);
    O is complete once that stream reaches this point (e.g. after stream.synchronize()), and
    the input tensors must be kept alive until then."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous CPU bf16 tensor")
    B, H, N, d = _dims(q)
    if tuple(k.shape) != (B, H, N, d) or tuple(v.shape) != (B, H, N, d):
        raise ValueError("q, k, v shapes differ")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if block_mask is not None:
        if block_mask.is_cuda or block_mask.dtype != torch.uint8 or not block_mask.is_contiguous() \
                or tuple(block_mask.shape) != (B, H, -(-N // 128), -(-N // 64)):
            raise ValueError("block_mask must be a contiguous CPU uint8 [B, H, ceil(N/128), ceil(N/64)]")
    o = torch.empty_like(q, pin_memory=q.is_pinned()) if out is None else out
    if o.is_cuda or o.dtype != torch.bfloat16 or not o.is_contiguous() or o.shape != q.shape:
        raise ValueError("out must be a contiguous CPU bf16 tensor shaped like q")
    st = torch.cuda.current_stream() if stream is None else stream
    _check(_lib.sa_attn_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, d, float(sm_scale),
                                 _ptr(block_mask), ctypes.c_void_p(st.cuda_stream)), "sa_attn_fwd_host")
    return o


def sa_attn_fwd_quantized(q_i8, q_scale, k_i8, k_scale, v_fp8_t, v_scale, N: int,
                          sm_scale: float | None = None, block_mask=None, out=None):
    """The attention kernel on quantised inputs (layouts of sa_quantize_qk/v)."""
    _need(q_i8, torch.int8, "q_i8")
    _need(k_i8, torch.int8, "k_i8")
    _need(v_fp8_t, torch.uint8, "v_fp8_t")
    for t, n in ((q_scale, "q_scale"), (k_scale, "k_scale"), (v_scale, "v_scale")):
        _need(t, torch.float32, n)
    B, H, Np, d = _dims(q_i8)
    if Np != padded_len(N):
        raise ValueError("q_i8 is not padded to 128 * ceil(N/128) rows")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    m = _mask_arg(block_mask, B, H, N, q_i8.device)
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q_i8.device) if out is None else out
    _need(o, torch.bfloat16, "out")
    _check(_lib.sa_attn_fwd_quantized(_ptr(q_i8), _ptr(q_scale), _ptr(k_i8), _ptr(k_scale),
                                      _ptr(v_fp8_t), _ptr(v_scale), _ptr(o), B, H, N, d,
                                      float(sm_scale), _ptr(m), _stream(q_i8.device)),
           "sa_attn_fwd_quantized")
    return o


def sa_block_mask(q, k, keep_per_row: int, keep_diagonal: bool = False, out=None):
    """Keep mask uint8 [B,H,ceil(N/128),ceil(N/64)] for bf16 [B,H,N,d] CUDA q, k: the
    keep_per_row best key blocks per query block by pooled score (plus the diagonal)."""
    _need(q, torch.bfloat16, "q")
    _need(k, torch.bfloat16, "k")
    B, H, N, d = _dims(q)
    if tuple(k.shape) != (B, H, N, d):
        raise ValueError("q and k shapes differ")
    shape = (B, H, -(-N // 128), -(-N // 64))
    m = torch.empty(shape, dtype=torch.uint8, device=q.device) if out is None else out
    _need(m, torch.uint8, "out")
    _check(_lib.sa_block_mask(_ptr(q), _ptr(k), B, H, N, d, int(keep_per_row), int(bool(keep_diagonal)),
                              _ptr(m), _stream(q.device)), "sa_block_mask")
    return m


def sa_debug_pool(q, k):
    """Block means (qbar fp32 [B,H,ceil(N/128),d], kbar fp32 [B,H,ceil(N/64),d])."""
    _need(q, torch.bfloat16, "q")
    _need(k, torch.bfloat16, "k")
    B, H, N, d = _dims(q)
    qbar = torch.empty((B, H, -(-N // 128), d), dtype=torch.float32, device=q.device)
    kbar = torch.empty((B, H, -(-N // 64), d), dtype=torch.float32, device=q.device)
    _check(_lib.sa_debug_pool(_ptr(q), _ptr(k), B, H, N, d, _ptr(qbar), _ptr(kbar), _stream(q.device)),
           "sa_debug_pool")
    return qbar, kbar


def _matrix(t: torch.Tensor, name: str):
    if t.dim() != 2:
        raise ValueError(f"{name} must be a 2-D tensor")
    return int(t.shape[0]), int(t.shape[1])


def sa_w8a8_quantize(x: torch.Tensor):
    """128 x 128 block quantisation of bf16 x [rows, cols]: (codes int8 [rows, kpad],
    scales fp32 [ceil(rows/128), kpad/128]), kpad = 128 * ceil(cols/128)."""
    _need(x, torch.bfloat16, "x")
    rows, cols = _matrix(x, "x")
    kpad = -(-cols // 128) * 128
    codes = torch.empty((rows, kpad), dtype=torch.int8, device=x.device)
    scales = torch.empty((-(-rows // 128), kpad // 128), dtype=torch.float32, device=x.device)
    _check(_lib.sa_w8a8_quantize(_ptr(x), rows, cols, _ptr(codes), _ptr(scales), _stream(x.device)),
           "sa_w8a8_quantize")
    return codes, scales


def _w8a8_out(M, N, device, out):
    y = torch.empty((M, N), dtype=torch.bfloat16, device=device) if out is None else out
    _need(y, torch.bfloat16, "out")
    if tuple(y.shape) != (M, N):
        raise ValueError("out has the wrong shape")
    return y


def sa_w8a8_gemm(xq, wq, K: int, out=None):
    """bf16 y [M, N] = the block-scaled INT8 product of xq = (codes [M, kpad], scales) and
    wq = (codes [N, kpad], scales), as returned by sa_w8a8_quantize of x [M, K], w [N, K]."""
    (xc, xs), (wc, ws) = xq, wq
    for t, dt, name in ((xc, torch.int8, "x codes"), (xs, torch.float32, "x scales"),
                        (wc, torch.int8, "w codes"), (ws, torch.float32, "w scales")):
        _need(t, dt, name)
    M, kpad = _matrix(xc, "x codes")
    N, kpad_w = _matrix(wc, "w codes")
    if kpad != kpad_w or kpad != -(-int(K) // 128) * 128:
        raise ValueError("codes widths do not match K")
    y = _w8a8_out(M, N, xc.device, out)
    _check(_lib.sa_w8a8_gemm(_ptr(xc), _ptr(xs), _ptr(wc), _ptr(ws), M, N, int(K), _ptr(y), _stream(xc.device)),
           "sa_w8a8_gemm")
    return y


def sa_w8a8_linear(x: torch.Tensor, wq, out=None):
    """bf16 y [M, N] = W8A8 linear layer of bf16 x [M, K] with the pre-quantised weight
    wq = (codes [N, kpad], scales) of w [N, K]."""
    wc, ws = wq
    _need(x, torch.bfloat16, "x")
    _need(wc, torch.int8, "w codes")
    _need(ws, torch.float32, "w scales")
    M, K = _matrix(x, "x")
    N, kpad = _matrix(wc, "w codes")
    if kpad != -(-K // 128) * 128:
        raise ValueError("w codes width does not match K")
    y = _w8a8_out(M, N, x.device, out)
    _check(_lib.sa_w8a8_linear(_ptr(x), _ptr(wc), _ptr(ws), M, N, K, _ptr(y), _stream(x.device)),
           "sa_w8a8_linear")
    return y


SA_PHI_SOFTMAX, SA_PHI_ELU1 = 0, 1


def _sla_args(q, k, v, classes, proj):
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, name)
    B, H, N, d = _dims(q)
    if tuple(k.shape) != (B, H, N, d) or tuple(v.shape) != (B, H, N, d):
        raise ValueError("q, k and v shapes differ")
    _need(classes, torch.uint8, "classes")
    if tuple(classes.shape) != (B, H, -(-N // 128), -(-N // 64)):
        raise ValueError("classes must be uint8 [B, H, ceil(N/128), ceil(N/64)]")
    if proj is not None:
        _need(proj, torch.float32, "proj")
        if tuple(proj.shape) != (d, d):
            raise ValueError("proj must be fp32 [d, d]")
    return B, H, N, d


def sa_sla_linear(q, k, v, classes, phi: int = SA_PHI_SOFTMAX, proj=None, out=None):
    """SLA linear branch: fp32 [B,H,N,d] = proj-projected linear attention of each row over
    its marginal blocks (classes == 1); phi SA_PHI_SOFTMAX or SA_PHI_ELU1."""
    B, H, N, d = _sla_args(q, k, v, classes, proj)
    o = torch.empty((B, H, N, d), dtype=torch.float32, device=q.device) if out is None else out
    _need(o, torch.float32, "out")
    _check(_lib.sa_sla_linear(_ptr(q), _ptr(k), _ptr(v), _ptr(classes), B, H, N, d, int(phi), _ptr(proj), _ptr(o),
                              _stream(q.device)), "sa_sla_linear")
    return o


def sa_sla_fwd(q, k, v, classes, sm_scale: float | None = None, phi: int = SA_PHI_SOFTMAX, proj=None, out=None):
    """SLA forward: bf16 [B,H,N,d] = sparse quantised attention over the critical blocks
    (classes >= 2) + the projected linear branch over the marginal blocks (classes == 1)."""
    B, H, N, d = _sla_args(q, k, v, classes, proj)
    scale = 1.0 / math.sqrt(d) if sm_scale is None else float(sm_scale)
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q.device) if out is None else out
    _need(o, torch.bfloat16, "out")
    _check(_lib.sa_sla_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, d, scale, _ptr(classes), int(phi),
                           _ptr(proj), _stream(q.device)), "sa_sla_fwd")
    return o


def sa_debug_qk_s32(q_i8, k_i8, N: int):
    """int32 S [B,H,Npad,Npad] from the tcgen05 INT8 path (small problems only)."""
    _need(q_i8, torch.int8, "q_i8")
    _need(k_i8, torch.int8, "k_i8")
    B, H, Np, d = _dims(q_i8)
    s = torch.empty((B, H, Np, Np), dtype=torch.int32, device=q_i8.device)
    _check(_lib.sa_debug_qk_s32(_ptr(q_i8), _ptr(k_i8), B, H, N, d, _ptr(s),
                                _stream(q_i8.device)), "sa_debug_qk_s32")
    return s


def sa_debug_wait_timeout(timeout_us: int, device=None):
    dev = torch.device("cuda") if device is None else torch.device(device)
    _check(_lib.sa_debug_wait_timeout(int(timeout_us), _stream(dev)), "sa_debug_wait_timeout")


def sa_debug_mma_peak(kind: int, reps: int, device=None):
    """Launches the tensor-core rate kernel on the current stream (kind 0: kind::i8, 1: e4m3
    kind::f8f6f4); the caller times it.  Returns the operations it performs."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    _check(_lib.sa_debug_mma_peak(kind, reps, _stream(dev)), "sa_debug_mma_peak")
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    return float(sms) * reps * 4 * 2 * 128 * 256 * 32


def sa_get_device_status() -> int:
    """Synchronises the current device; returns and clears its device status word."""
    return int(_lib.sa_get_device_status())


def sa_workspace_bytes(B: int, H: int, N: int, d: int = 128) -> int:
    return int(_lib.sa_workspace_bytes(B, H, N, d))


def sa_release_workspace():
    _check(_lib.sa_release_workspace(), "sa_release_workspace")
