"""The C ABI without a GPU: the library loads, exports every entry point include/sa.h
declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    text = open(os.path.join(ROOT, "include", "sa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sa_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(libsa):
    names = declared_entry_points()
    assert len(names) >= 10
    lib = libsa.raw_library()
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_sizes(libsa):
    assert libsa.sa_status_string(0) == "SA_OK"
    assert libsa.sa_status_string(6) == "SA_ERR_DEVICE_TIMEOUT"
    assert [libsa.padded_len(n) for n in (0, 1, 128, 129, 75600)] == [0, 128, 128, 256, 75648]
    assert libsa.sa_workspace_bytes(1, 2, 1024, 96) == 0
    # d = 64: the d = 128 workspace plus four zero-padded 128-channel copies
    assert libsa.sa_workspace_bytes(1, 2, 1024, 64) >= libsa.sa_workspace_bytes(1, 2, 1024, 128) + 4 * 2 * 1024 * 128 * 2
    assert libsa.sa_workspace_bytes(1, 2, 0, 128) == 0
    ws = libsa.sa_workspace_bytes(1, 40, 75600, 128)
    assert 3 * 40 * 75648 * 128 <= ws < 3 * 40 * 75648 * 128 + (1 << 24)


FAKE = ctypes.c_void_p(1 << 20)       # 16-byte aligned, never dereferenced
ODD = ctypes.c_void_p((1 << 20) + 8)  # misaligned


@pytest.mark.parametrize("args,expect", [
    ((None, FAKE, FAKE, FAKE, 1, 1, 128, 128, 0.088, None, None), 1),   # null q
    ((FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 96, 0.088, None, None), 2),    # d not 64 or 128
    ((FAKE, FAKE, FAKE, ODD, 1, 1, 128, 128, 0.088, None, None), 3),    # misaligned o
    ((FAKE, FAKE, FAKE, FAKE, 1, 1, 0, 128, 0.088, None, None), 1),     # N = 0
    ((FAKE, FAKE, FAKE, FAKE, 0, 1, 128, 128, 0.088, None, None), 1),   # B = 0
    ((FAKE, FAKE, FAKE, FAKE, 1 << 20, 1 << 10, 128, 128, 0.088, None, None), 1),  # overflow
    ((FAKE, FAKE, FAKE, FAKE, 2, 32768, 128, 128, 0.088, None, None), 2),  # B*H > 65535
    ((FAKE, FAKE, FAKE, FAKE, 1, 1, 64 * 16385, 128, 0.088, FAKE, None), 2),  # mask rows > 16384 blocks
    ((FAKE, FAKE, FAKE, FAKE, 1, 1, 64 * 16385, 64, 0.088, FAKE, None), 2),   # the same at d = 64
    ((FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 128, 0.0, None, None), 1),     # sm_scale <= 0
    ((FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 128, float("nan"), None, None), 1),
])
def test_attn_fwd_argument_errors(libsa, args, expect):
    assert libsa.raw_library().sa_attn_fwd(*args) == expect
    # the host-buffer entry point validates the same way before touching CUDA
    assert libsa.raw_library().sa_attn_fwd_host(*args) == expect


def test_other_entry_points_argument_errors(libsa):
    lib = libsa.raw_library()
    assert lib.sa_quantize_qk(FAKE, None, 1, 1, 128, 128, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert lib.sa_quantize_qk(FAKE, FAKE, 1, 1, 128, 96, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 2
    assert lib.sa_quantize_v(FAKE, 1, 1, 128, 128, ODD, FAKE, None) == 3
    assert lib.sa_attn_fwd_quantized(FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, 1, 1, 128, 128,
                                     ctypes.c_float(0.088), None, None) == 1
    assert lib.sa_debug_qk_s32(FAKE, FAKE, 1, 1, -5, 128, FAKE, None) == 1
    assert lib.sa_debug_wait_timeout(0, None) == 1
    # the selector: keep_per_row >= 1; at most 4096 key blocks per row
    assert lib.sa_block_mask(FAKE, FAKE, 1, 1, 128, 128, 0, 0, FAKE, None) == 1
    assert lib.sa_block_mask(FAKE, FAKE, 1, 1, 128, 128, 1, 0, None, None) == 1
    assert lib.sa_block_mask(FAKE, FAKE, 1, 1, 4096 * 64 + 1, 128, 1, 0, FAKE, None) == 2
    assert lib.sa_debug_pool(FAKE, FAKE, 1, 1, 128, 128, ODD, FAKE, None) == 3


def test_w8a8_argument_errors(libsa):
    lib = libsa.raw_library()
    # quantiser: sizes >= 1, cols a multiple of 8, aligned pointers
    assert lib.sa_w8a8_quantize(FAKE, 0, 128, FAKE, FAKE, None) == 1
    assert lib.sa_w8a8_quantize(FAKE, 128, 100, FAKE, FAKE, None) == 2
    assert lib.sa_w8a8_quantize(FAKE, 128, 128, ODD, FAKE, None) == 3
    assert lib.sa_w8a8_quantize(None, 128, 128, FAKE, FAKE, None) == 1
    # GEMM: M, N, K >= 1; N a multiple of 8 (K is free: the codes are padded to 128)
    assert lib.sa_w8a8_gemm(FAKE, FAKE, FAKE, FAKE, 128, 0, 128, FAKE, None) == 1
    assert lib.sa_w8a8_gemm(FAKE, FAKE, FAKE, FAKE, 128, 100, 128, FAKE, None) == 2
    assert lib.sa_w8a8_gemm(FAKE, FAKE, FAKE, None, 128, 128, 128, FAKE, None) == 1
    assert lib.sa_w8a8_gemm(FAKE, FAKE, FAKE, FAKE, 128, 128, 128, ODD, None) == 3
    assert lib.sa_w8a8_linear(FAKE, FAKE, FAKE, -1, 128, 128, FAKE, None) == 1
    assert lib.sa_w8a8_linear(FAKE, FAKE, FAKE, 128, 12, 128, FAKE, None) == 2
    assert lib.sa_w8a8_linear(FAKE, FAKE, FAKE, 128, 128, 100, FAKE, None) == 2
    assert lib.sa_w8a8_linear(ODD, FAKE, FAKE, 128, 128, 128, FAKE, None) == 3


def test_sla_argument_errors(libsa):
    lib = libsa.raw_library()
    f = ctypes.c_float(0.088)
    # phi must be 0 or 1; classes required; at most 4096 key blocks; d = 128; aligned
    assert lib.sa_sla_linear(FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 128, 2, None, FAKE, None) == 1
    assert lib.sa_sla_linear(FAKE, FAKE, FAKE, None, 1, 1, 128, 128, 0, None, FAKE, None) == 1
    assert lib.sa_sla_linear(FAKE, FAKE, FAKE, FAKE, 1, 1, 4096 * 64 + 1, 128, 0, None, FAKE, None) == 2
    assert lib.sa_sla_linear(FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0, None, FAKE, None) == 2
    assert lib.sa_sla_linear(FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 128, 0, ODD, FAKE, None) == 3
    assert lib.sa_sla_fwd(FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 128, ctypes.c_float(0.0), FAKE, 0, None, None) == 1
    assert lib.sa_sla_fwd(FAKE, FAKE, FAKE, ODD, 1, 1, 128, 128, f, FAKE, 1, None, None) == 3
    assert lib.sa_sla_fwd(FAKE, FAKE, FAKE, FAKE, 1, 1, 0, 128, f, FAKE, 1, None, None) == 1


def test_causal_argument_errors(libsa):
    lib = libsa.raw_library()
    f = ctypes.c_float(0.088)
    assert lib.sa_attn_fwd_causal(None, FAKE, FAKE, FAKE, 1, 1, 128, 128, f, None, None) == 1
    assert lib.sa_attn_fwd_causal(FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 96, f, None, None) == 2
    # d = 64 is accepted by the forward calls (zero-padded to 128) but not by the others
    assert lib.sa_attn_fwd_causal(FAKE, FAKE, FAKE, ODD, 1, 1, 128, 64, f, None, None) == 3
    assert lib.sa_attn_fwd(FAKE, FAKE, FAKE, ODD, 1, 1, 128, 64, f, None, None) == 3
    assert lib.sa_attn_fwd(FAKE, FAKE, FAKE, FAKE, 0, 1, 128, 64, f, None, None) == 1
    assert lib.sa_quantize_qk(FAKE, FAKE, 1, 1, 128, 64, FAKE, FAKE, FAKE, FAKE, FAKE, None) == 2
    assert lib.sa_attn_fwd_causal(FAKE, FAKE, FAKE, ODD, 1, 1, 128, 128, f, None, None) == 3
    assert lib.sa_attn_fwd_causal(FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 128, ctypes.c_float(-1.0), None, None) == 1


def test_varlen_argument_errors(libsa):
    lib = libsa.raw_library()
    f = ctypes.c_float(0.088)
    lens = (ctypes.c_int * 3)(100, 0, 50)
    ok = (ctypes.c_int * 2)(100, 50)
    assert lib.sa_attn_fwd_varlen(FAKE, FAKE, FAKE, FAKE, 0, ok, 2, 128, f, 0, None) == 1
    assert lib.sa_attn_fwd_varlen(FAKE, FAKE, FAKE, FAKE, 2, None, 2, 128, f, 0, None) == 1
    assert lib.sa_attn_fwd_varlen(FAKE, FAKE, FAKE, FAKE, 3, lens, 2, 128, f, 0, None) == 1   # N = 0
    assert lib.sa_attn_fwd_varlen(FAKE, FAKE, FAKE, FAKE, 2, ok, 2, 64, f, 0, None) == 2
    assert lib.sa_attn_fwd_varlen(FAKE, FAKE, FAKE, ODD, 2, ok, 2, 128, f, 1, None) == 3
