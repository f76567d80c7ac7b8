"""The W8A8 linear layer on the GPU against the oracle: codes and block scales bit-exact,
and y bit-exact (the oracle's fp32 accumulator rounded once to bf16, nearest-even), over
ragged shapes that span several 128 x 256 output tiles and k-blocks, and on sampled rows of
the Wan2.1-14B feed-forward shape the benchmark times."""
import numpy as np
import pytest
import torch

from bit_quantized_attention_sa_b200.workloads import (LINEAR_WORKLOADS, f32_to_bf16_bits, make_linear_inputs,
                                                       make_linear_workload)

from _helpers import to_dev_bf16

pytestmark = pytest.mark.gpu


def _bf16(a):
    return f32_to_bf16_bits(np.asarray(a, np.float32))


def _y_bits(y: torch.Tensor) -> np.ndarray:
    return y.cpu().view(torch.int16).numpy().view(np.uint16)


def _dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("rows,cols", [(1, 8), (128, 128), (130, 296), (257, 136), (300, 1000), (4100, 5120)])
def test_quantize_bit_exact(oracle, libsa, cuda_ok, rows, cols):
    x, _ = make_linear_inputs(rows, 8, cols, seed=rows + cols)
    codes, scales = libsa.sa_w8a8_quantize(to_dev_bf16(x))
    rc, rs = oracle.w8a8_quantize(x)
    np.testing.assert_array_equal(scales.cpu().numpy(), rs)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)


def test_quantize_ties_zero_blocks_and_subnormals(oracle, libsa, cuda_ok):
    """Half-integer quotients (scale exactly 1, so x / s = x: ties go to even), an all-zero
    block (scale 0, codes 0) and a block of tiny values."""
    rng = np.random.default_rng(11)
    x = np.zeros((256, 384), np.float32)
    x[:128, :128] = rng.integers(-126, 127, size=(128, 128)) + 0.5
    x[0, 0] = 127.0
    x[128:, 128:256] = rng.standard_normal((128, 128)) * 1e-36
    x[:, 256:] = rng.standard_normal((256, 128)) * 300.0
    xb = _bf16(x)
    codes, scales = libsa.sa_w8a8_quantize(to_dev_bf16(xb))
    rc, rs = oracle.w8a8_quantize(xb)
    assert rs[0, 0] == 1.0 and rs[0, 1] == 0.0
    np.testing.assert_array_equal(scales.cpu().numpy(), rs)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)


@pytest.mark.parametrize("M,N,K", [(1, 8, 8), (128, 256, 128), (200, 136, 300), (129, 264, 1000),
                                   (300, 520, 2048), (1000, 1032, 384), (640, 768, 4096)])
def test_gemm_bit_exact(oracle, libsa, cuda_ok, M, N, K):
    x, w = make_linear_inputs(M, N, K, seed=M * 3 + N + K)
    xq, wq = oracle.w8a8_quantize(x), oracle.w8a8_quantize(w)
    y = libsa.sa_w8a8_gemm(tuple(_dev(a) for a in xq), tuple(_dev(a) for a in wq), K)
    assert libsa.sa_get_device_status() == 0
    ref = oracle.w8a8_gemm_rows(xq, wq, K, range(M))
    np.testing.assert_array_equal(_y_bits(y), _bf16(ref))


@pytest.mark.parametrize("M,N,K", [(300, 264, 1000), (2000, 1280, 640)])
def test_linear_equals_quantize_then_gemm(oracle, libsa, cuda_ok, M, N, K):
    x, w = make_linear_inputs(M, N, K, seed=M + 5 * N + K)
    xd = to_dev_bf16(x)
    wq = libsa.sa_w8a8_quantize(to_dev_bf16(w))
    y1 = libsa.sa_w8a8_linear(xd, wq)
    y2 = libsa.sa_w8a8_gemm(libsa.sa_w8a8_quantize(xd), wq, K)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    rows = [0, 1, 127, 128, M // 2, M - 1]
    ref = oracle.w8a8_gemm_rows(oracle.w8a8_quantize(x), oracle.w8a8_quantize(w), K, rows)
    np.testing.assert_array_equal(_y_bits(y1)[rows], _bf16(ref))


def test_exact_integer_inputs(oracle, libsa, cuda_ok):
    """Integer inputs whose block maxima are 127 have unit scales, so y is the exact integer
    product (every partial sum below 2^24) rounded to bf16."""
    rng = np.random.default_rng(12)
    M, N, K = 256, 512, 640
    x = rng.integers(-127, 128, size=(M, K)).astype(np.float32)
    w = rng.integers(-127, 128, size=(N, K)).astype(np.float32)
    for a in (x, w):
        a[::128, ::128] = 127.0
    y = libsa.sa_w8a8_linear(to_dev_bf16(_bf16(x)), libsa.sa_w8a8_quantize(to_dev_bf16(_bf16(w))))
    exact = (x.astype(np.int64) @ w.astype(np.int64).T).astype(np.float32)
    np.testing.assert_array_equal(_y_bits(y), _bf16(exact))


def test_full_size_ffn_sampled_rows(oracle, libsa, cuda_ok):
    """The Wan2.1-14B feed-forward up-projection at 720p (M = 75600 tokens, K = 5120,
    N = 13824) in the launch configuration the benchmark times; rows sampled from the
    first, last (ragged) and interior row blocks."""
    lw = LINEAR_WORKLOADS["wan14b-720p-ffn-up-m75600-n13824-k5120"]
    x, w = make_linear_workload(lw)
    wq = libsa.sa_w8a8_quantize(to_dev_bf16(w))
    y = libsa.sa_w8a8_linear(to_dev_bf16(x), wq)
    assert libsa.sa_get_device_status() == 0
    rows = [0, 1, 127, 128, 37001, 75519, 75520, 75599]
    ref = oracle.w8a8_gemm_rows(oracle.w8a8_quantize(x), oracle.w8a8_quantize(w), lw.K, rows)
    got = _y_bits(y[rows])
    np.testing.assert_array_equal(got, _bf16(ref))
