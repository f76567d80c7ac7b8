"""Pins of the W8A8 linear layer in the oracle (INT8 weights and activations, one scale per
128 x 128 block): the quantiser against an independent numpy restatement, the exact-integer
closed form, the single-k-block closed form, zero blocks, and the quantisation error
against the fp64 product."""
import numpy as np
import pytest

from bit_quantized_attention_sa_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits


def _bf16(a):
    return f32_to_bf16_bits(np.asarray(a, np.float32))


def _numpy_quantize(x_bits):
    x = bf16_bits_to_f32(x_bits)
    rows, cols = x.shape
    rb, cb = -(-rows // 128), -(-cols // 128)
    codes = np.zeros((rows, cb * 128), np.int8)
    scales = np.zeros((rb, cb), np.float32)
    for a in range(rb):
        for b in range(cb):
            blk = x[a * 128:(a + 1) * 128, b * 128:(b + 1) * 128]
            s = np.float32(np.abs(blk).max()) / np.float32(127.0)
            scales[a, b] = s
            c = np.zeros(blk.shape) if s == 0 else np.clip(np.rint(blk / s), -127, 127)
            codes[a * 128:a * 128 + blk.shape[0], b * 128:b * 128 + blk.shape[1]] = c
    return codes, scales


@pytest.mark.parametrize("rows,cols", [(1, 1), (128, 128), (130, 300), (257, 129), (64, 512)])
def test_quantizer_matches_numpy(oracle, rows, cols):
    rng = np.random.default_rng(rows * 7 + cols)
    x = _bf16(rng.standard_normal((rows, cols)) * rng.choice([0.01, 1.0, 30.0], size=(rows, 1)))
    codes, scales = oracle.w8a8_quantize(x)
    rc, rs = _numpy_quantize(x)
    np.testing.assert_array_equal(scales, rs)
    np.testing.assert_array_equal(codes, rc)


def _integer_blocks(rng, rows, cols):
    x = rng.integers(-127, 128, size=(rows, cols)).astype(np.float32)
    for a in range(0, rows, 128):
        for b in range(0, cols, 128):
            x[a, b] = 127.0  # every block's max |x| is 127, so its scale is exactly 1
    return x


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (200, 130, 300), (129, 257, 1000)])
def test_exact_integer_case(oracle, M, N, K):
    rng = np.random.default_rng(M + N + K)
    x, w = _integer_blocks(rng, M, K), _integer_blocks(rng, N, K)
    xq, wq = oracle.w8a8_quantize(_bf16(x)), oracle.w8a8_quantize(_bf16(w))
    assert (xq[1] == 1.0).all() and (wq[1] == 1.0).all()
    rows = list(range(M))
    y = oracle.w8a8_gemm_rows(xq, wq, K, rows)
    exact = x.astype(np.int64) @ w.astype(np.int64).T
    assert np.abs(exact).max() < 2 ** 24  # every partial sum is exact in fp32
    np.testing.assert_array_equal(y, exact.astype(np.float32))


def test_single_k_block_is_one_rounding(oracle):
    rng = np.random.default_rng(5)
    x, w = _bf16(rng.standard_normal((150, 100))), _bf16(rng.standard_normal((140, 100)))
    (x8, sx), (w8, sw) = oracle.w8a8_quantize(x), oracle.w8a8_quantize(w)
    y = oracle.w8a8_gemm_rows((x8, sx), (w8, sw), 100, list(range(150)))
    S = x8.astype(np.int64) @ w8.astype(np.int64).T
    s = (sx[np.arange(150) // 128, 0][:, None] * sw[np.arange(140) // 128, 0][None, :]).astype(np.float32)
    np.testing.assert_array_equal(y, S.astype(np.float32) * s)


def test_zero_blocks_contribute_nothing(oracle):
    rng = np.random.default_rng(6)
    x = rng.standard_normal((128, 384)).astype(np.float32)
    x[:, 128:256] = 0.0
    w = rng.standard_normal((128, 384)).astype(np.float32)
    xq, wq = oracle.w8a8_quantize(_bf16(x)), oracle.w8a8_quantize(_bf16(w))
    assert xq[1][0, 1] == 0.0 and not xq[0][:, 128:256].any()
    x2 = x.copy()
    x2[:, 128:256] = 0.0
    w2 = w.copy()
    w2[:, 128:256] = rng.standard_normal((128, 128))  # changes nothing the zero block meets
    y1 = oracle.w8a8_gemm_rows(xq, wq, 384, range(128))
    y2 = oracle.w8a8_gemm_rows(xq, oracle.w8a8_quantize(_bf16(w2)), 384, range(128))
    np.testing.assert_array_equal(y1, y2)


def test_error_against_fp64_product(oracle):
    rng = np.random.default_rng(7)
    x = _bf16(rng.standard_normal((256, 1024)))
    w = _bf16(rng.standard_normal((256, 1024)) * 0.05)
    y = oracle.w8a8_gemm_rows(oracle.w8a8_quantize(x), oracle.w8a8_quantize(w), 1024, range(256))
    ref = bf16_bits_to_f32(x).astype(np.float64) @ bf16_bits_to_f32(w).astype(np.float64).T
    # each code is off by at most half a step (scale/2): the product error is bounded by
    # sum over k of (|x| sw/2 + |w| sx/2 + sx sw/4); random signs make it far smaller
    cos = float((y.astype(np.float64) * ref).sum() / np.linalg.norm(y) / np.linalg.norm(ref))
    assert cos > 0.9995
    assert np.abs(y - ref).max() < 0.05 * np.abs(ref).max()
