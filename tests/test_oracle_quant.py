"""Pins for the oracle's quantisation prologue: Q INT8 per 128-token block, K smoothed by
its per-channel mean then INT8 per 64-token block, V FP8 e4m3 per channel (transposed).

Each pin would fail on a plausible slip: a wrong block size, a missing smoothing step,
truncation instead of round-half-even, a /128 or /255 scale, a transposed V layout,
scales taken over padded rows.
"""
from fractions import Fraction

import numpy as np

from bit_quantized_attention_sa_b200.workloads import (bf16_bits_to_f32, f32_to_bf16_bits,
                                                       make_inputs)


def bf(x):
    return f32_to_bf16_bits(np.asarray(x, np.float32))


def test_exact_integer_case(oracle):
    """Integer Q/K in [-127,127] whose every block reaches +-127 and whose K channel means
    are 0 quantise to themselves with unit scales."""
    rng = np.random.default_rng(0)
    B, H, N, d = 1, 2, 256, 128
    q = rng.integers(-127, 128, (B, H, N, d)).astype(np.float32)
    q[:, :, ::128, 0] = 127.0
    half = rng.integers(-126, 127, (B, H, N // 2, d)).astype(np.float32)
    half[:, :, ::64, 1] = 127.0                         # every 64-token block reaches 127
    k = np.concatenate([half, -half], axis=2)           # channel sums are exactly 0
    assert np.all(k.sum(axis=2) == 0)
    q_i8, sq, k_i8, sk, mean, exact = oracle.quantize_qk(bf(q), bf(k))
    assert exact
    assert np.all(mean == 0.0)
    assert np.all(sq == 1.0) and np.all(sk == 1.0)
    assert np.array_equal(q_i8[:, :, :N].astype(np.float32), q)
    assert np.array_equal(k_i8[:, :, :N].astype(np.float32), k)


def test_round_half_even_ties(oracle):
    """With scale 1 (block amax 127), halves round to the even integer."""
    N, d = 128, 128
    q = np.zeros((1, 1, N, d), np.float32)
    q[0, 0, 0, 0] = 127.0
    ties = [0.5, 1.5, 2.5, 3.5, -0.5, -1.5, -2.5, 126.5, -126.5]
    expect = [0, 2, 2, 4, 0, -2, -2, 126, -126]
    q[0, 0, 1, :len(ties)] = ties
    k = np.zeros_like(q)
    q_i8, sq, *_ = oracle.quantize_qk(bf(q), bf(k))
    assert sq[0, 0, 0] == 1.0
    assert q_i8[0, 0, 1, :len(ties)].tolist() == expect


def test_scale_and_rounding_bound(oracle):
    """scale = amax/127 per block; every code within half a step of x/scale (plus the
    fp32 rounding of the quotient, at most 128 * 2^-24 of a step); the block-max element
    maps to +-127; codes never leave [-127, 127]."""
    q, k, _, _ = make_inputs(1, 2, 1000, seed=11, outliers=True)
    q_i8, sq, k_i8, sk, mean, _ = oracle.quantize_qk(q, k)
    qf = bf16_bits_to_f32(q)
    N = 1000
    for bh in range(2):
        b, h = divmod(bh, 2)
        for i in range(sq.shape[2]):
            blk = qf[b, h, 128 * i:min(N, 128 * i + 128)]
            amax = np.abs(blk).max()
            assert sq[b, h, i] == np.float32(amax) / np.float32(127.0)
            codes = q_i8[b, h, 128 * i:min(N, 128 * i + 128)].astype(np.float64)
            err = np.abs(blk.astype(np.float64) - codes * float(sq[b, h, i]))
            assert err.max() <= (0.5 + 128 * 2.0 ** -23) * float(sq[b, h, i])
            assert np.abs(codes).max() == 127
        ks = bf16_bits_to_f32(k)[b, h] - mean[b, h][None, :]
        for j in range(sk.shape[2]):
            blk = ks[64 * j:min(N, 64 * j + 64)]
            assert sk[b, h, j] == np.float32(np.abs(blk).max()) / np.float32(127.0)
            codes = k_i8[b, h, 64 * j:min(N, 64 * j + 64)].astype(np.float64)
            err = np.abs(blk.astype(np.float64) - codes * float(sk[b, h, j]))
            assert err.max() <= (0.5 + 128 * 2.0 ** -23) * float(sk[b, h, j])
    assert np.all(q_i8[:, :, N:] == 0) and np.all(k_i8[:, :, N:] == 0)


def test_block_boundaries(oracle):
    """A spike at token 128 changes only Q block 1; a +/- pair at tokens 64/65 (mean
    unchanged) changes only K block 1."""
    q, k, _, _ = make_inputs(1, 1, 384, seed=5)
    kb = bf16_bits_to_f32(k).copy()
    kb[0, 0, 64, 7], kb[0, 0, 65, 7] = 1.0, -1.0
    base = oracle.quantize_qk(q, bf(kb))
    q2 = bf16_bits_to_f32(q).copy()
    q2[0, 0, 128, 3] = 64.0
    k2 = kb.copy()
    k2[0, 0, 64, 7], k2[0, 0, 65, 7] = 64.0, -64.0       # same channel sum
    pert = oracle.quantize_qk(bf(q2), bf(k2))
    dq = base[1] != pert[1]
    assert dq.tolist() == [[[False, True, False]]]
    dk = base[3] != pert[3]
    assert dk[0, 0].tolist() == [False, True, False, False, False, False]
    assert np.array_equal(base[4], pert[4])  # means unchanged (exact fp64 sums)


def test_smoothing_shift_invariance(oracle):
    """Adding the same vector delta to every key row leaves the smoothed K, hence k_i8
    and scale_k, bit-identical (inputs chosen so every mean is exact)."""
    rng = np.random.default_rng(9)
    N, d = 256, 128                                      # N a power of two: exact means
    k = rng.integers(-40, 41, (1, 1, N, d)).astype(np.float32) / 4.0
    delta = rng.integers(-24, 25, (1, 1, 1, d)).astype(np.float32)
    q = np.ones_like(k)
    a = oracle.quantize_qk(bf(q), bf(k))
    b = oracle.quantize_qk(bf(q), bf(k + delta))
    assert a[5] and b[5]
    assert np.array_equal(a[2], b[2]) and np.array_equal(a[3], b[3])
    assert np.array_equal(b[4][0, 0] - a[4][0, 0], delta[0, 0, 0])


def test_mean_is_the_exact_mean(oracle):
    """For bf16 inputs of moderate range the fp64 sums are exact, so the mean is the
    exact rational mean rounded to fp32 (computed here with Python integers)."""
    q, k, _, _ = make_inputs(1, 2, 777, seed=21)
    _, _, _, _, mean, exact = oracle.quantize_qk(q, k)
    assert exact
    kf = bf16_bits_to_f32(k).astype(np.float64)
    # every bf16 value is an integer multiple of 2^-133; sum those integers exactly
    scale = 2.0 ** 133
    for h in range(2):
        for c in range(0, 128, 17):
            ints = [int(x * scale) for x in kf[0, h, :, c]]
            total = sum(ints)
            m = Fraction(total, 777) / Fraction(2 ** 133)
            assert mean[0, h, c] == np.float32(float(m))


def test_v_scale_codes_and_layout(oracle):
    """Per-channel scale amax/448; the channel max maps to +-448 (0x7E/0xFE); V is stored
    channel-major (transposed) with zero padding; a single non-zero element lands at
    [c, t]."""
    v = np.zeros((1, 1, 200, 128), np.float32)
    v[0, 0, 37, 5] = -3.0
    vt, sv = oracle.quantize_v(bf(v))
    assert vt.shape == (1, 1, 128, 256)
    assert sv[0, 0, 5] == np.float32(3.0) / np.float32(448.0)
    nz = np.argwhere(vt != 0)
    assert nz.tolist() == [[0, 0, 5, 37]] and vt[0, 0, 5, 37] == 0xFE
    _, _, vr, _ = make_inputs(1, 1, 300, seed=2)
    vt, sv = oracle.quantize_v(vr)
    vf = bf16_bits_to_f32(vr)[0, 0]
    dec = np.array([oracle.e4m3_to_f32(c) for c in range(256)], np.float32)
    deq = dec[vt[0, 0, :, :300]].T * sv[0, 0][None, :]
    rel = np.abs(deq - vf) / np.maximum(np.abs(vf), 1e-30)
    normal = np.abs(vf) / sv[0, 0][None, :] >= 2.0 ** -6
    assert rel[normal].max() <= 2.0 ** -4 * (1 + 1e-6)       # half an e4m3 ulp
    amax_idx = np.abs(vf).argmax(axis=0)
    assert np.all((vt[0, 0, np.arange(128), amax_idx] & 0x7F) == 0x7E)
    assert np.all(vt[0, 0, :, 300:] == 0)


def test_zero_blocks(oracle):
    q = np.zeros((1, 1, 130, 128), np.float32)
    q[0, 0, 129, 0] = 1.0
    k = np.zeros_like(q)
    v = np.zeros_like(q)
    q_i8, sq, k_i8, sk, mean, _ = oracle.quantize_qk(bf(q), bf(k))
    assert sq[0, 0, 0] == 0 and np.all(q_i8[0, 0, :128] == 0)
    assert np.all(sk == 0) and np.all(k_i8 == 0)
    vt, sv = oracle.quantize_v(bf(v))
    assert np.all(sv == 0) and np.all(vt == 0)
