"""Pins of the causal mode of the oracle: the last row equals the non-causal row bit for
bit, the first row is its own dequantised value, keys after a row do not reach the exact
fp64 causal reference, the exact reference against an independent numpy causal softmax,
and the quantised causal rows against the exact causal ones."""
import math

import numpy as np
import pytest

from bit_quantized_attention_sa_b200.workloads import bf16_bits_to_f32, make_inputs


def _scale():
    return 1.0 / math.sqrt(128)


@pytest.mark.parametrize("N", [1, 64, 65, 200, 1000])
def test_last_row_equals_non_causal(oracle, N):
    q, k, v, _ = make_inputs(1, 2, N, seed=130 + N, outliers=True)
    qk, vq = oracle.quantize_qk(q, k), oracle.quantize_v(v)
    rows = [(bh, N - 1) for bh in range(2)]
    np.testing.assert_array_equal(oracle.attn_rows(qk, vq, N, _scale(), rows, causal=True),
                                  oracle.attn_rows(qk, vq, N, _scale(), rows))


def test_first_row_is_its_dequantised_value(oracle):
    N = 300
    q, k, v, _ = make_inputs(1, 1, N, seed=131, outliers=True)
    qk, vq = oracle.quantize_qk(q, k), oracle.quantize_v(v)
    got = oracle.attn_rows(qk, vq, N, _scale(), [(0, 0)], causal=True)[0]
    v_t, sv = vq
    deq = np.array([oracle.e4m3_to_f32(int(v_t[0, 0, c, 0])) for c in range(128)], np.float32) * sv[0, 0]
    # one key: p8 = 448, l = 448, O = 448 * v8 * sv / 448
    np.testing.assert_allclose(got, deq, rtol=2e-7, atol=0)


def _numpy_causal(q, k, v, rows):
    qf, kf, vf = (bf16_bits_to_f32(a).astype(np.float64) for a in (q, k, v))
    out = []
    for bh, r in rows:
        s = kf[0, bh, : r + 1] @ qf[0, bh, r] * _scale()
        p = np.exp(s - s.max())
        out.append(p @ vf[0, bh, : r + 1] / p.sum())
    return np.array(out)


def test_exact_causal_against_numpy_and_future_invariance(oracle):
    N = 500
    q, k, v, _ = make_inputs(1, 2, N, seed=132)
    rows = [(bh, r) for bh in range(2) for r in (0, 1, 63, 64, 127, 128, 300, 499)]
    got = oracle.exact_rows(q, k, v, _scale(), rows, causal=True)
    np.testing.assert_allclose(got, _numpy_causal(q, k, v, rows), rtol=1e-12, atol=1e-12)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 301:], v2[:, :, 301:] = k[:, :, :199], v[:, :, :199]
    past = [(bh, r) for bh, r in rows if r <= 300]
    np.testing.assert_array_equal(oracle.exact_rows(q, k2, v2, _scale(), past, causal=True),
                                  oracle.exact_rows(q, k, v, _scale(), past, causal=True))


@pytest.mark.parametrize("N", [2, 63, 129, 700])
def test_quantised_causal_close_to_exact_causal(oracle, N):
    q, k, v, _ = make_inputs(1, 2, N, seed=133 + N)
    qk, vq = oracle.quantize_qk(q, k), oracle.quantize_v(v)
    rows = [(bh, r) for bh in range(2) for r in sorted({0, 1, N // 2, N - 1})]
    got = oracle.attn_rows(qk, vq, N, _scale(), rows, causal=True).astype(np.float64)
    ref = oracle.exact_rows(q, k, v, _scale(), rows, causal=True)
    vf = np.abs(bf16_bits_to_f32(v)).astype(np.float64)
    for n, (bh, r) in enumerate(rows):
        # a row with few keys keeps the FP8 rounding of V (half an e4m3 step, 2^-4 relative)
        # undiluted; the softmax weights' own FP8 rounding adds a little on top
        bound = 0.0625 * vf[0, bh, : r + 1].max() + 0.02
        assert np.abs(got[n] - ref[n]).max() <= bound, (r, np.abs(got[n] - ref[n]).max(), bound)
    cos = (got * ref).sum() / np.linalg.norm(got) / np.linalg.norm(ref)
    assert cos > 0.999
