"""The d = 64 definition equals the d = 128 definition on inputs whose upper 64 channels
are zero, bit for bit, in the oracle: zero channels add nothing to S, leave every block
maximum (scales and codes) unchanged, have K mean 0 and V scale 0.  This is the identity the
GPU's d = 64 calls rely on (they run the d = 128 kernels on zero-padded copies)."""
import math

import numpy as np
import pytest

from bit_quantized_attention_sa_b200.workloads import make_inputs


def _pad(x):
    out = np.zeros(x.shape[:-1] + (128,), np.uint16)
    out[..., :64] = x
    return out


@pytest.mark.parametrize("N,causal", [(1, False), (200, False), (700, True), (1000, False)])
def test_d64_equals_zero_padded_d128(oracle, N, causal):
    q, k, v, _ = make_inputs(1, 2, N, d=64, seed=170 + N, outliers=True)
    rows = [(bh, r) for bh in range(2) for r in sorted({0, N // 3, N - 1})]
    scale = 1.0 / math.sqrt(64)
    o64 = oracle.attn_rows(oracle.quantize_qk(q, k), oracle.quantize_v(v), N, scale, rows, None, 2, causal=causal)
    qp, kp, vp = _pad(q), _pad(k), _pad(v)
    o128 = oracle.attn_rows(oracle.quantize_qk(qp, kp), oracle.quantize_v(vp), N, scale, rows, None, 2,
                            causal=causal)
    np.testing.assert_array_equal(o128[:, :64], o64)
    assert not o128[:, 64:].any()
