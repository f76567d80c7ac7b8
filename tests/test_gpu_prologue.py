"""GPU prologue (sa_quantize_qk, sa_quantize_v) against the oracle, bit for bit: INT8
codes, scales, K means, FP8 V codes and V scales, on the small parity workload, ragged
lengths, and the full-size workloads."""
import numpy as np
import pytest

from bit_quantized_attention_sa_b200.workloads import WORKLOADS, make_inputs, make_workload

from _helpers import to_dev_bf16

pytestmark = pytest.mark.gpu


def check_prologue(oracle, libsa, q, k, v):
    qd, kd, vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    g_q8, g_sq, g_k8, g_sk, g_mean = [t.cpu().numpy() for t in libsa.sa_quantize_qk(qd, kd)]
    g_vt, g_sv = [t.cpu().numpy() for t in libsa.sa_quantize_v(vd)]
    assert libsa.sa_get_device_status() == 0
    r_q8, r_sq, r_k8, r_sk, r_mean, exact = oracle.quantize_qk(q, k)
    r_vt, r_sv = oracle.quantize_v(v)
    if exact:
        assert np.array_equal(g_mean.view(np.uint32), r_mean.view(np.uint32))
    else:  # the fp64 sums were not exact: the summation orders may differ in the last bit
        assert np.abs(g_mean - r_mean).max() <= 1e-6 * max(1.0, np.abs(r_mean).max())
    assert np.array_equal(g_sq.view(np.uint32), r_sq.view(np.uint32))
    assert np.array_equal(g_q8, r_q8)
    # K codes and scales depend on the K mean: on every head whose 128 means equal the
    # oracle's bit for bit they must be identical; a head whose means differ (possible only
    # when the oracle reports an inexact fp64 sum) is counted, not skipped silently
    B, H = q.shape[0], q.shape[1]
    same_mean = np.all(g_mean.reshape(B * H, -1).view(np.uint32) == r_mean.reshape(B * H, -1).view(np.uint32), axis=1)
    g_k8h, r_k8h = g_k8.reshape(B * H, -1), r_k8.reshape(B * H, -1)
    g_skh, r_skh = g_sk.reshape(B * H, -1).view(np.uint32), r_sk.reshape(B * H, -1).view(np.uint32)
    k_mismatch = int(sum(np.count_nonzero(g_k8h[h] != r_k8h[h]) + np.count_nonzero(g_skh[h] != r_skh[h])
                         for h in range(B * H) if same_mean[h]))
    print(f"K mean heads bit-identical: {int(same_mean.sum())}/{B * H}; "
          f"k8/scale_k mismatches on those heads: {k_mismatch}")
    assert k_mismatch == 0
    if exact:
        assert same_mean.all()
    else:  # a differing mean is off by at most one unit in the last place
        d_ulp = np.abs(g_mean.view(np.int32).astype(np.int64) - r_mean.view(np.int32).astype(np.int64))
        assert d_ulp.max() <= 1
    assert np.array_equal(g_sv.view(np.uint32), r_sv.view(np.uint32))
    assert np.array_equal(g_vt, r_vt)
    return exact


@pytest.mark.parametrize("B,H,N", [(1, 2, 1024), (1, 1, 1), (1, 1, 63), (2, 3, 65),
                                   (1, 2, 129), (1, 1, 200), (1, 2, 1030), (1, 1, 4097)])
def test_prologue_bit_exact_small(oracle, libsa, cuda_ok, B, H, N):
    q, k, v, _ = make_inputs(B, H, N, seed=100 + N, outliers=(N % 2 == 1))
    assert check_prologue(oracle, libsa, q, k, v)


def test_prologue_zero_and_constant_blocks(oracle, libsa, cuda_ok):
    """All-zero Q/K blocks and V channels give scale 0 and zero codes; identical key rows
    give an exactly zero smoothed K."""
    from bit_quantized_attention_sa_b200.workloads import f32_to_bf16_bits
    rng = np.random.default_rng(3)
    x = rng.standard_normal((1, 1, 300, 128)).astype(np.float32)
    q = x.copy()
    q[0, 0, :128] = 0.0
    k = np.broadcast_to(x[:, :, :1], x.shape).copy()
    v = x.copy()
    v[..., 5] = 0.0
    check_prologue(oracle, libsa, f32_to_bf16_bits(q), f32_to_bf16_bits(k), f32_to_bf16_bits(v))


@pytest.mark.parametrize("name", ["wan1.3b-480p-h12-n32760", "wan14b-720p-h40-n75600"])
def test_prologue_bit_exact_full_size(oracle, libsa, cuda_ok, name):
    q, k, v, _ = make_workload(WORKLOADS[name])
    check_prologue(oracle, libsa, q, k, v)
