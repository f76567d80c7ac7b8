"""The block-mask producer on the GPU against the oracle: block means and masks bit-exact
(integer output: any difference is a bug), at small and full sizes, and the sparse
attention driven by the produced mask against the oracle's attention with the oracle's
mask."""
import numpy as np
import pytest
import torch

from bit_quantized_attention_sa_b200.workloads import WORKLOADS, make_inputs, make_workload

from _helpers import O_MAX_ABS, O_MIN_COS, cosine, gpu_rows, sm_scale, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N", [1, 63, 64, 65, 129, 1000, 3000])
def test_pool_bit_exact(oracle, libsa, cuda_ok, N):
    q, k, _, _ = make_inputs(1, 3, N, seed=60 + N, outliers=True)
    qb, kb = libsa.sa_debug_pool(to_dev_bf16(q), to_dev_bf16(k))
    rq, _ = oracle.pool(q, 128)
    rk, _ = oracle.pool(k, 64)
    np.testing.assert_array_equal(qb.cpu().numpy(), rq)
    np.testing.assert_array_equal(kb.cpu().numpy(), rk)


@pytest.mark.parametrize("B,H,N,keep,diag", [(1, 1, 1, 1, False), (1, 2, 65, 1, True), (1, 2, 1000, 3, False),
                                              (2, 1, 3000, 5, True), (1, 2, 2048, 32, False),
                                              (1, 1, 1500, 100, True), (1, 3, 5000, 8, False)])
def test_block_mask_bit_exact(oracle, libsa, cuda_ok, B, H, N, keep, diag):
    q, k, _, _ = make_inputs(B, H, N, seed=70 + N + keep, outliers=True)
    got = libsa.sa_block_mask(to_dev_bf16(q), to_dev_bf16(k), keep, diag).cpu().numpy()
    ref = oracle.block_mask(q, k, keep, diag)[0]
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("name,heads,keep", [("wan14b-480p-h40-n32760", 3, 51), ("wan14b-720p-h40-n75600", 2, 118)])
def test_block_mask_full_size_heads(oracle, libsa, cuda_ok, name, heads, keep):
    w = WORKLOADS[name]
    q, k, _, _ = make_workload(w)
    q, k = np.ascontiguousarray(q[:, :heads]), np.ascontiguousarray(k[:, :heads])
    got = libsa.sa_block_mask(to_dev_bf16(q), to_dev_bf16(k), keep, True).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.block_mask(q, k, keep, True)[0])


def test_block_mask_largest_row(oracle, libsa, cuda_ok):
    """4096 key blocks per row (N = 262144), the selector's limit; rows checked on a sample
    (the oracle's rank rule is quadratic in the row length)."""
    N = 4096 * 64
    q, k, _, _ = make_inputs(1, 1, N, seed=81, outliers=False)
    got = libsa.sa_block_mask(to_dev_bf16(q), to_dev_bf16(k), 300, False).cpu().numpy()
    qbar, _ = oracle.pool(q, 128)
    kbar, _ = oracle.pool(k, 64)
    rows = [0, 1, 777, 2047]
    ref = oracle.mask_from_scores(oracle.block_scores(np.ascontiguousarray(qbar[:, :, rows]), kbar), 300)
    np.testing.assert_array_equal(got[:, :, rows], ref)
    assert (got.sum(axis=-1) == 300).all()


def test_sparse_attention_with_produced_mask(oracle, libsa, cuda_ok):
    q, k, v, _ = make_inputs(1, 2, 4000, seed=82, outliers=True)
    qd, kd, vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    m = libsa.sa_block_mask(qd, kd, 9, True)
    o = libsa.sa_attn_fwd(qd, kd, vd, block_mask=m)
    assert libsa.sa_get_device_status() == 0
    ref_mask = oracle.block_mask(q, k, 9, True)[0]
    np.testing.assert_array_equal(m.cpu().numpy(), ref_mask)
    rows = [(bh, r) for bh in range(2) for r in range(0, 4000, 37)]
    ref = oracle.attn_rows(oracle.quantize_qk(q, k), oracle.quantize_v(v), 4000, sm_scale(), rows, ref_mask, 2)
    got = gpu_rows(o, rows)
    assert np.abs(got - ref).max() <= O_MAX_ABS
    assert cosine(got, ref) >= O_MIN_COS


def test_block_mask_exact_ties_go_to_lower_index(oracle, libsa, cuda_ok):
    """Copies of one 64-token key block score identically: the GPU's radix selection must
    break those ties by block index exactly like the oracle's rank rule."""
    q, k, _, _ = make_inputs(1, 2, 3000, seed=83, outliers=False)
    k = k.copy()
    src = k[:, :, 5 * 64:6 * 64].copy()
    for j in (9, 17, 30, 41, 44):
        k[:, :, j * 64:(j + 1) * 64] = src
    for keep in (1, 3, 4, 6, 20):
        got = libsa.sa_block_mask(to_dev_bf16(q), to_dev_bf16(k), keep, False).cpu().numpy()
        ref, _, _, scores, _ = oracle.block_mask(q, k, keep, False)
        assert (scores[..., 9] == scores[..., 5]).all()
        np.testing.assert_array_equal(got, ref)
