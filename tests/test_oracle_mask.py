"""Pins of the block-mask producer in the oracle (the selector ahead of the block skip):
block means against numpy, pooled scores against an fp64 einsum, the selection rule against
an independent stable sort, and invariants and closed forms of the whole selector."""
import numpy as np
import pytest

from bit_quantized_attention_sa_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits, make_inputs


def _numpy_block_means(x_bits, blk):
    x = bf16_bits_to_f32(x_bits).astype(np.float64)
    B, H, N, d = x.shape
    nb = -(-N // blk)
    out = np.empty((B, H, nb, d), np.float32)
    for b in range(nb):
        out[:, :, b] = (x[:, :, b * blk:min(N, (b + 1) * blk)].mean(axis=2)).astype(np.float32)
    return out


@pytest.mark.parametrize("N", [1, 63, 64, 65, 127, 128, 129, 1000])
def test_pool_matches_numpy_means(oracle, N):
    q, k, _, _ = make_inputs(1, 2, N, seed=40 + N, outliers=True)
    for x, blk in ((q, 128), (k, 64)):
        got, exact = oracle.pool(x, blk)
        assert exact  # bf16 sums of up to 128 values fit fp64 exactly here
        np.testing.assert_array_equal(got, _numpy_block_means(x, blk))


def test_scores_match_fp64_einsum(oracle):
    q, k, _, _ = make_inputs(2, 2, 700, seed=41, outliers=True)
    qbar, _ = oracle.pool(q, 128)
    kbar, _ = oracle.pool(k, 64)
    got = oracle.block_scores(qbar, kbar)
    ref = np.einsum("bhic,bhjc->bhij", qbar.astype(np.float64), kbar.astype(np.float64))
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def _numpy_mask(scores, keep):
    B, H, nq, nk = scores.shape
    out = np.zeros(scores.shape, np.uint8)
    j = np.arange(nk)
    for b in range(B):
        for h in range(H):
            for i in range(nq):
                order = np.lexsort((j, -scores[b, h, i]))  # score descending, index ascending
                out[b, h, i, order[:keep]] = 1
    return out


@pytest.mark.parametrize("keep", [1, 3, 7, 16, 40])
def test_selection_rule_against_stable_sort_with_ties(oracle, keep):
    rng = np.random.default_rng(keep)
    scores = rng.integers(-4, 5, size=(1, 2, 5, 16)).astype(np.float64)  # many exact ties
    scores[0, 1, 2] = 0.0                                                  # a row of ties
    got = oracle.mask_from_scores(scores, keep)
    np.testing.assert_array_equal(got, _numpy_mask(scores, keep))
    assert (got.sum(axis=-1) == min(keep, 16)).all()


def test_diagonal_blocks_are_added(oracle):
    rng = np.random.default_rng(3)
    scores = rng.standard_normal((1, 1, 6, 11))
    got = oracle.mask_from_scores(scores, 2, keep_diagonal=True)
    base = oracle.mask_from_scores(scores, 2)
    for i in range(6):
        for jj in (2 * i, 2 * i + 1):
            if jj < 11:
                assert got[0, 0, i, jj] == 1
    assert ((got >= base).all()) and (got.sum() <= base.sum() + 11)


def _scale_bits(x_bits, f):
    return f32_to_bf16_bits(bf16_bits_to_f32(x_bits) * np.float32(f))


def test_mask_invariant_under_scaling_q_by_two(oracle):
    q, k, _, _ = make_inputs(1, 2, 1500, seed=42, outliers=True)
    m1 = oracle.block_mask(q, k, 4)[0]
    m2 = oracle.block_mask(_scale_bits(q, 2.0), k, 4)[0]  # exact in bf16, fp32 and fp64
    np.testing.assert_array_equal(m1, m2)


def test_swapping_two_key_blocks_swaps_mask_columns(oracle):
    q, k, _, _ = make_inputs(1, 1, 1024, seed=43, outliers=False)
    a, b = 3, 11
    k2 = k.copy()
    k2[:, :, a * 64:(a + 1) * 64], k2[:, :, b * 64:(b + 1) * 64] = k[:, :, b * 64:(b + 1) * 64], k[:, :, a * 64:(a + 1) * 64]
    m1, _, _, s1, _ = oracle.block_mask(q, k, 5)
    m2 = oracle.block_mask(q, k2, 5)[0]
    # no exact ties among the scores (else the index tie-break would differ)
    assert all(len(np.unique(r)) == r.size for r in s1.reshape(-1, s1.shape[-1]))
    m1[..., [a, b]] = m1[..., [b, a]]
    np.testing.assert_array_equal(m1, m2)


def test_planted_key_block_is_selected(oracle):
    """A key block whose tokens all point along query block i's mean, scaled up, scores
    highest in row i."""
    q, k, _, _ = make_inputs(1, 1, 2048, seed=44, outliers=False)
    i, jstar = 5, 23
    qmean = bf16_bits_to_f32(q)[0, 0, i * 128:(i + 1) * 128].mean(axis=0)
    k2 = k.copy()
    k2[0, 0, jstar * 64:(jstar + 1) * 64] = f32_to_bf16_bits(np.tile(40.0 * qmean / np.linalg.norm(qmean), (64, 1)).astype(np.float32))
    m = oracle.block_mask(q, k2, 1)[0]
    assert m[0, 0, i, jstar] == 1 and m[0, 0, i].sum() == 1


def test_keep_all_and_keep_one(oracle):
    q, k, _, _ = make_inputs(1, 2, 900, seed=45, outliers=True)
    nk = -(-900 // 64)
    assert (oracle.block_mask(q, k, nk)[0] == 1).all()
    assert (oracle.block_mask(q, k, 10 * nk)[0] == 1).all()
    assert (oracle.block_mask(q, k, 1)[0].sum(axis=-1) == 1).all()
