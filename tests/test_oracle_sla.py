"""Pins of the SLA linear branch in the oracle: the factorised form computed with library
feature maps (scipy's softmax, torch's elu) in a different association, closed forms (one
key, identical keys, no marginal block), invariants (convex combination, constant V
columns, linearity of the projection) and the class semantics (only class 1 counts)."""
import numpy as np
import pytest
import scipy.special
import torch

from bit_quantized_attention_sa_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits, make_inputs

QBLK, KBLK = 128, 64


def _classes(rng, B, H, N, p_marg=0.4, p_crit=0.2):
    nq, nk = -(-N // QBLK), -(-N // KBLK)
    u = rng.random((B, H, nq, nk))
    return np.where(u < p_crit, 2, np.where(u < p_crit + p_marg, 1, 0)).astype(np.uint8)


def _phi_lib(x: np.ndarray, phi: int) -> np.ndarray:
    if phi == 0:
        return scipy.special.softmax(x, axis=-1)
    return torch.nn.functional.elu(torch.from_numpy(x)).numpy() + 1.0


def _factorised(q, k, v, classes, phi, proj, rows):
    """phi(q)^T (sum phi(k) v^T) / (phi(q) . sum phi(k)) over each row's marginal keys."""
    B, H, N, d = q.shape
    qf, kf, vf = (bf16_bits_to_f32(a).astype(np.float64) for a in (q, k, v))
    out = np.zeros((len(rows), d))
    for n, (bh, r) in enumerate(rows):
        b, h = divmod(bh, H)
        marg = np.repeat(classes[b, h, r // QBLK] == 1, KBLK)[:N]
        if not marg.any():
            continue
        pk = _phi_lib(kf[b, h][marg], phi)
        state = pk.T @ vf[b, h][marg]          # d x d
        z = pk.sum(axis=0)                     # d
        pq = _phi_lib(qf[b, h, r][None, :], phi)[0]
        ol = (pq @ state) / (pq @ z)
        out[n] = ol if proj is None else proj.astype(np.float64) @ ol
    return out


@pytest.mark.parametrize("phi", [0, 1])
@pytest.mark.parametrize("N", [1, 65, 200, 700])
def test_matches_factorised_form_with_library_feature_maps(oracle, phi, N):
    rng = np.random.default_rng(N + 10 * phi)
    q, k, v, _ = make_inputs(1, 2, N, seed=90 + N, outliers=True)
    classes = _classes(rng, 1, 2, N)
    proj = rng.standard_normal((128, 128)).astype(np.float32) / 11.0
    rows = [(bh, r) for bh in range(2) for r in sorted(set([0, N - 1, N // 2, min(N - 1, 130)]))]
    for pr in (None, proj):
        got = oracle.sla_linear_rows(q, k, v, classes, phi, pr, rows)
        ref = _factorised(q, k, v, classes, phi, pr, rows)
        np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-11)


@pytest.mark.parametrize("phi", [0, 1])
def test_single_marginal_key_returns_its_value(oracle, phi):
    """N = 129: key block 2 holds the single token 128; if it is the only marginal block,
    every row of the query block returns v[128]."""
    N = 129
    q, k, v, _ = make_inputs(1, 1, N, seed=91)
    classes = np.zeros((1, 1, 2, 3), np.uint8)
    classes[0, 0, 0, 2] = 1
    classes[0, 0, 0, 0] = 2  # critical: not part of the linear branch
    got = oracle.sla_linear_rows(q, k, v, classes, phi, None, [(0, 0), (0, 77), (0, 127), (0, 128)])
    np.testing.assert_allclose(got[:3], np.tile(bf16_bits_to_f32(v[0, 0, 128]), (3, 1)), rtol=0, atol=1e-15)
    assert not got[3].any()  # query block 1 has no marginal block


@pytest.mark.parametrize("phi", [0, 1])
def test_identical_keys_average_the_values(oracle, phi):
    N = 256
    q, k, v, _ = make_inputs(1, 1, N, seed=92)
    k = np.tile(k[:, :, :1], (1, 1, N, 1))
    classes = np.ones((1, 1, 2, 4), np.uint8)
    got = oracle.sla_linear_rows(q, k, v, classes, phi, None, [(0, 5), (0, 200)])
    mean_v = bf16_bits_to_f32(v[0, 0]).astype(np.float64).mean(axis=0)
    np.testing.assert_allclose(got, np.tile(mean_v, (2, 1)), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("phi", [0, 1])
def test_convex_combination_and_constant_columns(oracle, phi):
    rng = np.random.default_rng(93)
    N = 500
    q, k, v, _ = make_inputs(1, 1, N, seed=93, outliers=True)
    vf = bf16_bits_to_f32(v).copy()
    vf[..., 7] = 3.25
    v = f32_to_bf16_bits(vf)
    classes = _classes(rng, 1, 1, N, p_marg=0.6, p_crit=0.0)
    classes[..., 0] = 1  # every row has a marginal block
    rows = [(0, r) for r in range(0, N, 37)]
    got = oracle.sla_linear_rows(q, k, v, classes, phi, None, rows)
    np.testing.assert_allclose(got[:, 7], 3.25, rtol=1e-13)
    for n, (_, r) in enumerate(rows):
        marg = np.repeat(classes[0, 0, r // QBLK] == 1, KBLK)[:N]
        lo = vf[0, 0][marg].min(axis=0).astype(np.float64)
        hi = vf[0, 0][marg].max(axis=0).astype(np.float64)
        assert (got[n] >= lo - 1e-12).all() and (got[n] <= hi + 1e-12).all()


def test_no_marginal_block_gives_zero_and_other_classes_are_ignored(oracle):
    rng = np.random.default_rng(94)
    N = 300
    q, k, v, _ = make_inputs(1, 1, N, seed=94)
    classes = rng.choice(np.array([0, 2, 3], np.uint8), size=(1, 1, 3, 5))
    rows = [(0, r) for r in (0, 150, 299)]
    assert not oracle.sla_linear_rows(q, k, v, classes, 0, None, rows).any()
    # changing keys and values outside the marginal blocks changes nothing
    classes[0, 0, :, 1] = 1
    base = oracle.sla_linear_rows(q, k, v, classes, 1, None, rows)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, :64] = k[:, :, 128:192]
    v2[:, :, 128:] = v[:, :, :172]
    np.testing.assert_array_equal(oracle.sla_linear_rows(q, k2, v2, classes, 1, None, rows), base)


def test_projection_is_applied_to_the_branch_output(oracle):
    rng = np.random.default_rng(95)
    N = 256
    q, k, v, _ = make_inputs(1, 2, N, seed=95)
    classes = _classes(rng, 1, 2, N, p_marg=0.7)
    classes[..., 1] = 1
    rows = [(bh, r) for bh in range(2) for r in (3, 131, 255)]
    proj = rng.standard_normal((128, 128)).astype(np.float32)
    plain = oracle.sla_linear_rows(q, k, v, classes, 0, None, rows)
    ident = oracle.sla_linear_rows(q, k, v, classes, 0, np.eye(128, dtype=np.float32), rows)
    np.testing.assert_array_equal(plain, ident)
    projected = oracle.sla_linear_rows(q, k, v, classes, 0, proj, rows)
    np.testing.assert_allclose(projected, plain @ proj.astype(np.float64).T, rtol=1e-12, atol=1e-12)
