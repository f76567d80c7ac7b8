"""The seeded input generators: determinism, bf16 rounding, offsets, outlier channels and
the block-mask recipe."""
import numpy as np
import torch

from bit_quantized_attention_sa_b200.workloads import (WORKLOADS, bf16_bits_to_f32,
                                                       f32_to_bf16_bits, make_inputs)


def test_deterministic_and_seed_sensitive():
    a = make_inputs(1, 2, 300, seed=5, outliers=True, mask_density=0.1)
    b = make_inputs(1, 2, 300, seed=5, outliers=True, mask_density=0.1)
    c = make_inputs(1, 2, 300, seed=6, outliers=True, mask_density=0.1)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    assert not np.array_equal(a[0], c[0])


def test_bf16_rounding_matches_library_cast():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 37
    ours = f32_to_bf16_bits(x)
    lib = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, lib)
    assert np.array_equal(bf16_bits_to_f32(ours), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_offsets_and_outliers():
    q, k, v, _ = make_inputs(1, 3, 4000, seed=9, outliers=True)
    kf = bf16_bits_to_f32(k)
    qf = bf16_bits_to_f32(q)
    for h in range(3):
        mean = kf[0, h].mean(axis=0)
        assert 1.0 < mean.std() < 3.5                  # per-channel offsets ~ N(0, 2^2)
        qstd = qf[0, h].std(axis=0)
        assert (qstd > 5).sum() == 1 and (qstd < 1.2).sum() == 127
        kc = kf[0, h] - mean
        assert (kc.std(axis=0) > 5).sum() == 1
    assert abs(bf16_bits_to_f32(v).std() - 1) < 0.01


def test_mask_recipe():
    _, _, _, m = make_inputs(1, 2, 32760, seed=1004, mask_density=0.0965)
    nq, nk = 256, 512
    assert m.shape == (1, 2, nq, nk) and m.dtype == np.uint8
    for i in range(nq):
        assert m[0, 0, i, 2 * i] == 1 and m[0, 0, i, 2 * i + 1] == 1
    dens = m.mean()
    assert 0.09 < dens < 0.11


def test_named_workloads():
    assert [w.N for w in WORKLOADS.values()] == [1024, 32760, 32760, 75600, 32760]
    assert [w.H for w in WORKLOADS.values()] == [2, 12, 40, 40, 40]
    w = WORKLOADS["wan14b-720p-h40-n75600"]
    assert abs(w.dense_ops - 1.1705e14) / 1.1705e14 < 1e-3
