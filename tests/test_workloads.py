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


def test_sla_classes_recipe():
    from bit_quantized_attention_sa_b200.workloads import make_sla_classes
    a = make_sla_classes(1, 3, 5000, 0.1, 0.4, seed=3)
    assert np.array_equal(a, make_sla_classes(1, 3, 5000, 0.1, 0.4, seed=3))
    nq, nk = -(-5000 // 128), -(-5000 // 64)
    assert a.shape == (1, 3, nq, nk) and a.dtype == np.uint8
    assert set(np.unique(a)) <= {0, 1, 2}
    for i in range(nq):  # diagonal blocks are always critical
        for j in (2 * i, 2 * i + 1):
            if j < nk:
                assert (a[:, :, i, j] == 2).all()
    off = np.ones(a.shape, bool)
    for i in range(nq):
        off[:, :, i, 2 * i:2 * i + 2] = False
    frac = [(a[off] == c).mean() for c in (2, 1, 0)]
    assert abs(frac[0] - 0.1) < 0.02 and abs(frac[1] - 0.4) < 0.03 and abs(frac[2] - 0.5) < 0.03


def test_linear_inputs_recipe():
    from bit_quantized_attention_sa_b200.workloads import make_linear_inputs
    x, w = make_linear_inputs(5000, 64, 512, seed=4)
    x2, w2 = make_linear_inputs(5000, 64, 512, seed=4)
    assert np.array_equal(x, x2) and np.array_equal(w, w2)
    assert x.shape == (5000, 512) and w.shape == (64, 512) and x.dtype == np.uint16
    xf, wf = bf16_bits_to_f32(x), bf16_bits_to_f32(w)
    # round(1 % of 512) = 5 activation channels scaled by 8; the rest ~ N(0, 1)
    std = xf.std(axis=0)
    assert (std > 4).sum() == 5 and abs(np.median(std) - 1.0) < 0.05
    assert abs(wf.std() * np.sqrt(512) - 1.0) < 0.05
    # chunked draws (4096 rows at a time) continue one stream: rows past 4096 differ from
    # the first rows and keep the same statistics
    assert not np.array_equal(x[:100], x[4096:4196])
    assert abs(xf[4096:].std(axis=0)[std < 4].mean() - 1.0) < 0.05
