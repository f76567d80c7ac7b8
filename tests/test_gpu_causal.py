"""Causal attention on the GPU against the oracle's causal rows: rows on both sides of every
64-key boundary of the diagonal blocks, ragged tails, a user block mask intersected with the
causal pattern, the last row against the non-causal masked kernel, and full size at 480p."""
import numpy as np
import pytest
import torch

from bit_quantized_attention_sa_b200.workloads import WORKLOADS, make_inputs, make_workload

from _helpers import O_MAX_ABS, O_MIN_COS, cosine, gpu_rows, sm_scale, to_dev_bf16

pytestmark = pytest.mark.gpu


def _boundary_rows(B, H, N):
    picks = {0, 1, 62, 63, 64, 65, 126, 127, 128, 129, 191, 192, 255, 256, N // 2, N - 2, N - 1}
    return [(bh, r) for bh in range(B * H) for r in sorted(picks) if 0 <= r < N]


def _check(oracle, q, k, v, o, rows, mask=None):
    B, H, N, _ = q.shape
    ref = oracle.attn_rows(oracle.quantize_qk(q, k), oracle.quantize_v(v), N, sm_scale(), rows, mask, 2,
                           causal=True)
    got = gpu_rows(o, rows)
    assert np.abs(got - ref).max() <= O_MAX_ABS
    assert cosine(got, ref) >= O_MIN_COS


@pytest.mark.parametrize("B,H,N", [(1, 2, 1), (1, 2, 65), (1, 2, 300), (2, 1, 1000), (1, 2, 3000)])
def test_causal_matches_oracle(oracle, libsa, cuda_ok, B, H, N):
    q, k, v, _ = make_inputs(B, H, N, seed=140 + N, outliers=True)
    o = libsa.sa_attn_fwd_causal(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v))
    assert libsa.sa_get_device_status() == 0
    _check(oracle, q, k, v, o, _boundary_rows(B, H, N))


@pytest.mark.parametrize("N", [1000, 1024, 1100])
def test_last_row_equals_non_causal(libsa, cuda_ok, N):
    """The last row sees every key: the causal run takes the same steps on the same values as
    the non-causal one, bit for bit, both without a mask (the two-tile kernel) and with every
    block kept (the masked kernel)."""
    q, k, v, _ = make_inputs(1, 2, N, seed=150 + N, outliers=True)
    qd, kd, vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    ones = torch.ones((1, 2, -(-N // 128), -(-N // 64)), dtype=torch.uint8, device="cuda")
    oc = libsa.sa_attn_fwd_causal(qd, kd, vd)
    od = libsa.sa_attn_fwd(qd, kd, vd)
    assert torch.equal(oc[:, :, N - 1].view(torch.int16), od[:, :, N - 1].view(torch.int16))
    ocm = libsa.sa_attn_fwd_causal(qd, kd, vd, block_mask=ones)
    om = libsa.sa_attn_fwd(qd, kd, vd, block_mask=ones)
    assert torch.equal(ocm[:, :, N - 1].view(torch.int16), om[:, :, N - 1].view(torch.int16))


def test_causal_with_block_mask(oracle, libsa, cuda_ok):
    B, H, N = 1, 2, 2000
    q, k, v, _ = make_inputs(B, H, N, seed=151, outliers=True)
    rng = np.random.default_rng(151)
    nq, nk = -(-N // 128), -(-N // 64)
    mask = (rng.random((B, H, nq, nk)) < 0.5).astype(np.uint8)
    for i in range(nq):
        mask[:, :, i, 2 * i] = 1  # every row keeps its own first diagonal block
    o = libsa.sa_attn_fwd_causal(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v),
                                 block_mask=torch.from_numpy(mask).cuda())
    assert libsa.sa_get_device_status() == 0
    _check(oracle, q, k, v, o, _boundary_rows(B, H, N), mask)


def test_causal_full_size_480p(oracle, libsa, cuda_ok):
    w = WORKLOADS["wan14b-480p-h40-n32760"]
    q, k, v, _ = make_workload(w)
    o = libsa.sa_attn_fwd_causal(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), w.sm_scale)
    assert libsa.sa_get_device_status() == 0
    rows = [(0, 0), (0, 127), (5, 128), (11, 5000), (23, 16447), (39, 32639), (39, 32640), (17, 32759)]
    ref = oracle.attn_rows(oracle.quantize_qk(q, k), oracle.quantize_v(v), w.N, w.sm_scale, rows, None, 2,
                           causal=True)
    got = gpu_rows(o, rows)
    assert np.abs(got - ref).max() <= O_MAX_ABS
    assert cosine(got, ref) >= O_MIN_COS


def test_masked_out_zero_scale_block_leaves_the_max(oracle, libsa, cuda_ok):
    """A step whose keys all come after the row (tile 0 in its pair's second step) must not
    raise the row maximum, even where those key blocks have scale 0.  Keys 128-255 are zero
    and the other keys are +8 / -8 rows that cancel, so the K mean is exactly 0 and blocks 2
    and 3 quantise to scale 0; tile 0's queries are -8, so its real logits are about -720.
    A maximum of 0 taken from the masked blocks would scale O and its row sum by e^-720 = 0
    and return zeros.  Both kernels: no mask (two-tile kernel) and all blocks kept."""
    from bit_quantized_attention_sa_b200.workloads import f32_to_bf16_bits
    B, H, N = 1, 1, 512
    rng = np.random.default_rng(161)
    q = rng.standard_normal((B, H, N, 128)).astype(np.float32)
    q[:, :, :128] = -8.0
    k = np.zeros((B, H, N, 128), np.float32)
    k[:, :, 0:128] = 8.0
    k[:, :, 256:384] = -8.0
    v = rng.standard_normal((B, H, N, 128)).astype(np.float32)
    qb, kb, vb = f32_to_bf16_bits(q), f32_to_bf16_bits(k), f32_to_bf16_bits(v)
    qk = oracle.quantize_qk(qb, kb)
    assert np.all(qk[4] == 0) and np.all(qk[3][0, 0, 2:4] == 0)  # K mean 0; blocks 2, 3 scale 0
    rows = [(0, r) for r in (0, 1, 63, 64, 100, 127, 128, 200, 255, 256, 400, 511)]
    ref = oracle.attn_rows(qk, oracle.quantize_v(vb), N, sm_scale(), rows, None, 2, causal=True)
    assert np.abs(ref[:6]).max() > 0.05  # the tile-0 rows are far from zero
    qd, kd, vd = to_dev_bf16(qb), to_dev_bf16(kb), to_dev_bf16(vb)
    ones = torch.ones((B, H, N // 128, N // 64), dtype=torch.uint8, device="cuda")
    for o in (libsa.sa_attn_fwd_causal(qd, kd, vd), libsa.sa_attn_fwd_causal(qd, kd, vd, block_mask=ones)):
        assert libsa.sa_get_device_status() == 0
        got = gpu_rows(o, rows)
        assert np.abs(got - ref).max() <= O_MAX_ABS
        assert cosine(got, ref) >= O_MIN_COS
