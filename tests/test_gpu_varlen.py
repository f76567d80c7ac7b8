"""The packed variable-length entry point: each sequence of the batch comes out bit for bit
as its own sa_attn_fwd (or sa_attn_fwd_causal) call, for ragged lengths including 1, 64 and
non-multiples of 128, and a sampled row matches the oracle."""
import numpy as np
import pytest
import torch

from bit_quantized_attention_sa_b200.workloads import make_inputs

from _helpers import O_MAX_ABS, O_MIN_COS, cosine, sm_scale, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_per_sequence_calls(oracle, libsa, cuda_ok, causal):
    H, lens = 2, [1, 200, 129, 1000, 64, 333]
    seqs = [make_inputs(1, H, n, seed=160 + n, outliers=True)[:3] for n in lens]
    packed = [torch.cat([to_dev_bf16(s[t]).reshape(-1) for s in seqs]) for t in range(3)]
    o = libsa.sa_attn_fwd_varlen(*packed, lens, H, causal=causal)
    assert libsa.sa_get_device_status() == 0
    off = 0
    for n, (q, k, v) in zip(lens, seqs):
        qd, kd, vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
        ref = libsa.sa_attn_fwd_causal(qd, kd, vd) if causal else libsa.sa_attn_fwd(qd, kd, vd)
        got = o[off:off + H * n * 128].reshape(1, H, n, 128)
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), n
        off += H * n * 128
    # one sequence against the oracle
    q, k, v = seqs[3]
    rows = [(bh, r) for bh in range(H) for r in (0, 127, 128, 640, 999)]
    start = H * (lens[0] + lens[1] + lens[2]) * 128
    blk = o[start:start + H * 1000 * 128].reshape(H, 1000, 128).float().cpu().numpy()
    got = np.stack([blk[bh, r] for bh, r in rows])
    ref = oracle.attn_rows(oracle.quantize_qk(q, k), oracle.quantize_v(v), 1000, sm_scale(), rows, None, 2,
                           causal=causal)
    assert np.abs(got - ref).max() <= O_MAX_ABS
    assert cosine(got, ref) >= O_MIN_COS


def _check_against_own_calls(libsa, lens, H, causal, seed):
    seqs = [make_inputs(1, H, n, seed=seed + i, outliers=(i % 2 == 0))[:3] for i, n in enumerate(lens)]
    packed = [torch.cat([to_dev_bf16(s[t]).reshape(-1) for s in seqs]) for t in range(3)]
    o = libsa.sa_attn_fwd_varlen(*packed, lens, H, causal=causal)
    assert libsa.sa_get_device_status() == 0
    off = 0
    for n, (q, k, v) in zip(lens, seqs):
        qd, kd, vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
        ref = libsa.sa_attn_fwd_causal(qd, kd, vd) if causal else libsa.sa_attn_fwd(qd, kd, vd)
        got = o[off:off + H * n * 128].reshape(1, H, n, 128)
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), n
        off += H * n * 128


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_64_short_sequences_one_launch_each_equal_own_call(libsa, cuda_ok, causal):
    """64 sequences of 1 to 512 tokens: one group, i.e. one prologue and one attention
    launch for the whole batch; every sequence bit for bit as its own call."""
    lens = [int(n) for n in np.random.default_rng(77).integers(1, 513, size=64)]
    lens[0], lens[1] = 1, 512
    _check_against_own_calls(libsa, lens, 2, causal, seed=3000)


def test_varlen_groups_of_mixed_lengths(libsa, cuda_ok):
    """One long sequence and forty short ones: the padding rule splits them into two groups
    (the long one with the first 25 short ones, then the rest); results unchanged."""
    _check_against_own_calls(libsa, [40000] + [1000] * 40, 1, False, seed=3100)
