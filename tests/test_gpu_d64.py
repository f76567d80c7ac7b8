"""Head size 64 on the GPU (the d = 128 kernels on zero-padded copies) against the
oracle's native d = 64 rows: dense, causal and block-masked, ragged lengths."""
import math

import numpy as np
import pytest
import torch

from bit_quantized_attention_sa_b200.workloads import make_inputs, sample_rows

from _helpers import O_MAX_ABS, O_MIN_COS, cosine, gpu_rows, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,N,mode", [(1, 2, 1, "dense"), (1, 2, 300, "dense"), (2, 1, 1000, "dense"),
                                        (1, 2, 700, "causal"), (1, 3, 2000, "mask")])
def test_d64_matches_oracle(oracle, libsa, cuda_ok, B, H, N, mode):
    q, k, v, _ = make_inputs(B, H, N, d=64, seed=180 + N, outliers=True)
    scale = 1.0 / math.sqrt(64)
    qd, kd, vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    mask = None
    if mode == "mask":
        rng = np.random.default_rng(N)
        mask = (rng.random((B, H, -(-N // 128), -(-N // 64))) < 0.4).astype(np.uint8)
        o = libsa.sa_attn_fwd(qd, kd, vd, block_mask=torch.from_numpy(mask).cuda())
    elif mode == "causal":
        o = libsa.sa_attn_fwd_causal(qd, kd, vd)
    else:
        o = libsa.sa_attn_fwd(qd, kd, vd)
    assert libsa.sa_get_device_status() == 0
    assert o.shape == (B, H, N, 64)
    rows = sample_rows(B, H, N, 6, seed=N)
    ref = oracle.attn_rows(oracle.quantize_qk(q, k), oracle.quantize_v(v), N, scale, rows, mask, 2,
                           causal=(mode == "causal"))
    got = gpu_rows(o, rows)
    assert np.abs(got - ref).max() <= O_MAX_ABS
    assert cosine(got, ref) >= O_MIN_COS
