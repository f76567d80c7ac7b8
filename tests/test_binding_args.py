"""The Python binding's argument marshalling without a GPU: wrong devices, dtypes and shapes
are rejected with ValueError before any native call."""
import pytest
import torch


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_attention_entry_points_reject_cpu_and_bad_shapes(libsa):
    q = _bf16(1, 2, 64, 128)
    with pytest.raises(ValueError):
        libsa.sa_attn_fwd(q, q, q)                      # CPU tensors
    with pytest.raises(ValueError):
        libsa.sa_attn_fwd_causal(q, q, q)
    with pytest.raises(ValueError):
        libsa.sa_block_mask(q, q, 1)
    with pytest.raises(ValueError):
        libsa.sa_attn_fwd_varlen(q.reshape(-1), q.reshape(-1), q.reshape(-1), [64], 2)


def test_w8a8_entry_points_validate(libsa):
    x = _bf16(128, 256)
    with pytest.raises(ValueError):
        libsa.sa_w8a8_quantize(x)                       # CPU tensor
    with pytest.raises(ValueError):
        libsa.sa_w8a8_quantize(torch.zeros(128, 256))   # fp32, not bf16
    codes = torch.zeros(128, 256, dtype=torch.int8)
    scales = torch.zeros(1, 2)
    with pytest.raises(ValueError):
        libsa.sa_w8a8_gemm((codes, scales), (codes, scales), 256)


def test_sla_entry_points_validate(libsa):
    q = _bf16(1, 2, 300, 128)
    cls = torch.zeros(1, 2, 3, 5, dtype=torch.uint8)
    with pytest.raises(ValueError):
        libsa.sa_sla_linear(q, q, q, cls)               # CPU tensors
    with pytest.raises(ValueError):
        libsa.sa_sla_fwd(q, q, q, cls)
