"""Shared helpers for the GPU parity tests (not collected)."""
import math

import numpy as np
import torch


def to_dev_bf16(a: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> CUDA bfloat16 tensor (bit-identical)."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def to_host_f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def cosine(a, b) -> float:
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    den = np.linalg.norm(a) * np.linalg.norm(b)
    return float(a @ b / den) if den > 0 else float(np.array_equal(a, b))


def sm_scale(d=128):
    return 1.0 / math.sqrt(d)


# tolerance for O against the oracle (bf16 output, ex2.approx vs expf, tensor-core fp32
# accumulation order): max-abs and cosine
O_MAX_ABS = 2e-2
O_MIN_COS = 0.9995


def gpu_rows(o: torch.Tensor, rows):
    """Rows [(bh, r), ...] of a [B,H,N,d] CUDA output as fp32 numpy [len(rows), d]."""
    B, H, N, d = o.shape
    flat = o.reshape(B * H, N, d)
    idx_bh = torch.tensor([r[0] for r in rows], device=o.device)
    idx_r = torch.tensor([r[1] for r in rows], device=o.device)
    return to_host_f32(flat[idx_bh, idx_r])
