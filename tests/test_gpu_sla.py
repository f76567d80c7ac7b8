"""The SLA path on the GPU against the oracle: the linear branch over the marginal blocks
(fp32, both feature maps, with and without a projection) and the full SLA forward (sparse
quantised attention over the critical blocks plus the projected linear branch), on ragged
and full-size shapes, and the degenerate class maps."""
import numpy as np
import pytest
import torch

from bit_quantized_attention_sa_b200.workloads import WORKLOADS, make_inputs, make_sla_classes, make_workload, sample_rows

from _helpers import O_MAX_ABS, O_MIN_COS, cosine, gpu_rows, sm_scale, to_dev_bf16

pytestmark = pytest.mark.gpu

LIN_RTOL, LIN_ATOL = 1e-4, 1e-4  # fp32 factorised sums against the fp64 weighted average


def _proj(seed, d=128):
    return (np.random.default_rng(seed).standard_normal((d, d)) / np.sqrt(d)).astype(np.float32)


def _rows(B, H, N, per_head=6, seed=7):
    rows = sample_rows(B, H, N, per_head, seed)
    if N > 32768:  # more than 256 query blocks: rows of the second query-block tile too
        rows = rows + [(0, 32768 + 5), (B * H - 1, N - 1)]
    return rows


@pytest.mark.parametrize("B,H,N", [(1, 2, 1), (1, 2, 200), (2, 1, 1000), (1, 3, 3000), (1, 2, 40000)])
@pytest.mark.parametrize("phi", [0, 1])
def test_linear_branch_matches_oracle(oracle, libsa, cuda_ok, B, H, N, phi):
    q, k, v, _ = make_inputs(B, H, N, seed=100 + N + phi, outliers=True)
    classes = make_sla_classes(B, H, N, 0.2, 0.45, seed=N + phi)
    rows = _rows(B, H, N)
    qd, kd, vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    cd = torch.from_numpy(classes).cuda()
    for proj in (None, _proj(N)):
        pd = None if proj is None else torch.from_numpy(proj).cuda()
        got = gpu_rows(libsa.sa_sla_linear(qd, kd, vd, cd, phi=phi, proj=pd), rows)
        ref = oracle.sla_linear_rows(q, k, v, classes, phi, proj, rows)
        np.testing.assert_allclose(got, ref, rtol=LIN_RTOL, atol=LIN_ATOL)


@pytest.mark.parametrize("B,H,N,phi", [(1, 2, 300, 0), (1, 2, 2000, 1), (2, 2, 4000, 0)])
def test_sla_forward_matches_oracle(oracle, libsa, cuda_ok, B, H, N, phi):
    q, k, v, _ = make_inputs(B, H, N, seed=110 + N, outliers=True)
    classes = make_sla_classes(B, H, N, 0.1, 0.4, seed=N)
    proj = _proj(N + 1)
    o = libsa.sa_sla_fwd(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), torch.from_numpy(classes).cuda(),
                         phi=phi, proj=torch.from_numpy(proj).cuda())
    assert libsa.sa_get_device_status() == 0
    rows = _rows(B, H, N, per_head=8)
    crit = (classes >= 2).astype(np.uint8)
    ref = oracle.attn_rows(oracle.quantize_qk(q, k), oracle.quantize_v(v), N, sm_scale(), rows, crit, 2)
    ref = ref.astype(np.float64) + oracle.sla_linear_rows(q, k, v, classes, phi, proj, rows)
    got = gpu_rows(o, rows)
    assert np.abs(got - ref).max() <= O_MAX_ABS
    assert cosine(got, ref) >= O_MIN_COS


def test_degenerate_class_maps(oracle, libsa, cuda_ok):
    B, H, N = 1, 2, 1000
    q, k, v, _ = make_inputs(B, H, N, seed=120, outliers=True)
    qd, kd, vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    nq, nk = -(-N // 128), -(-N // 64)
    zeros = torch.zeros((B, H, nq, nk), dtype=torch.uint8, device="cuda")
    # nothing kept: O = 0
    assert not libsa.sa_sla_fwd(qd, kd, vd, zeros).float().abs().max().item()
    # everything critical: exactly the masked quantised attention with every block kept
    all2 = torch.full_like(zeros, 2)
    o_sla = libsa.sa_sla_fwd(qd, kd, vd, all2)
    o_att = libsa.sa_attn_fwd(qd, kd, vd, block_mask=torch.ones_like(zeros))
    assert torch.equal(o_sla.float(), o_att.float())  # values equal (a -0.0 may come back as +0.0)
    # everything marginal: the sparse part is 0 and O is the linear branch rounded to bf16
    all1 = torch.ones_like(zeros)
    o_lin = libsa.sa_sla_fwd(qd, kd, vd, all1, phi=1)
    lin = libsa.sa_sla_linear(qd, kd, vd, all1, phi=1)
    assert torch.equal(o_lin.float(), lin.to(torch.bfloat16).float())
    rows = _rows(B, H, N)
    ref = oracle.sla_linear_rows(q, k, v, np.ones((B, H, nq, nk), np.uint8), 1, None, rows)
    np.testing.assert_allclose(gpu_rows(lin, rows), ref, rtol=LIN_RTOL, atol=LIN_ATOL)


def test_full_size_480p_sampled_rows(oracle, libsa, cuda_ok):
    """Wan2.1-14B at 480p (H = 40, N = 32760): 10 % critical and 40 % marginal blocks."""
    w = WORKLOADS["wan14b-480p-h40-n32760"]
    q, k, v, _ = make_workload(w)
    classes = make_sla_classes(w.B, w.H, w.N, 0.0965, 0.4, seed=7)
    proj = _proj(3)
    qd, kd, vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    cd, pd = torch.from_numpy(classes).cuda(), torch.from_numpy(proj).cuda()
    lin = libsa.sa_sla_linear(qd, kd, vd, cd, phi=0, proj=pd)
    o = libsa.sa_sla_fwd(qd, kd, vd, cd, phi=0, proj=pd)
    assert libsa.sa_get_device_status() == 0
    rows = [(0, 0), (7, 12345), (39, 32759), (21, 32640)]
    ref_lin = oracle.sla_linear_rows(q, k, v, classes, 0, proj, rows)
    np.testing.assert_allclose(gpu_rows(lin, rows), ref_lin, rtol=LIN_RTOL, atol=LIN_ATOL)
    crit = (classes >= 2).astype(np.uint8)
    ref = oracle.attn_rows(oracle.quantize_qk(q, k), oracle.quantize_v(v), w.N, w.sm_scale, rows, crit, 2)
    ref = ref.astype(np.float64) + ref_lin
    got = gpu_rows(o, rows)
    assert np.abs(got - ref).max() <= O_MAX_ABS
    assert cosine(got, ref) >= O_MIN_COS
