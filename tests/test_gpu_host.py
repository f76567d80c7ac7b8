"""sa_attn_fwd_host: the forward on host buffers, with the heads split into chunks whose
uploads and downloads overlap the computation.  Its output must be bit-identical to
sa_attn_fwd's on the same inputs, for several chunks (a short last one included), with and
without a keep mask, and the call must complete on the stream it was given."""
import numpy as np
import pytest
import torch

from bit_quantized_attention_sa_b200.workloads import make_inputs

from _helpers import to_dev_bf16

pytestmark = pytest.mark.gpu


def _host_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()


def _mask(B, H, N, density, seed):
    rng = np.random.default_rng(seed)
    m = (rng.random((B, H, -(-N // 128), -(-N // 64))) < density).astype(np.uint8)
    m[..., 0] = 1  # every row keeps at least one block
    return m


# Chunks hold 64 MB of q: N = 75600 gives 3 heads a chunk (7 heads: 3 + 3 + 1), N = 32760
# gives 7 (16 heads: 7 + 7 + 2).
@pytest.mark.parametrize("B,H,N,density", [(1, 7, 75600, None), (2, 8, 32760, 0.3), (1, 2, 1030, None)])
def test_host_pipeline_matches_device_forward(libsa, cuda_ok, B, H, N, density):
    q, k, v, _ = make_inputs(B, H, N, seed=700 + H, outliers=True)
    m = _mask(B, H, N, density, 7) if density is not None else None
    ref = libsa.sa_attn_fwd(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v),
                            block_mask=None if m is None else torch.from_numpy(m).cuda())
    hq, hk, hv = _host_bf16(q), _host_bf16(k), _host_bf16(v)
    hm = None if m is None else torch.from_numpy(m).pin_memory()
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        got = libsa.sa_attn_fwd_host(hq, hk, hv, block_mask=hm, stream=st)
    st.synchronize()
    assert libsa.sa_get_device_status() == 0
    assert torch.equal(got.view(torch.int16), ref.cpu().view(torch.int16))


def test_host_pipeline_twice_reuses_staging(libsa, cuda_ok):
    """A second call right after the first (same staging slots, no synchronisation in
    between) still gives the first call's results for both."""
    B, H, N = 1, 5, 75600
    ins = [make_inputs(B, H, N, seed=s, outliers=False)[:3] for s in (1, 2)]
    refs = [libsa.sa_attn_fwd(*[to_dev_bf16(a) for a in x]).cpu() for x in ins]
    outs, keep = [], []
    for x in ins:
        # the host inputs must outlive the asynchronous copies: keep them until the sync
        keep.append([_host_bf16(a) for a in x])
        outs.append(libsa.sa_attn_fwd_host(*keep[-1]))
    torch.cuda.current_stream().synchronize()
    for got, ref in zip(outs, refs):
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
