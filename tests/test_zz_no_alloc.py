"""sa_quantize_qk_noalloc: the Q/K quantisation for callers that cannot allocate device
memory (their device memory belongs to a host framework or pool that has already reserved
the GPU, or their loop cannot take cudaMalloc's implicit synchronisation).  It keeps its
scratch in a fixed array inside the library and must give exactly what the allocating
sa_quantize_qk gives.  Collected last on purpose: if it fails, every other test has
already run."""
import ctypes

import numpy as np
import pytest
import torch

from bit_quantized_attention_sa_b200.workloads import make_inputs

from _helpers import to_dev_bf16

pytestmark = pytest.mark.gpu


def _outputs(q):
    B, H, N, d = q.shape
    Np, nq, nk = -(-N // 128) * 128, -(-N // 128), -(-N // 64)
    dev = q.device
    return (torch.empty((B, H, Np, d), dtype=torch.int8, device=dev),
            torch.empty((B, H, nq), dtype=torch.float32, device=dev),
            torch.empty((B, H, Np, d), dtype=torch.int8, device=dev),
            torch.empty((B, H, nk), dtype=torch.float32, device=dev),
            torch.empty((B, H, d), dtype=torch.float32, device=dev))


def _call_noalloc(lib, q, k, out=None):
    B, H, N, d = q.shape
    out = _outputs(q) if out is None else out
    P = ctypes.c_void_p
    st = lib.sa_quantize_qk_noalloc(P(q.data_ptr()), P(k.data_ptr()), B, H, N, d,
                                    *[P(t.data_ptr()) for t in out],
                                    P(torch.cuda.current_stream(q.device).cuda_stream))
    return st, out


def test_noalloc_matches_allocating_entry_point_twice(libsa, cuda_ok):
    """Two calls in a row (the second reuses the scratch the first one left behind) give
    outputs bit-identical to sa_quantize_qk's."""
    lib = libsa.raw_library()
    for call, (H, N) in enumerate([(3, 3000), (2, 1030)]):
        q, k, _, _ = make_inputs(1, H, N, seed=900 + call, outliers=True)
        qd, kd = to_dev_bf16(q), to_dev_bf16(k)
        ref = libsa.sa_quantize_qk(qd, kd)
        st, got = _call_noalloc(lib, qd, kd)
        assert st == 0, libsa.sa_status_string(st)
        torch.cuda.synchronize()
        assert libsa.sa_get_device_status() == 0
        for r, g in zip(ref, got):
            assert torch.equal(r.view(torch.uint8) if r.dtype == torch.int8 else r.view(torch.int32),
                               g.view(torch.uint8) if g.dtype == torch.int8 else g.view(torch.int32))


def test_noalloc_rejects_sizes_beyond_its_scratch(libsa):
    """B * H * ceil(N/1024) above 4096 is refused before anything is launched."""
    lib = libsa.raw_library()
    fake = ctypes.c_void_p(1 << 20)
    st = lib.sa_quantize_qk_noalloc(fake, fake, 1, 4097, 1024, 128, fake, fake, fake, fake,
                                    fake, None)
    assert st == 7 and libsa.sa_status_string(st) == "SA_ERR_SCRATCH_LIMIT"


def test_noalloc_takes_no_device_memory(libsa, cuda_ok):
    """The call itself allocates nothing: with the library workspace released and the
    outputs allocated beforehand, the device's free memory is the same before and after a
    call whose allocating counterpart needs a workspace of hundreds of MB (which the same
    measurement does see)."""
    lib = libsa.raw_library()
    libsa.sa_release_workspace()
    # a first small call loads the library's module (and with it the fixed array) and
    # looks up the array's address
    q, k, _, _ = make_inputs(1, 1, 256, seed=950)
    st, _ = _call_noalloc(lib, to_dev_bf16(q), to_dev_bf16(k))
    assert st == 0
    torch.cuda.synchronize()
    q, k, _, _ = make_inputs(1, 16, 32760, seed=951)
    qd, kd = to_dev_bf16(q), to_dev_bf16(k)
    out = _outputs(qd)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    st, got = _call_noalloc(lib, qd, kd, out)
    assert st == 0, libsa.sa_status_string(st)
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    assert free1 == free0, (free0, free1)
    assert libsa.sa_get_device_status() == 0
    # the allocating entry point grows the library workspace for the same problem: free
    # memory drops by at least the workspace (its outputs, from torch, are smaller)
    need = libsa.sa_workspace_bytes(1, 16, 32760)
    assert need > 128 << 20
    ref = libsa.sa_quantize_qk(qd, kd)
    torch.cuda.synchronize()
    assert free1 - torch.cuda.mem_get_info()[0] >= need
    for r, g in zip(ref, got):
        assert torch.equal(r.view(torch.uint8) if r.dtype == torch.int8 else r.view(torch.int32),
                           g.view(torch.uint8) if g.dtype == torch.int8 else g.view(torch.int32))
    libsa.sa_release_workspace()
