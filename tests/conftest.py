import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle():
    import oracle as _oracle
    _oracle.build()
    return _oracle


@pytest.fixture(scope="session")
def libsa():
    """The built C-ABI library (built in-tree with nvcc if missing or stale)."""
    from bit_quantized_attention_sa_b200 import build as _build
    _build.build()
    from bit_quantized_attention_sa_b200 import binding
    return binding


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for tests marked gpu")
    return True
