"""Shared pytest set-up: the ``gpu`` marker and the repository root on sys.path."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def orc():
    from oracle import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def pa():
    """The CUDA library's binding; GPU tests fail (never skip) without a device."""
    import torch
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"
    from paged_kv_cache_390_b200 import build as _build
    _build.build()
    from paged_kv_cache_390_b200 import pa as _pa
    _pa.lib()
    return _pa
