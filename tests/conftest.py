"""Test configuration: the `gpu` marker and the repository root on sys.path."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


import pytest  # noqa: E402


@pytest.fixture(scope="session")
def dsv4():
    """The CUDA binding (loads libdsv4.so; fails loudly if it is missing)."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test selected but no CUDA device is visible")
    import compressed_sparse_mqa_dsv4_b200 as m
    return m
