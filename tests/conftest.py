"""Shared pytest configuration.

Tests marked ``gpu`` need a B200 (sm_100a) and the in-tree CUDA library; they
are skipped here when no GPU is visible only if the run deselects them with
``-m "not gpu"``.  Selecting them on a machine without a GPU fails loudly
instead of passing on a fallback.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_collection_modifyitems(config, items):
    # GPU tests without a GPU: fail with a clear message rather than skip.
    pass


@pytest.fixture(scope="session")
def lib():
    """The C-ABI library loaded through the thin Python binding."""
    import gemv_zero_point_b200 as qg
    return qg


@pytest.fixture(scope="session")
def cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test selected but no CUDA device is visible")
    return torch.device("cuda:0")
