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


def pytest_terminal_summary(terminalreporter):
    """Observed A8W4 output errors (see tests/a8w4_tol.py), worst per label."""
    mod = sys.modules.get("a8w4_tol")
    if not mod or not mod.OBSERVED:
        return
    worst = {}
    for label, st in mod.OBSERVED:
        cur = worst.setdefault(label or "(unlabelled)", dict(st, calls=0))
        cur["calls"] += 1
        for k, v in st.items():
            if k.startswith("max"):
                cur[k] = max(cur[k], v)
        cur["n"] = max(cur["n"], st["n"])
    tr = terminalreporter
    tr.write_sep("-", "A8W4 observed float error (worst over calls)")
    tr.write_line(f"{'label':44s} {'calls':>5s} {'max|dy|':>10s} {'rel|y|>=1':>10s} "
                  f"{'/max(|y|,1)':>11s} {'/max(|y|,.01)':>13s} {'/max(|y|,1e-3)':>14s}")
    for label, st in sorted(worst.items()):
        tr.write_line(f"{label[:44]:44s} {st['calls']:5d} {st['max_abs']:10.2e} "
                      f"{st['max_rel_where_abs_ge_1']:10.2e} {st['max_scaled']:11.2e} "
                      f"{st['max_scaled_floor_1e-2']:13.2e} {st['max_scaled_floor_1e-3']:14.2e}")


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
