"""Host-side parts of the benchmark, run without a GPU: every workload the
benchmark accepts has a CPU-oracle sample (the reference arm and the
cpu_baseline leg), and each names the source file its ncu traffic record is
keyed on."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("workload", bench.WORKLOAD_NAMES)
def test_oracle_sample_runs_for_every_workload(workload):
    rate, spent, desc = bench.oracle_sample(workload, small=True)
    assert rate > 0 and spent > 0 and desc


@pytest.mark.parametrize("workload", [w for w in bench.WORKLOAD_NAMES if w != "headline"])
def test_every_workload_names_its_kernel_source(workload):
    src = bench.KERNEL_SOURCES[workload]
    assert os.path.exists(os.path.join(ROOT, "gemv_zero_point_b200", "csrc", src))
    assert len(bench.source_digest(workload)) == 16
