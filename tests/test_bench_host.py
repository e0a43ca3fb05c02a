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


def test_power_capped_needs_a_lowered_clock():
    # the limiter's flag with the clock at its maximum keeps the burst peak
    assert not bench.power_capped({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0,
                                   "reasons": ["sw_power_cap"]})
    assert bench.power_capped({"sm_mhz": 1320.0, "sm_max_mhz": 1965.0,
                               "reasons": ["sw_power_cap"]})
    assert not bench.power_capped({"sm_mhz": 1320.0, "sm_max_mhz": 1965.0, "reasons": []})
    assert not bench.power_capped(None)
    # no clock figures recorded: trust the flag
    assert bench.power_capped({"reasons": ["sw_power_cap"]})
