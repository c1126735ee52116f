"""The CPU-baseline / reference leg of bench.py runs for every workload
(on a reduced token or row count; the oracle's sample covers a few output
rows): it must reach the oracle for each workload's recipe and report a
positive throughput.  No GPU involved."""
import pytest

import bench
from fp8_scaled_matrix_b200 import workloads as W


@pytest.mark.timeout(600)
@pytest.mark.parametrize("name", sorted(bench.WORKLOADS))
def test_cpu_baseline_runs_for_every_workload(name):
    idx, shape_index = bench.WORKLOADS[name]
    wl = W.make_workload(idx, shape_index, scale_down=128)
    b = bench.cpu_baseline(wl, 2)
    assert b["kind"] == "oracle" and b["value"] > 0 and b["cores"] >= 1
    assert "scaled to all rows" in b["sample"]
