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


@pytest.mark.timeout(600)
def test_training_step_sample_is_whole_token_groups():
    """The training step's oracle sample runs on whole 128-token groups (the
    transposed quantization's group length): the sample size is a multiple of
    128, at least one group and at most the workload's tokens."""
    wl = W.make_workload(14, 0, scale_down=64)          # 256 tokens
    assert wl.M == 256 and wl.flops == 6 * 2 * 256 * 5120 * 8192
    rows = bench.baseline_rows(wl, 0.5)
    assert rows % 128 == 0 and 128 <= rows <= wl.M
    tg, frac, tq, threads = bench.oracle_sample(wl, 130)   # rounds up to two groups
    assert frac == 1.0 and tg > 0 and tq > 0 and threads >= 1
