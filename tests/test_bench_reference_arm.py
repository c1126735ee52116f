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
    rows = bench.sample_rows(wl)
    assert rows % 128 == 0 and 128 <= rows <= wl.M
    tg, frac, tq, threads = bench.oracle_sample(wl, 130)   # rounds up to two groups
    assert frac == 1.0 and tg > 0 and tq > 0 and threads >= 1


def test_sample_rows_is_fixed_by_the_workload():
    """Both arms time the same sample: the row count depends on the workload
    only (no timing probe), stays within [8, M], and is a whole number of
    128-token groups for the training step."""
    for name in ("rowwise_4096", "blockwise_1x128_128x128", "grouped_e16"):
        idx, shape_index = bench.WORKLOADS[name]
        wl = W.make_workload(idx, shape_index, scale_down=64)
        r1, r2 = bench.sample_rows(wl), bench.sample_rows(wl)
        assert r1 == r2 and 8 <= r1 <= wl.M


@pytest.mark.timeout(600)
def test_dense_sample_is_a_proportional_slice():
    """Dense recipes: the sample quantizes r rows of A and the matching share
    of B, multiplies r output rows, and reports the rate over that slice."""
    wl = W.make_workload(2, 0, scale_down=128)            # 130 x 40 x 64 blockwise
    tq, tg, frac, threads = bench.oracle_dense_sample(wl, 65)
    assert frac == pytest.approx(65 / wl.M) and tq > 0 and tg > 0 and threads >= 1
    b = bench.cpu_baseline(wl, 65, repeats=2)
    assert b["sample_rows"] == 65 and b["extrapolated"] is True and b["value"] > 0


@pytest.mark.timeout(600)
def test_reference_arm_line_reports_the_steps_it_ran(capsys, monkeypatch):
    """--impl reference on rank 0: the line's ms_per_step is the measured time
    of the sampled steps it ran (so steps x ms_per_step fits the run), with
    the sample marked as extrapolated and its row count stated."""
    import json
    import time
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    t0 = time.perf_counter()
    assert bench.main(["--impl", "reference", "--workload", "tensorwise_256",
                       "--steps", "2", "--warmup", "3"]) == 0
    wall = time.perf_counter() - t0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 2
    assert line["extrapolated"] is True and line["sample_rows"] == 256
    assert line["ms_per_step"] * line["steps"] <= wall * 1e3
    assert line["value"] > 0 and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0
