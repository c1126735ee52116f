"""bench.py's multi-rank plumbing on two gloo ranks (CPU): the device time is
the max over ranks, the job throughput counts every rank's work, and the
reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank "measured" a different time; all must agree on the slowest
        ms = bench.max_over_ranks(1.0 + 2.0 * rank, torch.device("cpu"))
        value = bench.job_tflops(1e12, world, ms)
        out[rank] = (ms, value)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for ms, value in res.values():
        assert ms == 3.0                                  # max of 1.0 and 3.0
        assert value == pytest.approx(1e12 * 2 / 3e-3 / 1e12)   # both ranks' work / slowest time


def test_single_rank_is_identity():
    assert not dist.is_initialized()
    assert bench.max_over_ranks(4.25, torch.device("cpu")) == 4.25
    assert bench.job_tflops(2e12, 1, 1.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out == ""   # rank 1 prints nothing and does no work


def test_each_rank_takes_its_own_row_shard():
    """With N ranks, rank r multiplies the activation rows rotated by r * M / N:
    every rank sees all rows (same shape and distribution), no two ranks
    start at the same row, and rank 0 keeps the workload as generated."""
    a = torch.arange(12 * 3, dtype=torch.float32).view(12, 3)
    shards = [bench.rank_shard_rows(a, r, 4) for r in range(4)]
    assert torch.equal(shards[0], a)
    firsts = {int(s[0, 0]) for s in shards}
    assert len(firsts) == 4
    for r, s in enumerate(shards):
        assert s.shape == a.shape
        assert torch.equal(torch.sort(s[:, 0]).values, a[:, 0])   # the same rows, reordered
        assert torch.equal(s[(12 // 4) * r % 12], a[0])
