"""The exchange step of the sharded tensorwise quantization on two gloo ranks
(CPU): each rank holds a row shard of one tensor; after allreduce_amax every
rank holds max |x| of the WHOLE tensor (the one amax the tensorwise recipe's
scale is made of).  The shard maxima are taken on the CPU here (max |x| of
bf16 values is exact in fp32), so the test needs no GPU; the GPU steps around
the exchange are covered by tests/test_gpu_sharded_tensorwise.py."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from fp8_scaled_matrix_b200 import fp8sm
from fp8_scaled_matrix_b200 import workloads as W


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _tensor():
    g = W.generator(77)
    x = W.randn_bf16((96, 64), 1.0, g)
    x[70, 5] = 37.5          # the largest |x| lies in the second shard
    return x


SPLIT = 40                   # rank 0: rows [0, 40), rank 1: rows [40, 96)


def _shard_amax(x: torch.Tensor) -> float:
    return float(x.float().abs().max())


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = _tensor()
        shard = x[:SPLIT] if rank == 0 else x[SPLIT:]
        amax = torch.tensor([_shard_amax(shard)], dtype=torch.float32)
        local = float(amax[0])
        fp8sm.allreduce_amax(amax)
        out[rank] = (local, float(amax[0]))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_allreduce_amax_gives_the_whole_tensors_amax_on_every_rank():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(out)
    whole = float(_tensor().abs().max())
    assert whole == 37.5
    assert res[0][0] < whole and res[1][0] == whole     # the shard maxima differ
    assert res[0][1] == res[1][1] == whole              # after the exchange: the global one


def test_allreduce_amax_without_a_process_group_is_identity():
    assert not dist.is_initialized()
    a = torch.tensor([3.25])
    assert fp8sm.allreduce_amax(a) is a and float(a[0]) == 3.25
