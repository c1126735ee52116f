"""Sharded tensorwise quantization on the GPU: the two steps around the
ranks' all-reduce(MAX), with the shards of one tensor on one GPU and the
exchange done as a max of the shard results (what the all-reduce computes).
The concatenated shard codes and the common scale must equal the oracle's
tensorwise quantization of the whole tensor bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from fp8_scaled_matrix_b200 import fp8sm
from fp8_scaled_matrix_b200 import workloads as W
from helpers import codes_np

pytestmark = pytest.mark.gpu


def run_shards(x: torch.Tensor, splits):
    """x (rows, cols) CPU bf16, split at the given row offsets."""
    xd = x.cuda()
    bounds = [0] + list(splits) + [x.shape[0]]
    shards = [xd[a:b] for a, b in zip(bounds, bounds[1:])]
    maxima = [fp8sm.fp8_tensor_amax(s) for s in shards]
    amax = torch.stack(maxima).max(dim=0).values.contiguous()
    outs = [fp8sm.fp8_quantize_tensor_with_amax(s, amax) for s in shards]
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    return maxima, amax, outs


@pytest.mark.parametrize("rows,cols,splits", [
    (300, 512, [120]),
    (257, 136, [0, 100, 256]),     # an empty shard and a one-row shard
    (4096, 4096, [1000, 2048, 3001]),
])
def test_sharded_tensorwise_equals_whole_tensor_quantization(rows, cols, splits):
    g = W.generator(rows + cols)
    x = W.randn_bf16((rows, cols), 1.0, g)
    x.view(-1)[int(torch.randint(0, rows * cols, (1,), generator=g))] = -61.0
    maxima, amax, outs = run_shards(x, splits)
    q_want, s_want = oracle.quantize(W.bf16_bits(x), oracle.GROUP_TENSOR)
    q = np.concatenate([codes_np(o[0]) for o in outs])
    assert np.array_equal(q, q_want)
    for _, s in outs:
        assert s.cpu().numpy().view(np.uint32)[0] == s_want.view(np.uint32)[0]
    assert float(amax[0]) == 61.0
    bounds = [0] + list(splits) + [rows]
    for m, (a, b) in zip(maxima, zip(bounds, bounds[1:])):
        want = float(x[a:b].float().abs().max()) if b > a else 0.0
        assert float(m[0]) == want


def test_single_shard_equals_fp8_quantize_tensorwise():
    g = W.generator(5)
    x = W.randn_bf16((512, 768), 1.0, g).cuda()
    q1, s1 = fp8sm.fp8_quantize_tensorwise_sharded(x)     # no process group: one rank
    q2, s2 = fp8sm.fp8_quantize(x, fp8sm.FP8_SCALE_TENSOR)
    torch.cuda.synchronize()
    assert torch.equal(q1.cpu(), q2.cpu())
    assert torch.equal(s1.cpu().view(torch.int32), s2.cpu().view(torch.int32))


def test_all_zero_tensor_takes_the_floor_scale():
    x = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    amax = fp8sm.fp8_tensor_amax(x)
    q, s = fp8sm.fp8_quantize_tensor_with_amax(x, amax)
    torch.cuda.synchronize()
    assert float(amax[0]) == 0.0 and (q.cpu() == 0).all()
    assert s.cpu().numpy()[0] == np.float32(np.float32(1e-12) / np.float32(448.0))
