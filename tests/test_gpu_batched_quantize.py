"""Batched quantization of a stack of equal matrices (the (E, N, K) expert
weights of "Add _grouped_mm dispatch handler to Float8Tensor") in one launch:
each matrix's codes and scales equal the oracle's quantization of that
matrix (128x128), or of its transpose (1x128 / 128x128), bit for bit, and
equal the single-matrix entry points' results."""
import numpy as np
import pytest
import torch

import oracle
from fp8_scaled_matrix_b200 import fp8sm
from fp8_scaled_matrix_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,rows,cols", [(1, 128, 128), (3, 200, 256), (5, 256, 384), (16, 128, 1024)])
def test_batched_128x128_matches_oracle(B, rows, cols):
    g = W.generator(B * 100 + rows + cols)
    x = W.randn_bf16((B, rows, cols), 0.02, g, outlier_frac=0.002, outlier_mult=50.0)
    q, s = fp8sm.fp8_quantize_batched(x.cuda(), fp8sm.FP8_SCALE_BLOCK_128x128)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    q, s = q.cpu().numpy(), s.cpu().numpy().reshape(B, -1)
    for e in range(B):
        oq, osc = oracle.quantize(W.bf16_bits(x[e].contiguous()), oracle.GROUP_128x128)
        assert np.array_equal(q[e], oq), f"codes of matrix {e}"
        assert np.array_equal(s[e].view(np.uint32), osc.view(np.uint32)), f"scales of matrix {e}"


@pytest.mark.parametrize("recipe", [fp8sm.FP8_SCALE_BLOCK_1x128, fp8sm.FP8_SCALE_BLOCK_128x128])
@pytest.mark.parametrize("B,rows,cols", [(1, 128, 8), (3, 256, 200), (4, 384, 512)])
def test_batched_transposed_matches_oracle(recipe, B, rows, cols):
    g = W.generator(B * 31 + rows * 7 + cols + recipe)
    x = W.randn_bf16((B, rows, cols), 1.0, g, outlier_frac=0.002, outlier_mult=50.0)
    q, s = fp8sm.fp8_quantize_transposed_batched(x.cuda(), recipe)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    group = oracle.GROUP_1x128 if recipe == fp8sm.FP8_SCALE_BLOCK_1x128 else oracle.GROUP_128x128
    q, s = q.cpu().numpy(), s.cpu().numpy()
    for e in range(B):
        oq, osc = oracle.quantize(np.ascontiguousarray(W.bf16_bits(x[e]).T), group)
        assert np.array_equal(q[e], oq), f"codes of matrix {e}"
        assert np.array_equal(s[e].view(np.uint32), osc.view(np.uint32)), f"scales of matrix {e}"


def test_batched_equals_single_calls_on_the_moe_weights():
    wl = W.make_workload(4, 0)
    w = wl.b.cuda()                                   # (16, 4096, 4096)
    q, s = fp8sm.fp8_quantize_batched(w, fp8sm.FP8_SCALE_BLOCK_128x128)
    qt, st = fp8sm.fp8_quantize_transposed_batched(w, fp8sm.FP8_SCALE_BLOCK_128x128)
    for e in (0, 7, 15):
        q1, s1 = fp8sm.fp8_quantize(w[e], fp8sm.FP8_SCALE_BLOCK_128x128)
        qt1, st1 = fp8sm.fp8_quantize_transposed(w[e], fp8sm.FP8_SCALE_BLOCK_128x128)
        assert torch.equal(q[e], q1) and torch.equal(s[e].reshape(-1), s1.reshape(-1))
        assert torch.equal(qt[e], qt1) and torch.equal(st[e].reshape(-1), st1.reshape(-1))
    torch.cuda.synchronize()
    fp8sm.check_device_status()
