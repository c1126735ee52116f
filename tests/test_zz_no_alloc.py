"""fp8_quantize_noalloc: the quantize entry point for callers that cannot
allocate device memory (a plugin inside a host application that owns every
device allocation, a service whose memory plan is fixed at start-up).  It
uses the library's own fixed scratch instead of a caller workspace; its
results must equal fp8_quantize's bit for bit -- the quantizer's parity bar --
on two calls in a row (the second call must not see the first call's
leftover scratch), and the oracle's quantization of the same input.  Collected
last on purpose."""
import numpy as np
import pytest
import torch

import oracle
from fp8_scaled_matrix_b200 import fp8sm
from fp8_scaled_matrix_b200 import workloads as W

pytestmark = pytest.mark.gpu

ORACLE_GROUP = {fp8sm.FP8_SCALE_TENSOR: oracle.GROUP_TENSOR, fp8sm.FP8_SCALE_ROW: oracle.GROUP_ROW,
                fp8sm.FP8_SCALE_BLOCK_1x128: oracle.GROUP_1x128,
                fp8sm.FP8_SCALE_BLOCK_128x128: oracle.GROUP_128x128}
RECIPES = [fp8sm.FP8_SCALE_TENSOR, fp8sm.FP8_SCALE_ROW, fp8sm.FP8_SCALE_BLOCK_1x128,
           fp8sm.FP8_SCALE_BLOCK_128x128]


def _noalloc(x, recipe, stream=None):
    rows, cols = x.shape
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    s = torch.empty(max(fp8sm.scale_count(rows, cols, recipe), 1), dtype=torch.float32,
                    device="cuda")
    fp8sm.fp8_quantize_noalloc(x, recipe, q, s, stream=stream)
    return q, s


def _check_oracle(x, recipe, q, s):
    """Codes and scales equal the oracle's quantization of the same bf16 input."""
    qo, so = oracle.quantize(W.bf16_bits(x.cpu()), ORACLE_GROUP[recipe])
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s[:so.size].cpu().numpy().view(np.uint32), so.view(np.uint32))


@pytest.mark.parametrize("recipe", RECIPES)
def test_noalloc_matches_workspace_entry_point_twice(recipe):
    g = W.generator(424242 + recipe)
    # first call sees large values, the second small ones: a scratch amax left
    # over from the first call would change the second call's scale
    x1 = (W.randn_bf16((300, 1024), 1.0, g) * 64).to(torch.bfloat16).cuda()
    x2 = W.randn_bf16((300, 1024), 0.02, g).cuda()
    n = fp8sm.scale_count(300, 1024, recipe)
    outs = [_noalloc(x, recipe) for x in (x1, x2)]
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    for x, (q, s) in zip((x1, x2), outs):
        qr, sr = fp8sm.fp8_quantize(x, recipe)
        torch.cuda.synchronize()
        assert torch.equal(q.cpu(), qr.cpu())
        assert np.array_equal(s[:n].cpu().numpy().view(np.uint32),
                              sr[:n].cpu().numpy().view(np.uint32))
        _check_oracle(x, recipe, q, s)


def test_noalloc_empty_tensorwise_after_a_nonempty_call():
    """rows == 0 with the tensorwise recipe still writes one scale (the
    epsilon floor's): the scratch left by a large first call must not leak
    into it."""
    g = W.generator(4243)
    big = (W.randn_bf16((64, 512), 1.0, g) * 100).to(torch.bfloat16).cuda()
    empty = torch.empty(0, 512, dtype=torch.bfloat16, device="cuda")
    q1, s1 = _noalloc(big, fp8sm.FP8_SCALE_TENSOR)
    q2, s2 = _noalloc(empty, fp8sm.FP8_SCALE_TENSOR)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    _check_oracle(big, fp8sm.FP8_SCALE_TENSOR, q1, s1)
    _check_oracle(empty, fp8sm.FP8_SCALE_TENSOR, q2, s2)


@pytest.mark.parametrize("recipe", RECIPES)
def test_noalloc_on_a_side_stream_after_the_default_stream(recipe):
    """A call on a second stream, ordered after a call on the current stream
    (the shared scratch needs the calls ordered), matches the oracle."""
    g = W.generator(4244 + recipe)
    x1 = (W.randn_bf16((257, 768), 1.0, g) * 8).to(torch.bfloat16).cuda()
    x2 = W.randn_bf16((129, 384), 0.5, g).cuda()
    side = torch.cuda.Stream()
    q1, s1 = _noalloc(x1, recipe)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        q2, s2 = _noalloc(x2, recipe, stream=side)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    _check_oracle(x1, recipe, q1, s1)
    _check_oracle(x2, recipe, q2, s2)


@pytest.mark.parametrize("recipe", RECIPES)
def test_noalloc_replayed_from_a_cuda_graph(recipe):
    """The supported capture pattern: a first call outside any capture (it
    looks up the library's scratch), then a call captured in a CUDA graph;
    every replay writes the oracle's codes and scales (the outputs are
    cleared between replays, so a replay that did nothing would fail)."""
    g = W.generator(4245 + recipe)
    x = (W.randn_bf16((384, 512), 1.0, g) * 4).to(torch.bfloat16).cuda()
    _noalloc(x, recipe)
    torch.cuda.synchronize()
    q = torch.empty(384, 512, dtype=torch.uint8, device="cuda")
    s = torch.empty(max(fp8sm.scale_count(384, 512, recipe), 1), dtype=torch.float32,
                    device="cuda")
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        fp8sm.fp8_quantize_noalloc(x, recipe, q, s, stream=stream)
    for _ in range(2):
        q.zero_()
        s.zero_()
        torch.cuda.current_stream().synchronize()
        graph.replay()
        torch.cuda.synchronize()
        fp8sm.check_device_status()
        _check_oracle(x, recipe, q, s)


def test_noalloc_rejects_bad_arguments_like_fp8_quantize():
    x = torch.zeros(4, 100, dtype=torch.bfloat16, device="cuda")
    q = torch.empty(4, 100, dtype=torch.uint8, device="cuda")
    s = torch.empty(4, dtype=torch.float32, device="cuda")
    with pytest.raises(fp8sm.Fp8ValueError):
        fp8sm.fp8_quantize_noalloc(x, fp8sm.FP8_SCALE_BLOCK_1x128, q, s)


def test_noalloc_rejects_outputs_that_are_too_small():
    """The binding refuses caller buffers smaller than what the library
    writes, before any launch."""
    x = torch.zeros(4, 256, dtype=torch.bfloat16, device="cuda")
    ok_q = torch.empty(4, 256, dtype=torch.uint8, device="cuda")
    ok_s = torch.empty(8, dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        fp8sm.fp8_quantize_noalloc(x, fp8sm.FP8_SCALE_BLOCK_1x128, ok_q[:3], ok_s)
    with pytest.raises(ValueError):
        fp8sm.fp8_quantize_noalloc(x, fp8sm.FP8_SCALE_BLOCK_1x128, ok_q, ok_s[:7])
    with pytest.raises(ValueError):
        fp8sm.fp8_quantize_noalloc(x, fp8sm.FP8_SCALE_BLOCK_1x128, ok_q,
                                   ok_s.view(torch.int32))
