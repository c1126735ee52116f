"""fp8_quantize_noalloc: the quantize entry point for callers that cannot
allocate device memory (a plugin inside a host application that owns every
device allocation, a service whose memory plan is fixed at start-up).  It
uses the library's own fixed scratch instead of a caller workspace; its
results must equal fp8_quantize's bit for bit -- the quantizer's parity bar --
on two calls in a row (the second call must not see the first call's
leftover scratch).  Collected last on purpose."""
import numpy as np
import pytest
import torch

from fp8_scaled_matrix_b200 import fp8sm
from fp8_scaled_matrix_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _with_workspace(x, recipe):
    q, s = fp8sm.fp8_quantize(x, recipe)
    return q, s


@pytest.mark.parametrize("recipe", [fp8sm.FP8_SCALE_TENSOR, fp8sm.FP8_SCALE_ROW,
                                    fp8sm.FP8_SCALE_BLOCK_1x128,
                                    fp8sm.FP8_SCALE_BLOCK_128x128])
def test_noalloc_matches_workspace_entry_point_twice(recipe):
    g = W.generator(424242 + recipe)
    # first call sees large values, the second small ones: a scratch amax left
    # over from the first call would change the second call's scale
    x1 = (W.randn_bf16((300, 1024), 1.0, g) * 64).to(torch.bfloat16).cuda()
    x2 = W.randn_bf16((300, 1024), 0.02, g).cuda()
    n = fp8sm.scale_count(300, 1024, recipe)
    outs = []
    for x in (x1, x2):
        q = torch.empty(300, 1024, dtype=torch.uint8, device="cuda")
        s = torch.empty(n, dtype=torch.float32, device="cuda")
        fp8sm.fp8_quantize_noalloc(x, recipe, q, s)
        outs.append((q, s))
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    for x, (q, s) in zip((x1, x2), outs):
        qr, sr = _with_workspace(x, recipe)
        torch.cuda.synchronize()
        assert torch.equal(q.cpu(), qr.cpu())
        assert np.array_equal(s.cpu().numpy().view(np.uint32),
                              sr[:n].cpu().numpy().view(np.uint32))


def test_noalloc_rejects_bad_arguments_like_fp8_quantize():
    x = torch.zeros(4, 100, dtype=torch.bfloat16, device="cuda")
    q = torch.empty(4, 100, dtype=torch.uint8, device="cuda")
    s = torch.empty(4, dtype=torch.float32, device="cuda")
    with pytest.raises(fp8sm.Fp8ValueError):
        fp8sm.fp8_quantize_noalloc(x, fp8sm.FP8_SCALE_BLOCK_1x128, q, s)
