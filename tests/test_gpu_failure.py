"""Failure detection without a GPU fault: a pipeline wait that nothing will
complete gives up after its limit, the kernel records FP8_ERR_TIMEOUT in the
device status word and returns; the context stays usable."""
import numpy as np
import pytest
import torch

from fp8_scaled_matrix_b200 import fp8sm

pytestmark = pytest.mark.gpu


def test_timeout_probe_reports_status_and_context_survives():
    fp8sm.fp8_get_device_status()             # clear
    fp8sm.fp8_debug_timeout_probe(20000)      # 20 ms limit
    st = fp8sm.fp8_get_device_status()
    assert st == fp8sm.FP8_ERR_TIMEOUT
    assert "site 8" in fp8sm.fp8_last_error()
    # the context is still usable: a normal quantize + GEMM works afterwards
    x = torch.randn(128, 256, device="cuda").to(torch.bfloat16)
    q, s = fp8sm.fp8_quantize(x, fp8sm.FP8_SCALE_ROW)
    out = fp8sm.fp8_scaled_mm(q, q, s, s, fp8sm.FP8_MM_ROW_ROW, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fp8sm.fp8_get_device_status() == fp8sm.FP8_OK
    assert torch.isfinite(out).all()


def test_probe_rejects_bad_limits():
    with pytest.raises(fp8sm.Fp8ValueError):
        fp8sm.fp8_debug_timeout_probe(0)
