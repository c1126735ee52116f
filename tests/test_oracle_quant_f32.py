"""Pins for the oracle's fp32-input quantizer (used to check a GEMM epilogue
that quantizes its fp32 result): the same steps as the bf16 quantizer
("per-token scaling for fp8 linear", Highlights), pinned against torch's own
float8_e4m3fn cast and against the bf16 path on bf16-representable values."""
import numpy as np
import torch

import oracle
from fp8_scaled_matrix_b200 import workloads as W


def torch_cast(y: np.ndarray) -> np.ndarray:
    """torch's RNE float8_e4m3fn cast of fp32 values already in [-448, 448]."""
    return torch.from_numpy(y.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_power_of_two_scale_group_is_torch_cast():
    # one 1x128 group whose amax is exactly 448 * 2: scale 2, inverse 0.5 (exact)
    rng = np.random.default_rng(3)
    x = rng.uniform(-896.0, 896.0, size=(1, 128)).astype(np.float32)
    x[0, 17] = -896.0
    q, s = oracle.quantize_f32(x, oracle.GROUP_1x128)
    assert s.tolist() == [2.0]
    assert np.array_equal(q, torch_cast(x * np.float32(0.5)))


def test_rows_with_unit_scale_are_torch_cast():
    # rowwise groups with amax exactly 448: scale 1, values cast as they are
    rng = np.random.default_rng(4)
    x = rng.standard_normal((4, 96)).astype(np.float32) * 50
    x[:, 5] = 448.0
    q, s = oracle.quantize_f32(x, oracle.GROUP_ROW)
    assert np.array_equal(s, np.ones(4, np.float32))
    assert np.array_equal(q, torch_cast(x))


def test_matches_bf16_path_on_bf16_values():
    g = W.generator(12)
    xb = W.randn_bf16((130, 256), 1.0, g, outlier_frac=0.01, outlier_mult=40.0)
    bits = W.bf16_bits(xb)
    xf = xb.float().numpy()
    for group in (oracle.GROUP_TENSOR, oracle.GROUP_ROW, oracle.GROUP_1x128,
                  oracle.GROUP_128x128):
        q1, s1 = oracle.quantize(bits, group)
        q2, s2 = oracle.quantize_f32(xf, group)
        assert np.array_equal(q1, q2) and np.array_equal(s1.view(np.uint32), s2.view(np.uint32))


def test_epsilon_and_saturation():
    x = np.zeros((2, 128), np.float32)
    x[1, :] = 1e-3
    x[1, 7] = 5.0
    q, s = oracle.quantize_f32(x, oracle.GROUP_1x128)
    assert s[0] == np.float32(np.float32(1e-12) / np.float32(448.0))   # all-zero group
    assert not q[0].any()
    assert q[1, 7] == 0x7E                                             # amax -> +448
