"""Quantizer parity: CUDA codes and scales must equal the oracle's bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from fp8_scaled_matrix_b200 import fp8sm
from fp8_scaled_matrix_b200 import workloads as W
from helpers import QUANT_GROUP, codes_np

pytestmark = pytest.mark.gpu

R = {"tensor": fp8sm.FP8_SCALE_TENSOR, "row": fp8sm.FP8_SCALE_ROW,
     "1x128": fp8sm.FP8_SCALE_BLOCK_1x128, "128x128": fp8sm.FP8_SCALE_BLOCK_128x128}


def run_both(x_cpu: torch.Tensor, recipe: str, ld_pad: int = 0):
    rows, cols = x_cpu.shape
    if ld_pad:
        big = torch.zeros(rows, cols + ld_pad, dtype=torch.bfloat16)
        big[:, :cols] = x_cpu
        xd = big.cuda()[:, :cols]
    else:
        xd = x_cpu.cuda()
    q, s = fp8sm.fp8_quantize(xd, R[recipe])
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    qo, so = oracle.quantize(W.bf16_bits(x_cpu), QUANT_GROUP[recipe])
    n = fp8sm.scale_count(rows, cols, R[recipe])
    assert np.array_equal(codes_np(q), qo), f"codes differ ({recipe}, {rows}x{cols})"
    sg = s[:n].cpu().numpy()
    assert np.array_equal(sg.view(np.uint32), so[:n].view(np.uint32)), f"scales differ ({recipe})"


@pytest.mark.parametrize("recipe,rows,cols", [
    ("row", 300, 4104), ("row", 37, 8200), ("row", 5, 8), ("row", 129, 2048),
    ("row", 64, 1000), ("1x128", 301, 384), ("1x128", 7, 1152), ("1x128", 4, 128),
    ("128x128", 300, 640), ("128x128", 128, 128), ("128x128", 1, 256),
    ("tensor", 256, 256), ("tensor", 3000, 1000), ("tensor", 1, 8), ("tensor", 700, 4096),
    # the single-CTA tensorwise path holds up to 8192 8-element vectors
    ("tensor", 64, 1024), ("tensor", 257, 256), ("tensor", 1, 65536),
])
def test_quantize_parity_random(recipe, rows, cols):
    g = W.generator(rows * 7 + cols)
    x = W.randn_bf16((rows, cols), 1.0, g, outlier_frac=0.001, outlier_mult=50.0)
    run_both(x, recipe)


@pytest.mark.parametrize("recipe", ["row", "1x128", "128x128", "tensor"])
def test_quantize_parity_strided_input(recipe):
    g = W.generator(5)
    x = W.randn_bf16((200, 512), 0.02, g)
    run_both(x, recipe, ld_pad=64)


@pytest.mark.parametrize("recipe", ["row", "1x128", "128x128", "tensor"])
def test_quantize_special_values(recipe):
    rows, cols = 130, 256
    x = torch.zeros(rows, cols)
    x[1, :] = -0.0
    x[2, 0] = 448.0
    x[3, :] = 2.0 ** -120                        # bf16-representable tiny values
    x[4, 5] = 1e30                                # huge amax: the rest underflow to zero
    x[4, 6:40] = torch.linspace(-3, 3, 34)
    x[5, :] = torch.arange(cols) * 0.25 - 30.0    # many exact ties
    x[6, :] = float(2 ** 100)
    x[129, :] = -7.0
    run_both(x.to(torch.bfloat16), recipe)


def test_quantize_empty_shapes():
    # rows == 0: nothing written; cols == 0 rowwise: epsilon scales
    x = torch.empty(0, 128, dtype=torch.bfloat16, device="cuda")
    q, s = fp8sm.fp8_quantize(x, fp8sm.FP8_SCALE_ROW)
    x = torch.empty(3, 0, dtype=torch.bfloat16, device="cuda")
    q, s = fp8sm.fp8_quantize(x, fp8sm.FP8_SCALE_ROW)
    torch.cuda.synchronize()
    want = np.float32(oracle.EPS) / np.float32(448)
    assert (s.cpu().numpy() == want).all()
    x = torch.empty(0, 0, dtype=torch.bfloat16, device="cuda")
    q, s = fp8sm.fp8_quantize(x, fp8sm.FP8_SCALE_TENSOR)
    torch.cuda.synchronize()
    assert s.cpu().numpy()[0] == want
    fp8sm.check_device_status()


@pytest.mark.parametrize("idx,shape_index,which", [
    (0, 0, "a"), (0, 0, "b"), (1, 0, "a"), (1, 0, "b"),
    (2, 0, "a"), (2, 0, "b"), (2, 1, "a"), (2, 1, "b"),
    (3, 0, "a"), (3, 0, "b"), (4, 0, "a"),
])
def test_quantize_parity_full_size_workloads(idx, shape_index, which):
    wl = W.make_workload(idx, shape_index)
    recipe = {"tensor": ("tensor", "tensor"), "row": ("row", "row"),
              "1x128_128x128": ("1x128", "128x128"), "1x128_128x1": ("1x128", "1x128"),
              "grouped": ("row", "row")}[wl.recipe][0 if which == "a" else 1]
    x = wl.a if which == "a" else wl.b
    run_both(x, recipe)


def test_quantize_parity_grouped_weights():
    wl = W.make_workload(4)
    w2 = wl.b.reshape(-1, wl.K)          # (E*N, K): rowwise per (expert, channel)
    run_both(w2, "row")


def test_hardware_cast_matches_oracle_encoder_sweep():
    """The cast the kernels use (cvt.rn.satfinite to e4m3) against the oracle's
    bit-level encoder over every bf16 bit pattern scaled by several inverses.
    The inputs go through the rowwise quantizer with amax fixed by a sentinel
    column, so each pattern is cast exactly as in the product path."""
    pats = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = torch.from_numpy(pats.astype(np.int32).astype(np.uint32) << 16).view(torch.float32)
    keep = ~torch.isnan(f) & ~torch.isinf(f)
    vals = f[keep]
    # rows of 255 values + 1 sentinel that sets amax
    for sentinel in (448.0, 1.0, 3.0e5, 2.0 ** -100):
        n = vals.numel()
        per = 255
        rows = (n + per - 1) // per
        x = torch.zeros(rows, per + 1)
        x.view(-1)[:0] = 0
        flat = torch.zeros(rows * per)
        flat[:n] = vals.clamp(-sentinel, sentinel)
        x[:, :per] = flat.view(rows, per)
        x[:, per] = sentinel
        xb = x.to(torch.bfloat16)
        pad = (-xb.shape[1]) % 8
        xb = torch.nn.functional.pad(xb, (0, pad))
        run_both(xb, "row")
