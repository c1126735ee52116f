"""Scaled-GEMM parity against the oracle, per element:
|out - ref| <= 1e-2 |ref| + 1e-3 sum_k |a_k b_k| (scaled), on fp32 output and
on bf16 output.  Operands and scales come from the oracle's quantizer (so the
GEMM is tested on its own); the end-to-end tests quantize on the GPU."""
import numpy as np
import pytest
import torch

import oracle
from fp8_scaled_matrix_b200 import fp8sm
from fp8_scaled_matrix_b200 import workloads as W
from helpers import MM, OPERAND_GROUPS, QUANT_GROUP, check_gemm, codes_np, out_f64, sample_rows

pytestmark = pytest.mark.gpu

MMR = {"tensor": fp8sm.FP8_MM_TENSOR_TENSOR, "row": fp8sm.FP8_MM_ROW_ROW,
       "1x128_128x128": fp8sm.FP8_MM_1x128_128x128, "1x128_128x1": fp8sm.FP8_MM_1x128_128x1}
QR = {"tensor": fp8sm.FP8_SCALE_TENSOR, "row": fp8sm.FP8_SCALE_ROW,
      "1x128": fp8sm.FP8_SCALE_BLOCK_1x128, "128x128": fp8sm.FP8_SCALE_BLOCK_128x128}


def oracle_operands(wl):
    ga, gb = OPERAND_GROUPS[wl.recipe]
    qa, sa = oracle.quantize(W.bf16_bits(wl.a), QUANT_GROUP[ga])
    qb, sb = oracle.quantize(W.bf16_bits(wl.b), QUANT_GROUP[gb])
    return qa, sa, qb, sb


def gpu_gemm(qa, sa, qb, sb, recipe, bias, out_dtype):
    a = torch.from_numpy(qa).cuda()
    b = torch.from_numpy(qb).cuda()
    sad = torch.from_numpy(sa).cuda()
    sbd = torch.from_numpy(sb).cuda()
    bd = None if bias is None else bias.cuda()
    out = fp8sm.fp8_scaled_mm(a, b, sad, sbd, MMR[recipe], bias=bd, out_dtype=out_dtype)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    return out


CASES = [
    # recipe, M, N, K, bias
    ("tensor", 256, 256, 256, False),
    ("tensor", 1, 16, 16, False),
    ("tensor", 300, 272, 528, True),
    ("row", 300, 272, 528, True),
    ("row", 129, 512, 4096, True),
    ("row", 2048, 4096, 256, False),         # 256 tiles > SM count: persistent loop
    ("row", 4096, 4096, 256, True),          # 512 tiles: last wave split into 128-wide items
    ("row", 7, 48, 32, True),
    ("1x128_128x128", 260, 400, 384, False),
    ("1x128_128x128", 128, 256, 128, True),
    ("1x128_128x128", 1100, 2304, 1024, False),   # 81 tiles, 8 K blocks
    ("1x128_128x1", 130, 528, 256, False),
    ("1x128_128x1", 64, 16, 128, True),
    ("1x128_128x1", 2304, 4352, 512, False),       # 306 tiles: persistent loop
]


@pytest.mark.parametrize("recipe,M,N,K,bias", CASES)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_parity(recipe, M, N, K, bias, out_dtype):
    b_std = 0.02 if recipe != "1x128_128x1" else 1.0
    a_std = 1.0 if recipe != "1x128_128x1" else 1e-3
    wl = W.small_case(recipe, M, N, K, seed=M * 31 + N * 7 + K, a_std=a_std, b_std=b_std,
                      bias=bias)
    qa, sa, qb, sb = oracle_operands(wl)
    bias_bits = None if wl.bias is None else W.bf16_bits(wl.bias)
    out = gpu_gemm(qa, sa, qb, sb, recipe, wl.bias, out_dtype)
    ref, mag = oracle.scaled_mm(qa, qb, sa, sb, MM[recipe], bias_bits=bias_bits)
    check_gemm(out_f64(out), ref, mag, f"{recipe} {M}x{N}x{K} {out_dtype}")


@pytest.mark.parametrize("recipe", ["tensor", "row", "1x128_128x128", "1x128_128x1"])
def test_gemm_k_zero_writes_bias(recipe):
    if recipe.startswith("1x128"):
        pytest.skip("blockwise needs K % 128 == 0; K == 0 is covered by the dense recipes")
    M, N = 5, 32
    bias = torch.randn(N, generator=W.generator(3)).to(torch.bfloat16)
    a = torch.empty(M, 0, dtype=torch.uint8, device="cuda")
    b = torch.empty(N, 0, dtype=torch.uint8, device="cuda")
    s = torch.ones(max(M, N), device="cuda")
    out = fp8sm.fp8_scaled_mm(a, b, s, s, MMR[recipe], bias=bias.cuda(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    want = bias.double().numpy()[None, :].repeat(M, 0)
    assert np.array_equal(out_f64(out), want)


def test_gemm_integer_exact():
    """Integer-valued e4m3 inputs with power-of-two scales: exact in fp32."""
    rng = np.random.default_rng(1)
    av = rng.integers(-8, 9, size=(256, 512)).astype(np.float32)
    bv = rng.integers(-8, 9, size=(256, 512)).astype(np.float32)
    qa = torch.from_numpy(av).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    qb = torch.from_numpy(bv).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    out = gpu_gemm(qa, np.array([0.5], np.float32), qb, np.array([0.25], np.float32),
                   "tensor", None, torch.float32)
    want = (av.astype(np.int64) @ bv.astype(np.int64).T) * 0.125
    assert np.array_equal(out_f64(out), want.astype(np.float64))


FULL = [(1, 0), (2, 0), (2, 1), (3, 0), (3, 1), (0, 0)]


@pytest.mark.parametrize("idx,shape_index", FULL)
def test_end_to_end_full_size_sampled(idx, shape_index):
    """Full-size workload, launched as bench.py does: GPU quantize of both
    operands then the GEMM (bf16 out).  Checked on sampled rows (tile edges +
    random) against the oracle's quantize + GEMM of the same inputs."""
    wl = W.make_workload(idx, shape_index)
    ga, gb = OPERAND_GROUPS[wl.recipe]
    a, b = wl.a.cuda(), wl.b.cuda()
    qa, sa = fp8sm.fp8_quantize(a, QR[ga])
    qb, sb = fp8sm.fp8_quantize(b, QR[gb])
    bias = None if wl.bias is None else wl.bias.cuda()
    out = fp8sm.fp8_scaled_mm(qa, qb, sa, sb, MMR[wl.recipe], bias=bias)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    rows = sample_rows(wl.M, 40, seed=idx)
    oqa, osa = oracle.quantize(W.bf16_bits(wl.a), QUANT_GROUP[ga])
    oqb, osb = oracle.quantize(W.bf16_bits(wl.b), QUANT_GROUP[gb])
    bias_bits = None if wl.bias is None else W.bf16_bits(wl.bias)
    ref, mag = oracle.scaled_mm(oqa, oqb, osa, osb, MM[wl.recipe], bias_bits=bias_bits, rows=rows)
    got = out_f64(out)[rows]
    check_gemm(got, ref, mag, f"{wl.name} full size")
    # SQNR of the FP8 path against the unquantized product on the same rows
    # (quality check from the MoE handler's tests: output >= 20 dB)
    af = wl.a.double().numpy()[rows]
    bf = wl.b.double().numpy()
    exact = af @ bf.T + (0 if wl.bias is None else wl.bias.double().numpy()[None, :])
    err = got - exact
    sqnr = 10 * np.log10((exact ** 2).sum() / (err ** 2).sum())
    assert sqnr >= 20.0, sqnr


@pytest.mark.parametrize("recipe", ["row", "tensor", "1x128_128x128", "1x128_128x1"])
def test_gemm_banded_tile_order_large_b(recipe):
    """B's codes above 64 MiB (N = 8192, K = 8320): the dense kernels take
    their tiles in bands of 16 M tiles, N-major inside a band.  M = 2500 gives
    20 M tiles of 128 rows (a full band and a partial one).  Sampled rows of
    every band, fp32 output, against the oracle."""
    M, N, K = 2500, 8192, 8320
    b_std = 0.02 if recipe != "1x128_128x1" else 1.0
    a_std = 1.0 if recipe != "1x128_128x1" else 1e-3
    wl = W.small_case(recipe, M, N, K, seed=907 + len(recipe), a_std=a_std, b_std=b_std,
                      bias=recipe == "row")
    qa, sa, qb, sb = oracle_operands(wl)
    out = gpu_gemm(qa, sa, qb, sb, recipe, wl.bias, torch.float32)
    rows = sample_rows(M, 24, seed=7)
    bias_bits = None if wl.bias is None else W.bf16_bits(wl.bias)
    ref, mag = oracle.scaled_mm(qa, qb, sa, sb, MM[recipe], bias_bits=bias_bits, rows=rows)
    check_gemm(out_f64(out)[rows], ref, mag, f"{recipe} banded order")
