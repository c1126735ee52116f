"""MXFP8 (the "mxfp8" recipe of "Add _scaled_mm_v2 API", OCP Microscaling
definition) on the GPU against the oracle.

Quantizer: codes bit-exact against oracle.mx_quantize, scale bytes bit-exact
against oracle.mx_scales_to_tiles of the oracle's scales (padding included).
GEMM: operands and scales from the oracle, output within the GEMM tolerance
|out - ref| <= 1e-2 |ref| + 1e-3 mag of oracle.mx_scaled_mm; plus the full
blockwise-benchmark shapes quantized on the GPU, checked on sampled rows."""
import numpy as np
import pytest
import torch

import oracle
from fp8_scaled_matrix_b200 import fp8sm
from fp8_scaled_matrix_b200 import workloads as W
from helpers import check_gemm, out_f64, sample_rows

pytestmark = pytest.mark.gpu


def blocks_with_range(rows, cols, seed, spread=20):
    """N(0,1) values times a per-32-block power of two in 2^-spread..2^spread,
    one all-zero block and one block of negative zeros."""
    g = W.generator(seed)
    x = torch.randn(rows, cols, generator=g)
    mags = torch.randint(-spread, spread + 1, (rows, cols // 32), generator=g).float()
    x = x * torch.pow(2.0, mags).repeat_interleave(32, dim=1)
    x[0, :32] = 0.0
    if rows > 1:
        x[1, :32] = -0.0
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("rows,cols", [(1, 32), (7, 96), (128, 128), (130, 160), (300, 2048),
                                       (257, 4160), (16, 8192)])
def test_quantize_mx_bit_exact(rows, cols):
    x = blocks_with_range(rows, cols, rows * 7 + cols)
    q, sf = fp8sm.fp8_quantize_mx(x.cuda())
    torch.cuda.synchronize()
    oq, oe = oracle.mx_quantize(W.bf16_bits(x))
    tiles = oracle.mx_scales_to_tiles(oe)
    gq = q.cpu().numpy()
    bad = np.argwhere(gq != oq)
    assert bad.size == 0, f"{len(bad)} codes differ, first {bad[0]}"
    gs = sf.cpu().numpy()
    assert gs.size == tiles.size
    bad = np.flatnonzero(gs != tiles)
    assert bad.size == 0, f"{len(bad)} scale bytes differ, first at {bad[0]}"


def test_quantize_mx_row_stride():
    x = blocks_with_range(70, 256, 5)
    wide = torch.zeros(70, 320, dtype=torch.bfloat16)
    wide[:, :256] = x
    q, sf = fp8sm.fp8_quantize_mx(wide.cuda()[:, :256])
    torch.cuda.synchronize()
    oq, oe = oracle.mx_quantize(W.bf16_bits(x))
    assert np.array_equal(q.cpu().numpy(), oq)
    assert np.array_equal(sf.cpu().numpy(), oracle.mx_scales_to_tiles(oe))


def mx_operands(M, N, K, seed, a_spread=6, b_spread=6):
    a = blocks_with_range(M, K, seed, a_spread)
    b = blocks_with_range(N, K, seed + 1, b_spread)
    qa, ea = oracle.mx_quantize(W.bf16_bits(a))
    qb, eb = oracle.mx_quantize(W.bf16_bits(b))
    return qa, ea, qb, eb


CASES = [
    # M, N, K, bias
    (128, 256, 128, False),
    (1, 16, 32, False),
    (130, 272, 96, True),          # ragged M, N; K not a multiple of 128
    (300, 512, 4096, True),
    (257, 4352, 160, False),       # 17 N tiles, last one half empty
    (2048, 4096, 256, False),      # more tiles than SMs
    (4096, 4096, 256, True),       # last wave split into 128-wide items
]


@pytest.mark.parametrize("M,N,K,bias", CASES)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_mx_gemm_parity(M, N, K, bias, out_dtype):
    seed = M * 3 + N * 5 + K
    qa, ea, qb, eb = mx_operands(M, N, K, seed)
    g = W.generator(seed + 2)
    bb = (torch.randn(N, generator=g) * 0.5).to(torch.bfloat16) if bias else None
    out = fp8sm.fp8_scaled_mm_mx(
        torch.from_numpy(qa).cuda(), torch.from_numpy(qb).cuda(),
        torch.from_numpy(oracle.mx_scales_to_tiles(ea)).cuda(),
        torch.from_numpy(oracle.mx_scales_to_tiles(eb)).cuda(),
        bias=None if bb is None else bb.cuda(), out_dtype=out_dtype)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    rows = sample_rows(M, 64, seed=seed) if M > 256 else None
    ref, mag = oracle.mx_scaled_mm(qa, qb, ea, eb,
                                   bias_bits=None if bb is None else W.bf16_bits(bb), rows=rows)
    got = out_f64(out) if rows is None else out_f64(out)[rows]
    check_gemm(got, ref, mag, f"mx {M}x{N}x{K} {out_dtype}")


def test_mx_gemm_per_block_scales_reach_the_right_rows_and_columns():
    """Every (row, K block) and (column, K block) gets its own power of two
    in 2^-2 .. 2^2.  Each block then contributes at least 2^-8 / 16 of an
    output, so one misplaced scale (a factor of 2 or more on one block's
    term) moves the output by more than 1e-4 relative, far above fp32
    accumulation error."""
    M, N, K = 256, 512, 512
    qa = np.full((M, K), 0x38, np.uint8)    # 1.0
    qb = np.full((N, K), 0x38, np.uint8)
    rng = np.random.default_rng(9)
    ea = rng.integers(125, 130, (M, K // 32)).astype(np.uint8)
    eb = rng.integers(125, 130, (N, K // 32)).astype(np.uint8)
    out = fp8sm.fp8_scaled_mm_mx(
        torch.from_numpy(qa).cuda(), torch.from_numpy(qb).cuda(),
        torch.from_numpy(oracle.mx_scales_to_tiles(ea)).cuda(),
        torch.from_numpy(oracle.mx_scales_to_tiles(eb)).cuda(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref, mag = oracle.mx_scaled_mm(qa, qb, ea, eb)
    got = out_f64(out)
    bad = np.argwhere(np.abs(got - ref) > 1e-5 * np.abs(ref))
    assert bad.size == 0, f"{len(bad)} wrong, first {bad[0]}: {got[tuple(bad[0])]} vs {ref[tuple(bad[0])]}"


@pytest.mark.parametrize("shape_index", [0, 1])
def test_mx_end_to_end_full_size_sampled(shape_index):
    """The blockwise benchmark's shapes (16640 x {5120, 8192} x {8192, 5120}),
    quantized on the GPU (MXFP8) and multiplied; sampled rows against the
    oracle's quantize + GEMM of the same inputs, and SQNR against the
    unquantized product (>= 20 dB)."""
    wl = W.make_workload(2, shape_index)
    a, b = wl.a.cuda(), wl.b.cuda()
    qa, sa = fp8sm.fp8_quantize_mx(a)
    qb, sb = fp8sm.fp8_quantize_mx(b)
    out = fp8sm.fp8_scaled_mm_mx(qa, qb, sa, sb)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    rows = sample_rows(wl.M, 40, seed=shape_index)
    oqa, oea = oracle.mx_quantize(W.bf16_bits(wl.a))
    oqb, oeb = oracle.mx_quantize(W.bf16_bits(wl.b))
    ref, mag = oracle.mx_scaled_mm(oqa, oqb, oea, oeb, rows=rows)
    got = out_f64(out)[rows]
    check_gemm(got, ref, mag, f"mx full size {shape_index}")
    exact = wl.a.double().numpy()[rows] @ wl.b.double().numpy().T
    err = got - exact
    assert 10 * np.log10((exact ** 2).sum() / (err ** 2).sum()) >= 20.0
