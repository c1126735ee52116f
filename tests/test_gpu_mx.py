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
    (2500, 8192, 8320, True),      # B's codes above 64 MiB: banded tile order
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


# ------------------------------------------------ MXFP8 output (next layer's A)

def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()


def tile_words(M: int, N: int) -> np.ndarray:
    """Byte offsets of (row m, 128-column group j)'s 4 scale bytes in the
    scale-factor tiles of an (M, N) matrix: tile (m / 128, j), byte
    (m % 32) * 16 + (m % 128 / 32) * 4 + (block % 4)."""
    m = np.arange(M)[:, None]
    j = np.arange(N // 128)[None, :]
    return ((m // 128) * (N // 128) + j) * 512 + (m % 32) * 16 + (m % 128 // 32) * 4


def check_mx_output_property(y, q, tiles, what):
    """q, tiles are the MXFP8 quantization of the fp32 y: the oracle's
    fp32-input MXFP8 conversion of the kernel's own fp32 result must give the
    same codes and scale bytes (at each row's place in the scale-factor
    tiles).  Returns the block exponents e (scale 2^e)."""
    M, N = y.shape
    q_want, e8 = oracle.mx_quantize_f32(np.ascontiguousarray(y.astype(np.float32)))
    bad = np.argwhere(q_want != q)
    assert bad.size == 0, f"{what}: {len(bad)} codes differ, first {bad[0]}"
    off = tile_words(M, N)
    got_e = np.stack([tiles[off + k] for k in range(4)], axis=2).reshape(M, N // 32)
    bad = np.argwhere(got_e != e8)
    assert bad.size == 0, f"{what}: {len(bad)} scale bytes differ, first {bad[0]}"
    return e8.astype(np.int64) - 127


@pytest.mark.parametrize("M,N,K,bias", [(128, 256, 128, False), (130, 384, 96, True),
                                        (300, 512, 4096, True), (2048, 4096, 256, False),
                                        (4096, 4096, 256, True)])
def test_mx_output_parity(M, N, K, bias):
    seed = M + N * 3 + K * 7
    qa, ea, qb, eb = mx_operands(M, N, K, seed)
    g = W.generator(seed + 2)
    bb = (torch.randn(N, generator=g) * 0.5).to(torch.bfloat16) if bias else None
    args = (torch.from_numpy(qa).cuda(), torch.from_numpy(qb).cuda(),
            torch.from_numpy(oracle.mx_scales_to_tiles(ea)).cuda(),
            torch.from_numpy(oracle.mx_scales_to_tiles(eb)).cuda())
    bd = None if bb is None else bb.cuda()
    y = fp8sm.fp8_scaled_mm_mx(*args, bias=bd, out_dtype=torch.float32)
    q, tiles = fp8sm.fp8_scaled_mm_mx_quantized(*args, bias=bd)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    y, q, tiles = y.cpu().numpy(), q.cpu().numpy(), tiles.cpu().numpy()
    e = check_mx_output_property(y, q, tiles, f"mx out {M}x{N}x{K}")
    # rows past M in the last tile are written as zero
    if M % 128:
        pad = tile_words(((M + 127) // 128) * 128, N)[M:]
        assert not np.stack([tiles[pad + k] for k in range(4)]).any()
    # against the oracle's fp64 GEMM: GEMM tolerance, plus half an e4m3 step,
    # plus the saturation of the format (a block maximum lands in
    # [256, 512) * 2^e, and values past 448 * 2^e are clamped to it)
    rows = sample_rows(M, 48, seed=seed) if M > 256 else np.arange(M)
    ref, mag = oracle.mx_scaled_mm(qa, qb, ea, eb,
                                   bias_bits=None if bb is None else W.bf16_bits(bb), rows=rows)
    scale = np.ldexp(1.0, e[rows]).repeat(32, axis=1)
    deq = e4m3_decode(q[rows]) * scale
    gemm_tol = 1e-2 * np.abs(ref) + 1e-3 * mag
    clamp = np.maximum(np.abs(ref) + gemm_tol - 448.0 * scale, 0.0)
    tol = gemm_tol + 2.0 ** -4 * (np.abs(ref) + gemm_tol) + scale * 2.0 ** -10 + clamp
    bad = np.argwhere(np.abs(deq - ref) > tol)
    assert bad.size == 0, f"{len(bad)} out of tolerance, first {bad[0]}"


def test_mx_linear_chain_against_oracle():
    """X -> MXFP8 quantize -> GEMM1 with MXFP8 output -> GEMM2 (MXFP8), the
    16640-token layer pair 8192 -> 5120 -> 8192 (the linear-chain workload's
    tensors), sampled rows against the oracle's chain (MX quantize, fp64
    GEMM1 rounded to fp32, MX quantize of it, fp64 GEMM2) and SQNR >= 20 dB
    against the unquantized product."""
    wl = W.make_workload(8)
    f = fp8sm
    x, w1, w2 = wl.a.cuda(), wl.b.cuda(), wl.extra["b2"].cuda()
    qx, sx = f.fp8_quantize_mx(x)
    q1, s1 = f.fp8_quantize_mx(w1)
    q2, s2 = f.fp8_quantize_mx(w2)
    y1q, y1s = f.fp8_scaled_mm_mx_quantized(qx, q1, sx, s1)
    out = f.fp8_scaled_mm_mx(y1q, q2, y1s, s2, out_dtype=torch.float32)
    torch.cuda.synchronize()
    f.check_device_status()
    rows = sample_rows(wl.M, 40, seed=8)
    oqx, oex = oracle.mx_quantize(W.bf16_bits(wl.a))
    oq1, oe1 = oracle.mx_quantize(W.bf16_bits(wl.b))
    oq2, oe2 = oracle.mx_quantize(W.bf16_bits(wl.extra["b2"]))
    y1, _ = oracle.mx_scaled_mm(oqx, oq1, oex, oe1, rows=rows)
    oy1q, oy1e = oracle.mx_quantize_f32(y1.astype(np.float32))
    ref, mag = oracle.mx_scaled_mm(oy1q, oq2, oy1e, oe2)
    got = out.cpu().numpy().astype(np.float64)[rows]
    ok = oracle.within_tolerance(got, ref, mag)
    assert ok.all(), f"chain: {int((~ok).sum())} of {ok.size} out of tolerance"
    exact = (wl.a.double().numpy()[rows] @ wl.b.double().numpy().T) @ \
        wl.extra["b2"].double().numpy().T
    err = got - exact
    assert 10 * np.log10((exact ** 2).sum() / (err ** 2).sum()) >= 20.0
