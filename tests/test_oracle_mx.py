"""Pins for the oracle's MXFP8 functions ("mxfp8" recipe of "Add _scaled_mm_v2
API", defined by the OCP Microscaling specification: E8M0 power-of-two scale
per 32 elements along K, E4M3 elements).

The quantizer is pinned by hand-worked blocks, by the characterisation of the
shared exponent (the block maximum lands in [256, 512) once divided by the
scale, unless the E8M0 range clamps it), and by torch's own float8_e4m3fn cast
of the exactly scaled block.  The GEMM is pinned by closed forms, by exact
rational brute force, and by torch-decoded dequantize-then-matmul in fp64.
The scale-factor tile layout is pinned by worked positions and by being a
bijection onto the tile bytes."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from fp8_scaled_matrix_b200 import workloads as W


def bf16_bits(vals) -> np.ndarray:
    t = torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def torch_decode(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()


def test_handworked_blocks():
    # block 0: amax 1.0 -> e = 0 - 8 = -8 (byte 119); 1.0 * 2^8 = 256 -> 0x78,
    #          0.5 -> 128 = 0x70, -0.25 -> -64 = 0xE8 (E = 6 + 7)
    # block 1: amax 448 -> e = 8 - 8 = 0 (byte 127); 448 -> 0x7E, 1 -> 0x38
    # block 2: amax 480 (in [256, 512) * 2^0) -> e = 0; 480 saturates to 448
    # block 3: all zero -> e = -127 (byte 0); -0.0 keeps its sign (0x80)
    row = np.zeros(128, np.float32)
    row[0], row[1], row[2] = 1.0, 0.5, -0.25
    row[32], row[33] = 448.0, 1.0
    row[64], row[65] = 480.0, -480.0
    row[97] = -0.0
    q, e8 = oracle.mx_quantize(bf16_bits(row[None, :]))
    assert e8.tolist() == [[119, 127, 127, 0]]
    assert q[0, :3].tolist() == [0x78, 0x70, 0xE8]
    assert q[0, 32:34].tolist() == [0x7E, 0x38]
    assert q[0, 64:66].tolist() == [0x7E, 0xFE]
    assert q[0, 96] == 0x00 and q[0, 97] == 0x80


def test_tiny_block_clamps_exponent():
    # the smallest bf16 subnormal, 2^-133: floor(log2) - 8 = -141 clamps to
    # -127, so the element becomes 2^-133 * 2^127 = 2^-6 (code 0x08)
    bits = np.zeros((1, 32), np.uint16)
    bits[0, 3] = 0x0001
    q, e8 = oracle.mx_quantize(bits)
    assert e8[0, 0] == 0 and q[0, 3] == 0x08 and not np.delete(q[0], 3).any()


def _random_blocks(rows, cols, seed):
    g = W.generator(seed)
    x = torch.randn(rows, cols, generator=g)
    # per-block magnitudes spread over 2^-40 .. 2^40, some zero blocks
    mags = torch.randint(-40, 41, (rows, cols // 32), generator=g).float()
    x = x * torch.pow(2.0, mags).repeat_interleave(32, dim=1)
    x[0, :32] = 0.0
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("rows,cols,seed", [(7, 96, 1), (33, 256, 2), (130, 64, 3)])
def test_quantize_against_torch_cast(rows, cols, seed):
    xb = _random_blocks(rows, cols, seed)
    q, e8 = oracle.mx_quantize(W.bf16_bits(xb))
    x = xb.double().numpy().reshape(rows, cols // 32, 32)
    amax = np.abs(x).max(axis=2)
    e = e8.astype(np.int64) - 127
    nz = amax > 0
    clamped = e == -127
    # the block maximum divided by 2^e lies in [256, 512) unless clamped
    scaled = amax / np.ldexp(1.0, e)
    ok = (scaled >= 256) & (scaled < 512)
    assert (ok | (nz & clamped & (scaled < 256)) | (~nz & clamped)).all()
    # the codes are torch's RNE e4m3 cast of the exactly scaled values,
    # saturated to +-448
    y = np.clip(x / np.ldexp(1.0, e)[:, :, None], -448, 448).astype(np.float32)
    want = torch.from_numpy(y.reshape(rows, cols)).to(torch.float8_e4m3fn)
    assert np.array_equal(q, want.view(torch.uint8).numpy())


def test_quantize_rejects_ragged_blocks():
    with pytest.raises(ValueError):
        oracle.mx_quantize(np.zeros((2, 48), np.uint16))


def test_gemm_closed_forms():
    K = 96
    a = np.full((3, K), 0x38, np.uint8)        # 1.0
    b = np.full((2, K), 0x38, np.uint8)
    ea = np.full((3, K // 32), 127, np.uint8)  # 2^0
    eb = np.full((2, K // 32), 127, np.uint8)
    ref, mag = oracle.mx_scaled_mm(a, b, ea, eb)
    assert (ref == K).all() and (mag == K).all()
    ea[1, :] = 130                             # row 1: 2^3
    eb[0, 1] = 125                             # column 0, middle block: 2^-2
    ref, _ = oracle.mx_scaled_mm(a, b, ea, eb, bias_bits=bf16_bits([0.5, -2.0]))
    assert ref[0].tolist() == [32 + 8 + 32 + 0.5, 96 - 2.0]
    assert ref[1].tolist() == [8 * (32 + 8 + 32) + 0.5, 8 * 96 - 2.0]


def test_gemm_brute_force_fractions():
    rng = np.random.default_rng(5)
    M, N, K = 2, 3, 64
    a = rng.integers(0, 256, (M, K), dtype=np.uint8)
    b = rng.integers(0, 256, (N, K), dtype=np.uint8)
    a[(a & 0x7F) == 0x7F] = 0x11    # no NaN codes
    b[(b & 0x7F) == 0x7F] = 0x22
    ea = rng.integers(100, 150, (M, K // 32), dtype=np.uint8)
    eb = rng.integers(100, 150, (N, K // 32), dtype=np.uint8)
    ref, _ = oracle.mx_scaled_mm(a, b, ea, eb)

    def val(c):
        s = -1 if c & 0x80 else 1
        E, m = (c >> 3) & 0xF, c & 7
        return s * (Fraction(m, 8) * Fraction(1, 64) if E == 0
                    else (1 + Fraction(m, 8)) * Fraction(2) ** (E - 7))
    for i in range(M):
        for j in range(N):
            exact = sum(val(int(a[i, k])) * Fraction(2) ** (int(ea[i, k // 32]) - 127)
                        * val(int(b[j, k])) * Fraction(2) ** (int(eb[j, k // 32]) - 127)
                        for k in range(K))
            assert ref[i, j] == float(exact)


def test_gemm_dequantize_then_matmul():
    xa = _random_blocks(40, 160, 7)
    xb = _random_blocks(24, 160, 8)
    qa, ea = oracle.mx_quantize(W.bf16_bits(xa))
    qb, eb = oracle.mx_quantize(W.bf16_bits(xb))
    da = torch_decode(qa) * np.ldexp(1.0, ea.astype(np.int64) - 127).repeat(32, axis=1)
    db = torch_decode(qb) * np.ldexp(1.0, eb.astype(np.int64) - 127).repeat(32, axis=1)
    want = da @ db.T
    ref, mag = oracle.mx_scaled_mm(qa, qb, ea, eb)
    assert np.allclose(ref, want, rtol=1e-12, atol=1e-12 * mag.max())
    assert (mag >= np.abs(ref) * (1 - 1e-12)).all()
    rows = np.array([39, 0, 17])
    ref_r, _ = oracle.mx_scaled_mm(qa, qb, ea, eb, rows=rows)
    assert np.array_equal(ref_r, ref[rows])


def test_scale_tiles_worked_positions():
    rows, kb = 130, 6                       # 2 row tiles x 2 K tiles
    e8 = np.arange(rows * kb, dtype=np.int64).reshape(rows, kb) % 251 + 1
    t = oracle.mx_scales_to_tiles(e8.astype(np.uint8))
    assert t.size == 2 * 2 * 512
    KT = 2

    def at(r, k):
        return int(t[((r // 128) * KT + k // 4) * 512 + (r % 128 % 32) * 16
                     + (r % 128 // 32) * 4 + k % 4])
    assert t[0] == e8[0, 0] and t[16] == e8[1, 0] and t[4] == e8[32, 0]
    assert t[23] == e8[33, 3] and t[512] == e8[0, 4] and t[1024] == e8[128, 0]
    assert t[1024 + 16 + 512 + 1] == e8[129, 5]
    for r in range(rows):
        for k in range(kb):
            assert at(r, k) == e8[r, k]
    # every byte of the tiles is either one scale or zero padding
    assert (t != 0).sum() == rows * kb


def test_scale_tiles_is_a_bijection():
    rows, kb = 256, 8
    e8 = np.zeros((rows, kb), np.uint8)
    seen = set()
    for r in range(rows):
        for k in range(kb):
            e8[:] = 0
            e8[r, k] = 1
            pos = int(np.flatnonzero(oracle.mx_scales_to_tiles(e8))[0])
            assert pos not in seen
            seen.add(pos)
    assert len(seen) == rows * kb == oracle.mx_tile_bytes(rows, kb)


def test_quantize_f32_matches_bf16_path_on_bf16_values():
    xb = _random_blocks(45, 192, 11)
    q1, e1 = oracle.mx_quantize(W.bf16_bits(xb))
    q2, e2 = oracle.mx_quantize_f32(xb.float().numpy())
    assert np.array_equal(q1, q2) and np.array_equal(e1, e2)


def test_quantize_f32_against_torch_cast():
    # fp32 values with full 24-bit significands, spread over 2^-60 .. 2^60
    rng = np.random.default_rng(12)
    x = rng.standard_normal((20, 256)) * np.exp2(rng.integers(-60, 61, (20, 8))).repeat(32, axis=1)
    x = x.astype(np.float32)
    x[3, 64:96] = 0.0
    x[4, 5] = np.float32(2.0 ** -140)                 # a subnormal block maximum
    x[4, 0:5] = 0.0
    x[4, 6:32] = 0.0
    q, e8 = oracle.mx_quantize_f32(x)
    e = e8.astype(np.int64) - 127
    amax = np.abs(x.astype(np.float64)).reshape(20, 8, 32).max(axis=2)
    scaled = amax / np.ldexp(1.0, e)
    assert (((scaled >= 256) & (scaled < 512)) | (e == -127)).all()
    assert e8[4, 0] == 0 and e8[3, 2] == 0
    y = np.clip(x.astype(np.float64).reshape(20, 8, 32) / np.ldexp(1.0, e)[:, :, None], -448, 448)
    want = torch.from_numpy(y.reshape(20, 256).astype(np.float32)).to(torch.float8_e4m3fn)
    assert np.array_equal(q, want.view(torch.uint8).numpy())
