"""Pins for the oracle's scaled GEMM (dense recipes and grouped).

Pinned against:
  * hand-worked outputs (tests/golden/gemm_handworked.json) for every recipe,
    including the K-block-major scale layouts and an empty expert group;
  * brute force with exact rationals (Python Fractions on values decoded by
    torch's own float8_e4m3fn conversion) on tiny random shapes;
  * the identity scaled-mm == dequantize-then-matmul, computed a second way
    with numpy on torch-decoded operands;
  * exact integer results when scales are powers of two;
  * the grouped oracle equals the dense rowwise oracle applied group by group.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from fp8_scaled_matrix_b200 import workloads as W


def _codes(lst):
    return np.array([[int(c, 16) for c in row] for row in lst], dtype=np.uint8)


def _bf16_bits(vals):
    return W.bf16_bits(torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16))


def _encode_values(vals):
    """e4m3 codes for values that are exactly representable (torch's cast)."""
    t = torch.tensor(vals, dtype=torch.float32)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _decode_torch(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()


def test_handworked_dense(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "gemm_handworked.json")))["dense"]
    a, b = _codes(fx["a_codes"]), _codes(fx["b_codes"])
    assert np.array_equal(_decode_torch(a), np.array(fx["a_values"], dtype=np.float64))
    assert np.array_equal(_decode_torch(b), np.array(fx["b_values"], dtype=np.float64))
    rw = fx["rowwise"]
    ref, mag = oracle.scaled_mm(a, b, rw["sA"], rw["sB"], oracle.MM_ROW_ROW,
                                bias_bits=_bf16_bits(rw["bias"]))
    assert np.array_equal(ref, np.array(rw["out"]))
    assert np.array_equal(mag, np.array(rw["mag"]))
    tw = fx["tensorwise"]
    ref, _ = oracle.scaled_mm(a, b, tw["sA"], tw["sB"], oracle.MM_TENSOR_TENSOR)
    assert np.array_equal(ref, np.array(tw["out"]))


def test_handworked_blockwise(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "gemm_handworked.json")))["blockwise"]
    a = np.concatenate([np.full(128, 0x38), np.full(128, 0x40)]).astype(np.uint8)[None, :]
    b0 = np.concatenate([np.full(128, 0x30), np.full(128, 0x28)])
    b1 = np.full(256, 0x38)
    b = np.stack([b0, b1]).astype(np.uint8)
    sA = [2.0, 0.5]
    r = fx["1x128_128x128"]
    ref, _ = oracle.scaled_mm(a, b, sA, r["sB"], oracle.MM_1x128_128x128)
    assert np.array_equal(ref, np.array(r["out"]))
    r = fx["1x128_128x1"]
    ref, _ = oracle.scaled_mm(a, b, sA, r["sB"], oracle.MM_1x128_128x1)
    assert np.array_equal(ref, np.array(r["out"]))


def test_handworked_grouped(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "gemm_handworked.json")))["grouped"]
    a = _encode_values(fx["a_values"])
    b = _encode_values(fx["b_values"])
    ref, _ = oracle.grouped_scaled_mm(a, b, fx["sA"], np.array(fx["sB"]), fx["offs"])
    assert np.array_equal(ref, np.array(fx["out"]))
    # same result with an empty expert inserted in the middle
    b3 = np.stack([b[0], np.full_like(b[0], 0x7E), b[1]])
    sB3 = np.stack([np.array(fx["sB"][0]), np.array([1e6, 1e6]), np.array(fx["sB"][1])])
    ref3, _ = oracle.grouped_scaled_mm(a, b3, fx["sA"], sB3,
                                       fx["empty_group_variant"]["offs"])
    assert np.array_equal(ref3, np.array(fx["out"]))


def _random_codes(shape, seed):
    g = W.generator(seed)
    x = W.randn_bf16(shape, 1.0, g, outlier_frac=0.02, outlier_mult=30.0)
    q, _ = oracle.quantize(W.bf16_bits(x), oracle.GROUP_TENSOR)
    return q


def _scales(recipe, M, N, K, seed):
    rng = np.random.default_rng(seed)
    KB = K // 128 if K % 128 == 0 else 1
    if recipe == oracle.MM_TENSOR_TENSOR:
        return rng.uniform(0.01, 2, 1).astype(np.float32), rng.uniform(0.01, 2, 1).astype(np.float32)
    if recipe == oracle.MM_ROW_ROW:
        return rng.uniform(0.01, 2, M).astype(np.float32), rng.uniform(0.01, 2, N).astype(np.float32)
    sA = rng.uniform(0.01, 2, KB * M).astype(np.float32)
    if recipe == oracle.MM_1x128_128x128:
        return sA, rng.uniform(0.01, 2, KB * ((N + 127) // 128)).astype(np.float32)
    return sA, rng.uniform(0.01, 2, KB * N).astype(np.float32)


def _fraction_scale(recipe, sA, sB, M, N, m, n, kb):
    if recipe == oracle.MM_TENSOR_TENSOR:
        return Fraction(float(sA[0])) * Fraction(float(sB[0]))
    if recipe == oracle.MM_ROW_ROW:
        return Fraction(float(sA[m])) * Fraction(float(sB[n]))
    sa = Fraction(float(sA[kb * M + m]))
    if recipe == oracle.MM_1x128_128x128:
        return sa * Fraction(float(sB[kb * ((N + 127) // 128) + n // 128]))
    return sa * Fraction(float(sB[kb * N + n]))


@pytest.mark.parametrize("recipe,M,N,K", [
    (oracle.MM_TENSOR_TENSOR, 3, 4, 48),
    (oracle.MM_ROW_ROW, 4, 3, 80),
    (oracle.MM_1x128_128x128, 3, 130, 256),
    (oracle.MM_1x128_128x1, 2, 5, 384),
])
def test_brute_force_fractions(recipe, M, N, K):
    a = _random_codes((M, K), 11 + recipe)
    b = _random_codes((N, K), 21 + recipe)
    sA, sB = _scales(recipe, M, N, K, 31 + recipe)
    bias = _bf16_bits(np.random.default_rng(5).normal(0, 1, N).tolist())
    ref, mag = oracle.scaled_mm(a, b, sA, sB, recipe, bias_bits=bias)
    ad, bd = _decode_torch(a), _decode_torch(b)
    bias_f = torch.from_numpy(bias.view(np.int16)).view(torch.bfloat16).double().numpy()
    for m in range(M):
        for n in (range(N) if N < 10 else [0, 1, 127, 128, 129]):
            exact = Fraction(0)
            exact_mag = Fraction(0)
            for k in range(K):
                s = _fraction_scale(recipe, sA, sB, M, N, m, n, k // 128)
                p = Fraction(float(ad[m, k])) * Fraction(float(bd[n, k]))
                exact += s * p
                exact_mag += abs(s) * abs(p)
            exact += Fraction(float(bias_f[n]))
            assert abs(ref[m, n] - float(exact)) <= 1e-13 * float(exact_mag + abs(Fraction(float(bias_f[n])))) + 1e-300
            assert abs(mag[m, n] - float(exact_mag)) <= 1e-13 * float(exact_mag)


@pytest.mark.parametrize("recipe", [0, 1, 2, 3])
def test_identity_dequantize_then_matmul(recipe):
    M, N, K = 9, 140, 256
    a = _random_codes((M, K), 41)
    b = _random_codes((N, K), 42)
    sA, sB = _scales(recipe, M, N, K, 43)
    bias = _bf16_bits(np.random.default_rng(6).normal(0, 1, N).tolist())
    ref, mag = oracle.scaled_mm(a, b, sA, sB, recipe, bias_bits=bias)
    # second path inside the oracle
    ref2 = oracle.dequant_then_matmul(a, b, sA, sB, recipe, bias_bits=bias)
    # third path: numpy on torch-decoded operands, scales broadcast by hand
    ad, bd = _decode_torch(a), _decode_torch(b)
    KB = K // 128
    kidx = np.arange(K) // 128
    if recipe == 0:
        A = ad * float(sA[0]); B = bd * float(sB[0])
    elif recipe == 1:
        A = ad * sA.astype(np.float64)[:, None]; B = bd * sB.astype(np.float64)[:, None]
    else:
        A = ad * sA.astype(np.float64).reshape(KB, M).T[:, kidx]
        if recipe == 2:
            sBm = sB.astype(np.float64).reshape(KB, (N + 127) // 128).T[np.arange(N) // 128]
        else:
            sBm = sB.astype(np.float64).reshape(KB, N).T
        B = bd * sBm[:, kidx]
    bias_f = torch.from_numpy(bias.view(np.int16)).view(torch.bfloat16).double().numpy()
    ref3 = A @ B.T + bias_f[None, :]
    tol = 1e-12 * (mag + np.abs(bias_f)[None, :]) + 1e-300
    assert (np.abs(ref - ref2) <= tol).all()
    assert (np.abs(ref - ref3) <= tol).all()


def test_power_of_two_scales_give_exact_integers():
    # integer-valued e4m3 inputs (0..16) and power-of-two scales: exact result
    rng = np.random.default_rng(3)
    av = rng.integers(-16, 17, size=(5, 256)).astype(np.float32)
    bv = rng.integers(-16, 17, size=(6, 256)).astype(np.float32)
    a, b = _encode_values(av), _encode_values(bv)
    ref, _ = oracle.scaled_mm(a, b, [0.5], [4.0], oracle.MM_TENSOR_TENSOR)
    want = 2.0 * (av.astype(np.int64) @ bv.astype(np.int64).T)
    assert np.array_equal(ref, want.astype(np.float64))


def test_grouped_equals_dense_per_group():
    E, N, K = 4, 40, 96
    sizes = [5, 0, 17, 10]
    M = sum(sizes)
    a = _random_codes((M, K), 51)
    b = np.stack([_random_codes((N, K), 52 + e) for e in range(E)])
    rng = np.random.default_rng(9)
    sA = rng.uniform(0.1, 2, M).astype(np.float32)
    sB = rng.uniform(0.1, 2, (E, N)).astype(np.float32)
    offs = np.cumsum(sizes).astype(np.int32)
    ref, mag = oracle.grouped_scaled_mm(a, b, sA, sB, offs)
    start = 0
    for e, sz in enumerate(sizes):
        if sz:
            r, m = oracle.scaled_mm(a[start:start + sz], b[e], sA[start:start + sz], sB[e],
                                    oracle.MM_ROW_ROW)
            assert np.array_equal(ref[start:start + sz], r)
            assert np.array_equal(mag[start:start + sz], m)
        start += sz
    # row subset gives the same rows
    rows = np.array([0, 4, 5, 21, 31], dtype=np.int64)
    rs, ms = oracle.grouped_scaled_mm(a, b, sA, sB, offs, rows=rows)
    assert np.array_equal(rs, ref[rows])


def test_grouped_rejects_malformed_offs():
    a = np.zeros((4, 16), dtype=np.uint8)
    b = np.zeros((2, 8, 16), dtype=np.uint8)
    with pytest.raises(ValueError):
        oracle.grouped_scaled_mm(a, b, np.ones(4), np.ones((2, 8)), [3, 2])
    with pytest.raises(ValueError):
        oracle.grouped_scaled_mm(a, b, np.ones(4), np.ones((2, 8)), [1, 3])


def test_row_subset_matches_full():
    a = _random_codes((20, 256), 61)
    b = _random_codes((33, 256), 62)
    sA, sB = _scales(oracle.MM_1x128_128x1, 20, 33, 256, 63)
    ref, mag = oracle.scaled_mm(a, b, sA, sB, oracle.MM_1x128_128x1)
    rows = np.array([19, 0, 7], dtype=np.int64)
    r2, m2 = oracle.scaled_mm(a, b, sA, sB, oracle.MM_1x128_128x1, rows=rows)
    assert np.array_equal(r2, ref[rows]) and np.array_equal(m2, mag[rows])


def test_tolerance_rejects_plausible_mistakes():
    """The GEMM tolerance is tight enough to catch a dropped K block, a
    transposed scale layout or a missing bias on realistic data."""
    M, N, K = 16, 64, 512
    g = W.generator(77)
    x = W.randn_bf16((M, K), 1.0, g)
    w = W.randn_bf16((N, K), 0.02, g)
    qa, sa = oracle.quantize(W.bf16_bits(x), oracle.GROUP_1x128)
    qb, sb = oracle.quantize(W.bf16_bits(w), oracle.GROUP_1x128)
    ref, mag = oracle.scaled_mm(qa, qb, sa, sb, oracle.MM_1x128_128x1)
    # transposed B-scale layout (n-major instead of K-block-major)
    sb_t = sb.reshape(K // 128, N).T.copy().reshape(-1)
    bad, _ = oracle.scaled_mm(qa, qb, sa, sb_t, oracle.MM_1x128_128x1)
    assert not oracle.within_tolerance(bad, ref, mag).all()
    # one K block dropped
    qa2 = qa.copy(); qa2[:, 128:256] = 0
    bad2, _ = oracle.scaled_mm(qa2, qb, sa, sb, oracle.MM_1x128_128x1)
    assert not oracle.within_tolerance(bad2, ref, mag).all()
    assert oracle.within_tolerance(ref, ref, mag).all()
