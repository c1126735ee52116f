"""CPU oracle for the FP8 scaled matrix multiply and its dynamic quantizer.

TEST INFRASTRUCTURE ONLY: tests/, the smoke check in __graft_entry__.py and
the CPU-baseline leg of bench.py may use it; the product package
(fp8_scaled_matrix_b200) never imports it, and it imports nothing from there.

A thin ctypes wrapper over oracle/liboracle.so (plain C, see oracle.c): numpy
arrays in, numpy arrays out.  bf16 tensors travel as their uint16 bit
patterns, e4m3 tensors as their uint8 codes.
"""
import ctypes
import os

import numpy as np

from . import build as _build

GROUP_TENSOR, GROUP_ROW, GROUP_1x128, GROUP_128x128 = 0, 1, 2, 3
MM_TENSOR_TENSOR, MM_ROW_ROW, MM_1x128_128x128, MM_1x128_128x1 = 0, 1, 2, 3
EPS = np.float32(1e-12)

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.or_e4m3_decode.restype = ctypes.c_double
        L.or_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.or_e4m3_encode.restype = ctypes.c_uint8
        L.or_e4m3_encode.argtypes = [ctypes.c_float]
        L.or_e4m3_encode_bits.restype = None
        L.or_e4m3_encode_bits.argtypes = [P, I64, P]
        L.or_quantize.restype = ctypes.c_int
        L.or_quantize.argtypes = [P, I64, I64, I64, ctypes.c_int, P, P]
        L.or_quantize_f32.restype = ctypes.c_int
        L.or_quantize_f32.argtypes = [P, I64, I64, I64, ctypes.c_int, P, P]
        L.or_cast_with_inverse.restype = ctypes.c_int
        L.or_cast_with_inverse.argtypes = [P, I64, I64, I64, ctypes.c_float, P]
        L.or_scaled_mm.restype = ctypes.c_int
        L.or_scaled_mm.argtypes = [P, P, I64, I64, I64, P, P, ctypes.c_int, P,
                                   P, I64, P, P]
        L.or_dequant_then_matmul.restype = ctypes.c_int
        L.or_dequant_then_matmul.argtypes = [P, P, I64, I64, I64, P, P,
                                             ctypes.c_int, P, P]
        L.or_grouped_scaled_mm.restype = ctypes.c_int
        L.or_grouped_scaled_mm.argtypes = [P, P, I64, I64, I64, ctypes.c_int32,
                                           P, P, P, P, I64, P, P]
        L.or_mx_quantize.restype = ctypes.c_int
        L.or_mx_quantize.argtypes = [P, I64, I64, I64, P, P]
        L.or_mx_quantize_f32.restype = ctypes.c_int
        L.or_mx_quantize_f32.argtypes = [P, I64, I64, I64, P, P]
        L.or_mx_scales_to_tiles.restype = ctypes.c_int
        L.or_mx_scales_to_tiles.argtypes = [P, I64, I64, P]
        L.or_mx_scaled_mm.restype = ctypes.c_int
        L.or_mx_scaled_mm.argtypes = [P, P, I64, I64, I64, P, P, P, P, I64, P, P]
        L.or_num_threads.restype = ctypes.c_int
        L.or_num_threads.argtypes = []
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return lib().or_num_threads()


def e4m3_decode(code: int) -> float:
    return lib().or_e4m3_decode(int(code))


def e4m3_encode(y: float) -> int:
    return lib().or_e4m3_encode(float(y))


def e4m3_encode_bits(bits: np.ndarray) -> np.ndarray:
    """Encode fp32 values given as uint32 bit patterns."""
    bits = _c(bits, np.uint32)
    out = np.empty(bits.shape, dtype=np.uint8)
    lib().or_e4m3_encode_bits(_ptr(bits), bits.size, _ptr(out))
    return out


def scale_count(rows: int, cols: int, group: int) -> int:
    if group == GROUP_TENSOR:
        return 1
    if group == GROUP_ROW:
        return rows
    if group == GROUP_1x128:
        return (cols // 128) * rows
    return (cols // 128) * ((rows + 127) // 128)


def quantize(x_bits: np.ndarray, group: int):
    """Dynamic quantization of a bf16 matrix (uint16 bit patterns, 2-D).

    Returns (q uint8 (rows, cols), scales float32 (scale_count,))."""
    x_bits = _c(x_bits, np.uint16)
    rows, cols = x_bits.shape
    q = np.empty((rows, cols), dtype=np.uint8)
    s = np.empty(max(scale_count(rows, cols, group), 1), dtype=np.float32)
    rc = lib().or_quantize(_ptr(x_bits), rows, cols, cols, group, _ptr(q), _ptr(s))
    if rc != 0:
        raise ValueError("oracle quantize: bad arguments")
    return q, s[:scale_count(rows, cols, group)]


def quantize_f32(x: np.ndarray, group: int):
    """The same quantization steps on an fp32 matrix (2-D): for checking a
    GEMM epilogue that quantizes its fp32 result.

    Returns (q uint8 (rows, cols), scales float32 (scale_count,))."""
    x = _c(x, np.float32)
    rows, cols = x.shape
    q = np.empty((rows, cols), dtype=np.uint8)
    s = np.empty(max(scale_count(rows, cols, group), 1), dtype=np.float32)
    rc = lib().or_quantize_f32(_ptr(x), rows, cols, cols, group, _ptr(q), _ptr(s))
    if rc != 0:
        raise ValueError("oracle quantize_f32: bad arguments")
    return q, s[:scale_count(rows, cols, group)]


def cast_with_inverse(x_bits: np.ndarray, inv: float) -> np.ndarray:
    x_bits = _c(x_bits, np.uint16)
    rows, cols = x_bits.shape
    q = np.empty((rows, cols), dtype=np.uint8)
    rc = lib().or_cast_with_inverse(_ptr(x_bits), rows, cols, cols,
                                    np.float32(inv), _ptr(q))
    if rc != 0:
        raise ValueError("oracle cast: bad arguments")
    return q


def scaled_mm(a, b, sA, sB, recipe, bias_bits=None, rows=None):
    """Reference (ref, mag) of out = (A*sA) @ (B*sB)^T + bias, fp64.

    a: (M,K) uint8 codes; b: (N,K) uint8 codes; rows: optional row subset."""
    a = _c(a, np.uint8)
    b = _c(b, np.uint8)
    M, K = a.shape
    N = b.shape[0]
    assert b.shape[1] == K
    sA = _c(sA, np.float32)
    sB = _c(sB, np.float32)
    bias = None if bias_bits is None else _c(bias_bits, np.uint16)
    r = None if rows is None else _c(rows, np.int64)
    R = M if r is None else r.size
    ref = np.empty((R, N), dtype=np.float64)
    mag = np.empty((R, N), dtype=np.float64)
    rc = lib().or_scaled_mm(_ptr(a), _ptr(b), M, N, K, _ptr(sA), _ptr(sB),
                            recipe, _ptr(bias), _ptr(r), R, _ptr(ref), _ptr(mag))
    if rc != 0:
        raise ValueError("oracle scaled_mm: bad arguments")
    return ref, mag


def dequant_then_matmul(a, b, sA, sB, recipe, bias_bits=None):
    a = _c(a, np.uint8)
    b = _c(b, np.uint8)
    M, K = a.shape
    N = b.shape[0]
    sA = _c(sA, np.float32)
    sB = _c(sB, np.float32)
    bias = None if bias_bits is None else _c(bias_bits, np.uint16)
    ref = np.empty((M, N), dtype=np.float64)
    rc = lib().or_dequant_then_matmul(_ptr(a), _ptr(b), M, N, K, _ptr(sA),
                                      _ptr(sB), recipe, _ptr(bias), _ptr(ref))
    if rc != 0:
        raise ValueError("oracle dequant_then_matmul: bad arguments")
    return ref


def grouped_scaled_mm(a, b_experts, sA, sB, offs, rows=None):
    """Grouped rowwise reference: a (M_total,K), b_experts (E,N,K), sA (M_total,),
    sB (E,N), offs (E,) int32 cumulative ends.  Returns (ref, mag)."""
    a = _c(a, np.uint8)
    b = _c(b_experts, np.uint8)
    M, K = a.shape
    E, N, K2 = b.shape
    assert K2 == K
    sA = _c(sA, np.float32)
    sB = _c(sB, np.float32)
    offs = _c(offs, np.int32)
    r = None if rows is None else _c(rows, np.int64)
    R = M if r is None else r.size
    ref = np.empty((R, N), dtype=np.float64)
    mag = np.empty((R, N), dtype=np.float64)
    rc = lib().or_grouped_scaled_mm(_ptr(a), _ptr(b), M, N, K, E, _ptr(sA),
                                    _ptr(sB), _ptr(offs), _ptr(r), R, _ptr(ref),
                                    _ptr(mag))
    if rc != 0:
        raise ValueError("oracle grouped_scaled_mm: bad arguments")
    return ref, mag


def within_tolerance(out, ref, mag, rel=1e-2, abs_mag=1e-3):
    """Per-element GEMM check |out - ref| <= rel*|ref| + abs_mag*mag.

    Returns a boolean array."""
    out = np.asarray(out, dtype=np.float64)
    return np.abs(out - ref) <= rel * np.abs(ref) + abs_mag * mag


# ---------------------------------------------------------------- MXFP8

def mx_quantize(x_bits: np.ndarray):
    """MXFP8 quantization of a bf16 matrix (uint16 bit patterns, 2-D, cols % 32
    == 0): returns (q uint8 (rows, cols), e8 uint8 (rows, cols // 32))."""
    x_bits = _c(x_bits, np.uint16)
    rows, cols = x_bits.shape
    q = np.empty((rows, cols), dtype=np.uint8)
    e8 = np.empty((rows, max(cols // 32, 1)), dtype=np.uint8)
    rc = lib().or_mx_quantize(_ptr(x_bits), rows, cols, cols, _ptr(q), _ptr(e8))
    if rc != 0:
        raise ValueError("oracle mx_quantize: bad arguments")
    return q, e8[:, :cols // 32]


def mx_quantize_f32(x: np.ndarray):
    """The same MXFP8 conversion of an fp32 matrix (2-D, cols % 32 == 0)."""
    x = _c(x, np.float32)
    rows, cols = x.shape
    q = np.empty((rows, cols), dtype=np.uint8)
    e8 = np.empty((rows, max(cols // 32, 1)), dtype=np.uint8)
    rc = lib().or_mx_quantize_f32(_ptr(x), rows, cols, cols, _ptr(q), _ptr(e8))
    if rc != 0:
        raise ValueError("oracle mx_quantize_f32: bad arguments")
    return q, e8[:, :cols // 32]


def mx_tile_bytes(rows: int, kblocks: int) -> int:
    return ((rows + 127) // 128) * ((kblocks + 3) // 4) * 512


def mx_scales_to_tiles(e8: np.ndarray) -> np.ndarray:
    """(rows, kblocks) scale bytes -> the flat scale-factor tile layout."""
    e8 = _c(e8, np.uint8)
    rows, kblocks = e8.shape
    out = np.empty(max(mx_tile_bytes(rows, kblocks), 1), dtype=np.uint8)
    rc = lib().or_mx_scales_to_tiles(_ptr(e8), rows, kblocks, _ptr(out))
    if rc != 0:
        raise ValueError("oracle mx_scales_to_tiles: bad arguments")
    return out[:mx_tile_bytes(rows, kblocks)]


def mx_scaled_mm(a, b, ea, eb, bias_bits=None, rows=None):
    """MXFP8 GEMM reference (ref, mag), fp64: a (M,K), b (N,K) codes; ea
    (M, K/32), eb (N, K/32) plain scale bytes."""
    a = _c(a, np.uint8)
    b = _c(b, np.uint8)
    ea = _c(ea, np.uint8)
    eb = _c(eb, np.uint8)
    M, K = a.shape
    N = b.shape[0]
    bias = None if bias_bits is None else _c(bias_bits, np.uint16)
    r = None if rows is None else _c(rows, np.int64)
    R = M if r is None else r.size
    ref = np.empty((R, N), dtype=np.float64)
    mag = np.empty((R, N), dtype=np.float64)
    rc = lib().or_mx_scaled_mm(_ptr(a), _ptr(b), M, N, K, _ptr(ea), _ptr(eb), _ptr(bias),
                               _ptr(r), 0 if r is None else r.size, _ptr(ref), _ptr(mag))
    if rc != 0:
        raise ValueError("oracle mx_scaled_mm: bad arguments")
    return ref, mag
