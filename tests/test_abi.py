"""The C-ABI library loads on a machine without a GPU, exports every symbol
include/fp8sm.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest
import torch

from fp8_scaled_matrix_b200 import fp8sm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    src = open(os.path.join(ROOT, "include", "fp8sm.h")).read()
    return re.findall(r"FP8SM_API\s+[\w\s\*]+?\b(fp8_\w+)\s*\(", src)


def test_header_declares_expected_entry_points():
    syms = set(header_symbols())
    assert {"fp8_quantize", "fp8_scaled_mm", "fp8_grouped_scaled_mm",
            "fp8_get_device_status", "fp8_last_error"} <= syms


def test_library_exports_every_header_symbol(lib):
    for name in header_symbols():
        assert hasattr(lib, name), name
    assert set(fp8sm.EXPORTED) == set(header_symbols())
    assert lib.fp8_version() == 100


def test_workspace_sizes(lib):
    assert lib.fp8_quantize_workspace_bytes(fp8sm.FP8_SCALE_TENSOR, 256, 256) == 16
    for r in (fp8sm.FP8_SCALE_ROW, fp8sm.FP8_SCALE_BLOCK_1x128, fp8sm.FP8_SCALE_BLOCK_128x128):
        assert lib.fp8_quantize_workspace_bytes(r, 256, 256) == 0


P = ctypes.c_void_p
FAKE = P(1 << 20)  # never dereferenced: every call below fails validation first


@pytest.mark.parametrize("args,frag", [
    ((FAKE, 4, 100, 100, fp8sm.FP8_SCALE_ROW), "multiples of 8"),
    ((FAKE, 4, 200, 200, fp8sm.FP8_SCALE_BLOCK_1x128), "cols % 128"),
    ((FAKE, 4, 128, 64, fp8sm.FP8_SCALE_ROW), "ld_x < cols"),
    ((FAKE, -1, 128, 128, fp8sm.FP8_SCALE_ROW), "negative"),
    ((FAKE, 4, 128, 128, 7), "unknown recipe"),
    ((None, 4, 128, 128, fp8sm.FP8_SCALE_ROW), "null"),
])
def test_quantize_rejects_bad_arguments(lib, args, frag):
    x, rows, cols, ld, recipe = args
    st = lib.fp8_quantize(x, rows, cols, ld, recipe, FAKE, FAKE, None, 0, None)
    assert st == fp8sm.FP8_ERR_VALUE
    assert frag in lib.fp8_last_error().decode()


def test_quantize_tensorwise_needs_workspace(lib):
    st = lib.fp8_quantize(FAKE, 4, 128, 128, fp8sm.FP8_SCALE_TENSOR, FAKE, FAKE, None, 0, None)
    assert st == fp8sm.FP8_ERR_VALUE
    assert "workspace" in lib.fp8_last_error().decode()


def test_quantize_misaligned_pointer(lib):
    st = lib.fp8_quantize(P((1 << 20) + 2), 4, 128, 128, fp8sm.FP8_SCALE_ROW, FAKE, FAKE,
                          None, 0, None)
    assert st == fp8sm.FP8_ERR_VALUE and "aligned" in lib.fp8_last_error().decode()


@pytest.mark.parametrize("args,status,frag", [
    ((FAKE, 256, 128, 128, fp8sm.FP8_SCALE_ROW), fp8sm.FP8_ERR_UNSUPPORTED, "1x128 and 128x128"),
    ((FAKE, 256, 128, 128, fp8sm.FP8_SCALE_TENSOR), fp8sm.FP8_ERR_UNSUPPORTED, "1x128 and 128x128"),
    ((FAKE, 200, 128, 128, fp8sm.FP8_SCALE_BLOCK_1x128), fp8sm.FP8_ERR_VALUE, "rows must be a multiple of 128"),
    ((FAKE, 256, 100, 100, fp8sm.FP8_SCALE_BLOCK_1x128), fp8sm.FP8_ERR_VALUE, "multiples of 8"),
    ((FAKE, 256, 128, 64, fp8sm.FP8_SCALE_BLOCK_128x128), fp8sm.FP8_ERR_VALUE, "ld_x < cols"),
    ((None, 256, 128, 128, fp8sm.FP8_SCALE_BLOCK_1x128), fp8sm.FP8_ERR_VALUE, "null"),
    ((P((1 << 20) + 2), 256, 128, 128, fp8sm.FP8_SCALE_BLOCK_1x128), fp8sm.FP8_ERR_VALUE, "aligned"),
    ((FAKE, 256, 128, 128, 9), fp8sm.FP8_ERR_VALUE, "unknown recipe"),
])
def test_quantize_transposed_rejects_bad_arguments(lib, args, status, frag):
    x, rows, cols, ld, recipe = args
    st = lib.fp8_quantize_transposed(x, rows, cols, ld, recipe, FAKE, FAKE, None)
    assert st == status
    assert frag in lib.fp8_last_error().decode()


def test_quantize_transposed_empty_is_a_noop_without_cuda(lib):
    assert lib.fp8_quantize_transposed(None, 0, 128, 128, fp8sm.FP8_SCALE_BLOCK_1x128,
                                       None, None, None) == fp8sm.FP8_OK
    assert lib.fp8_quantize_transposed(None, 256, 0, 0, fp8sm.FP8_SCALE_BLOCK_128x128,
                                       None, None, None) == fp8sm.FP8_OK


@pytest.mark.parametrize("M,N,K,recipe,frag", [
    (128, 100, 128, fp8sm.FP8_MM_ROW_ROW, "N must be a multiple of 16"),
    (128, 128, 100, fp8sm.FP8_MM_ROW_ROW, "K must be a multiple of 16"),
    (128, 128, 144, fp8sm.FP8_MM_1x128_128x128, "K % 128"),
    (128, 128, 144, fp8sm.FP8_MM_1x128_128x1, "K % 128"),
    (-1, 128, 128, fp8sm.FP8_MM_ROW_ROW, "negative"),
    (128, 128, 128, 9, "unknown recipe"),
])
def test_scaled_mm_rejects_bad_arguments(lib, M, N, K, recipe, frag):
    st = lib.fp8_scaled_mm(FAKE, FAKE, M, N, K, FAKE, FAKE, recipe, None,
                           fp8sm.FP8_OUT_BF16, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE
    assert frag in lib.fp8_last_error().decode()


def test_scaled_mm_null_and_alignment(lib):
    st = lib.fp8_scaled_mm(None, FAKE, 128, 128, 128, FAKE, FAKE, fp8sm.FP8_MM_ROW_ROW,
                           None, fp8sm.FP8_OUT_BF16, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE
    st = lib.fp8_scaled_mm(FAKE, P((1 << 20) + 8), 128, 128, 128, FAKE, FAKE,
                           fp8sm.FP8_MM_ROW_ROW, None, fp8sm.FP8_OUT_BF16, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and "aligned" in lib.fp8_last_error().decode()
    st = lib.fp8_scaled_mm(FAKE, FAKE, 128, 128, 128, FAKE, FAKE, fp8sm.FP8_MM_ROW_ROW,
                           None, 5, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and "out_dtype" in lib.fp8_last_error().decode()


def test_empty_gemm_is_a_noop_without_cuda(lib):
    # M == 0 or N == 0 returns before any CUDA call
    assert lib.fp8_scaled_mm(None, None, 0, 128, 128, None, None, fp8sm.FP8_MM_ROW_ROW,
                             None, fp8sm.FP8_OUT_BF16, None, None) == fp8sm.FP8_OK
    assert lib.fp8_scaled_mm(None, None, 64, 0, 128, None, None, fp8sm.FP8_MM_ROW_ROW,
                             None, fp8sm.FP8_OUT_BF16, None, None) == fp8sm.FP8_OK


@pytest.mark.parametrize("M,N,K,recipe,frag", [
    (128, 192, 128, fp8sm.FP8_MM_ROW_ROW, "N must be a multiple of 128"),
    (128, 128, 0, fp8sm.FP8_MM_ROW_ROW, "K must be a positive multiple of 16"),
    (128, 128, 100, fp8sm.FP8_MM_TENSOR_TENSOR, "K must be a positive multiple of 16"),
    (128, 128, 144, fp8sm.FP8_MM_1x128_128x128, "K % 128"),
    (128, 128, 144, fp8sm.FP8_MM_1x128_128x1, "K % 128"),
    (128, -128, 128, fp8sm.FP8_MM_ROW_ROW, "negative"),
    (128, 128, 128, 7, "unknown recipe"),
])
def test_scaled_mm_quantized_rejects_bad_arguments(lib, M, N, K, recipe, frag):
    st = lib.fp8_scaled_mm_quantized(FAKE, FAKE, M, N, K, FAKE, FAKE, recipe, None,
                                     FAKE, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE
    assert frag in lib.fp8_last_error().decode()


def test_scaled_mm_quantized_null_alignment_and_empty(lib):
    st = lib.fp8_scaled_mm_quantized(FAKE, FAKE, 128, 128, 128, FAKE, FAKE,
                                     fp8sm.FP8_MM_ROW_ROW, None, FAKE, None, None)
    assert st == fp8sm.FP8_ERR_VALUE and "null" in lib.fp8_last_error().decode()
    st = lib.fp8_scaled_mm_quantized(FAKE, FAKE, 128, 128, 128, FAKE, FAKE,
                                     fp8sm.FP8_MM_ROW_ROW, None, P((1 << 20) + 4), FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and "misaligned" in lib.fp8_last_error().decode()
    st = lib.fp8_scaled_mm_quantized(FAKE, FAKE, 128, 128, 128, FAKE, FAKE,
                                     fp8sm.FP8_MM_ROW_ROW, None, FAKE, P((1 << 20) + 2), None)
    assert st == fp8sm.FP8_ERR_VALUE and "misaligned" in lib.fp8_last_error().decode()
    assert lib.fp8_scaled_mm_quantized(None, None, 0, 128, 128, None, None,
                                       fp8sm.FP8_MM_ROW_ROW, None, None, None,
                                       None) == fp8sm.FP8_OK


@pytest.mark.parametrize("M,N,K,recipe,status,frag", [
    (128, 128, 128, fp8sm.FP8_MM_ROW_ROW, fp8sm.FP8_ERR_UNSUPPORTED, "1x128_128x128"),
    (128, 128, 128, 9, fp8sm.FP8_ERR_VALUE, "unknown recipe"),
    (100, 128, 128, fp8sm.FP8_MM_1x128_128x128, fp8sm.FP8_ERR_VALUE, "multiples of 128"),
    (128, 192, 128, fp8sm.FP8_MM_1x128_128x128, fp8sm.FP8_ERR_VALUE, "multiples of 128"),
    (128, 128, 144, fp8sm.FP8_MM_1x128_128x128, fp8sm.FP8_ERR_VALUE, "K must be"),
    (128, 128, 0, fp8sm.FP8_MM_1x128_128x128, fp8sm.FP8_ERR_VALUE, "K must be"),
    (-128, 128, 128, fp8sm.FP8_MM_1x128_128x128, fp8sm.FP8_ERR_VALUE, "negative"),
])
def test_scaled_mm_quantized_dual_rejects_bad_arguments(lib, M, N, K, recipe, status, frag):
    st = lib.fp8_scaled_mm_quantized_dual(FAKE, FAKE, M, N, K, FAKE, FAKE, recipe, None,
                                          FAKE, FAKE, FAKE, FAKE, None)
    assert st == status
    assert frag in lib.fp8_last_error().decode()


def test_scaled_mm_quantized_dual_null_alignment_and_empty(lib):
    r = fp8sm.FP8_MM_1x128_128x128
    st = lib.fp8_scaled_mm_quantized_dual(FAKE, FAKE, 128, 128, 128, FAKE, FAKE, r, None,
                                          FAKE, FAKE, None, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and "null" in lib.fp8_last_error().decode()
    st = lib.fp8_scaled_mm_quantized_dual(FAKE, FAKE, 128, 128, 128, FAKE, FAKE, r, None,
                                          FAKE, FAKE, P((1 << 20) + 8), FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and "misaligned" in lib.fp8_last_error().decode()
    st = lib.fp8_scaled_mm_quantized_dual(FAKE, FAKE, 128, 128, 128, FAKE, FAKE, r, None,
                                          FAKE, FAKE, FAKE, P((1 << 20) + 2), None)
    assert st == fp8sm.FP8_ERR_VALUE and "misaligned" in lib.fp8_last_error().decode()
    assert lib.fp8_scaled_mm_quantized_dual(None, None, 0, 128, 128, None, None, r, None,
                                            None, None, None, None, None) == fp8sm.FP8_OK


def test_tensor_amax_and_cast_reject_bad_arguments(lib):
    st = lib.fp8_tensor_amax(FAKE, 4, 12, 12, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and "multiples of 8" in lib.fp8_last_error().decode()
    st = lib.fp8_tensor_amax(FAKE, 4, 16, 8, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and "ld_x < cols" in lib.fp8_last_error().decode()
    st = lib.fp8_tensor_amax(FAKE, 4, 16, 16, None, None)
    assert st == fp8sm.FP8_ERR_VALUE and "amax" in lib.fp8_last_error().decode()
    st = lib.fp8_tensor_amax(P((1 << 20) + 8), 4, 16, 16, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and "aligned" in lib.fp8_last_error().decode()
    st = lib.fp8_quantize_tensor_with_amax(FAKE, 4, 16, 16, FAKE, FAKE, None, None)
    assert st == fp8sm.FP8_ERR_VALUE and "out_scale" in lib.fp8_last_error().decode()
    st = lib.fp8_quantize_tensor_with_amax(FAKE, 4, 16, 16, FAKE, None, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and "out_fp8" in lib.fp8_last_error().decode()
    st = lib.fp8_quantize_tensor_with_amax(FAKE, -1, 16, 16, FAKE, FAKE, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and "negative" in lib.fp8_last_error().decode()


def test_grouped_requires_offs(lib):
    st = lib.fp8_grouped_scaled_mm(FAKE, FAKE, 64, 128, 128, 4, FAKE, FAKE, None,
                                   fp8sm.FP8_OUT_BF16, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and "offs is required" in lib.fp8_last_error().decode()
    st = lib.fp8_grouped_scaled_mm(FAKE, FAKE, 64, 128, 128, 0, FAKE, FAKE, FAKE,
                                   fp8sm.FP8_OUT_BF16, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE


def test_python_binding_rejects_host_tensors():
    x = torch.zeros(4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fp8sm.fp8_quantize(x, fp8sm.FP8_SCALE_ROW)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="no fallback"):
        saved = fp8sm._lib
        fp8sm._lib = None
        try:
            fp8sm.load_library(str(tmp_path / "nope.so"))
        finally:
            fp8sm._lib = saved


def test_mx_scale_bytes(lib):
    assert lib.fp8_mx_scale_bytes(128, 128) == 512
    assert lib.fp8_mx_scale_bytes(129, 128) == 1024
    assert lib.fp8_mx_scale_bytes(1, 32) == 512
    assert lib.fp8_mx_scale_bytes(16640, 8192) == 130 * 64 * 512
    assert lib.fp8_mx_scale_bytes(0, 64) == 0


@pytest.mark.parametrize("rows,cols,ld,frag", [
    (128, 48, 48, "multiple of 32"),
    (128, 64, 60, "ld_x"),
    (128, 64, 68, "ld_x"),
    (-1, 64, 64, "negative"),
])
def test_quantize_mx_rejects_bad_arguments(lib, rows, cols, ld, frag):
    st = lib.fp8_quantize_mx(FAKE, rows, cols, ld, FAKE, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and frag in lib.fp8_last_error().decode()


def test_quantize_mx_null_alignment_and_empty(lib):
    assert lib.fp8_quantize_mx(FAKE, 4, 64, 64, FAKE, None, None) == fp8sm.FP8_ERR_VALUE
    st = lib.fp8_quantize_mx(FAKE, 4, 64, 64, FAKE, P((1 << 20) + 8), None)
    assert st == fp8sm.FP8_ERR_VALUE and "aligned" in lib.fp8_last_error().decode()
    assert lib.fp8_quantize_mx(None, 0, 64, 64, None, None, None) == fp8sm.FP8_OK


@pytest.mark.parametrize("M,N,K,frag", [
    (128, 128, 0, "positive multiple of 32"),
    (128, 128, 48, "positive multiple of 32"),
    (128, 120, 64, "N must be a multiple of 16"),
    (128, -16, 64, "negative"),
])
def test_scaled_mm_mx_rejects_bad_arguments(lib, M, N, K, frag):
    st = lib.fp8_scaled_mm_mx(FAKE, FAKE, M, N, K, FAKE, FAKE, None, fp8sm.FP8_OUT_BF16,
                              FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and frag in lib.fp8_last_error().decode()


def test_scaled_mm_mx_null_alignment_dtype_and_empty(lib):
    st = lib.fp8_scaled_mm_mx(FAKE, FAKE, 64, 64, 64, None, FAKE, None, fp8sm.FP8_OUT_BF16,
                              FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and "null" in lib.fp8_last_error().decode()
    st = lib.fp8_scaled_mm_mx(FAKE, FAKE, 64, 64, 64, FAKE, P((1 << 20) + 4), None,
                              fp8sm.FP8_OUT_BF16, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and "aligned" in lib.fp8_last_error().decode()
    st = lib.fp8_scaled_mm_mx(FAKE, FAKE, 64, 64, 64, FAKE, FAKE, None, 7, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and "out_dtype" in lib.fp8_last_error().decode()
    assert lib.fp8_scaled_mm_mx(None, None, 0, 64, 64, None, None, None, fp8sm.FP8_OUT_BF16,
                                None, None) == fp8sm.FP8_OK


@pytest.mark.parametrize("M,N,K,frag", [
    (128, 192, 64, "N must be a multiple of 128"),
    (128, 128, 0, "positive multiple of 32"),
    (128, 128, 80, "positive multiple of 32"),
    (-2, 128, 64, "negative"),
])
def test_scaled_mm_mx_quantized_rejects_bad_arguments(lib, M, N, K, frag):
    st = lib.fp8_scaled_mm_mx_quantized(FAKE, FAKE, M, N, K, FAKE, FAKE, None, FAKE, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and frag in lib.fp8_last_error().decode()


def test_scaled_mm_mx_quantized_null_alignment_and_empty(lib):
    st = lib.fp8_scaled_mm_mx_quantized(FAKE, FAKE, 64, 128, 64, FAKE, FAKE, None, FAKE, None,
                                        None)
    assert st == fp8sm.FP8_ERR_VALUE and "null" in lib.fp8_last_error().decode()
    st = lib.fp8_scaled_mm_mx_quantized(FAKE, FAKE, 64, 128, 64, FAKE, FAKE, None, FAKE,
                                        P((1 << 20) + 4), None)
    assert st == fp8sm.FP8_ERR_VALUE and "aligned" in lib.fp8_last_error().decode()
    assert lib.fp8_scaled_mm_mx_quantized(None, None, 0, 128, 64, None, None, None, None, None,
                                          None) == fp8sm.FP8_OK


@pytest.mark.parametrize("M,N,K,E,frag", [
    (64, 128, 48, 2, "MXFP8 needs K"),
    (64, 128, 0, 2, "MXFP8 needs K"),
    (64, 120, 64, 2, "multiples of 16"),
    (64, 128, 64, 0, "expert count"),
])
def test_grouped_mx_rejects_bad_arguments(lib, M, N, K, E, frag):
    st = lib.fp8_grouped_scaled_mm_mx(FAKE, FAKE, M, N, K, E, FAKE, FAKE, FAKE,
                                      fp8sm.FP8_OUT_BF16, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and frag in lib.fp8_last_error().decode()


def test_grouped_padded_tokens(lib):
    assert lib.fp8_grouped_padded_tokens(0, 4) == 512
    assert lib.fp8_grouped_padded_tokens(300, 2) == (3 + 2) * 128
    assert lib.fp8_grouped_padded_tokens(32768, 16) == (256 + 16) * 128


@pytest.mark.parametrize("args,frag", [
    ((FAKE, 64, 100, 100, FAKE, 2), "multiples of 8"),
    ((FAKE, 64, 128, 128, None, 2), "offs is required"),
    ((FAKE, 64, 128, 128, FAKE, 0), "expert count"),
    ((FAKE, 64, 128, 128, FAKE, 4096), "expert count"),
    ((FAKE, -1, 128, 128, FAKE, 2), "negative"),
])
def test_quantize_transposed_grouped_rejects_bad_arguments(lib, args, frag):
    x, T, cols, ld, offs, E = args
    st = lib.fp8_quantize_transposed_grouped(x, T, cols, ld, offs, E, FAKE, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and frag in lib.fp8_last_error().decode()


@pytest.mark.parametrize("M,N,T,E,frag", [
    (100, 128, 64, 2, "M must be a multiple of 128"),
    (128, 100, 64, 2, "N must be a multiple of 16"),
    (128, 128, 64, 0, "expert count"),
])
def test_grouped_wgrad_rejects_bad_arguments(lib, M, N, T, E, frag):
    st = lib.fp8_grouped_scaled_mm_wgrad(FAKE, FAKE, M, N, T, E, FAKE, FAKE, FAKE,
                                         fp8sm.FP8_OUT_BF16, FAKE, None)
    assert st == fp8sm.FP8_ERR_VALUE and frag in lib.fp8_last_error().decode()


@pytest.mark.parametrize("fn,args,status,frag", [
    ("fp8_quantize_batched", (FAKE, 2, 128, 100, 100, fp8sm.FP8_SCALE_BLOCK_128x128),
     fp8sm.FP8_ERR_VALUE, "cols % 128"),
    ("fp8_quantize_batched", (FAKE, 2, 128, 128, 128, fp8sm.FP8_SCALE_BLOCK_1x128),
     fp8sm.FP8_ERR_UNSUPPORTED, "only the 128x128"),
    ("fp8_quantize_batched", (FAKE, -1, 128, 128, 128, fp8sm.FP8_SCALE_BLOCK_128x128),
     fp8sm.FP8_ERR_VALUE, "bad batch"),
    ("fp8_quantize_transposed_batched", (FAKE, 2, 100, 128, 128, fp8sm.FP8_SCALE_BLOCK_1x128),
     fp8sm.FP8_ERR_VALUE, "rows must be a multiple of 128"),
    ("fp8_quantize_transposed_batched", (FAKE, 2, 128, 128, 128, fp8sm.FP8_SCALE_ROW),
     fp8sm.FP8_ERR_UNSUPPORTED, "only the 1x128 and 128x128"),
])
def test_batched_quantize_rejects_bad_arguments(lib, fn, args, status, frag):
    st = getattr(lib, fn)(*args, FAKE, FAKE, None)
    assert st == status and frag in lib.fp8_last_error().decode()


def test_batched_quantize_empty_is_a_noop(lib):
    assert lib.fp8_quantize_batched(None, 0, 128, 128, 128, fp8sm.FP8_SCALE_BLOCK_128x128,
                                    None, None, None) == fp8sm.FP8_OK
    assert lib.fp8_quantize_transposed_batched(None, 3, 0, 128, 128, fp8sm.FP8_SCALE_BLOCK_1x128,
                                               None, None, None) == fp8sm.FP8_OK


def test_binding_rejects_caller_outputs_smaller_than_the_library_writes():
    """fp8_quantize / fp8_quantize_noalloc write through the raw pointers of
    caller-passed outputs: the binding refuses, before any launch, buffers of
    the wrong dtype, non-contiguous ones and ones smaller than the codes
    (rows x cols bytes) or the recipe's scale count."""
    x = torch.zeros(256, 384, dtype=torch.bfloat16)
    q = torch.empty(256, 384, dtype=torch.uint8)
    for recipe in (fp8sm.FP8_SCALE_TENSOR, fp8sm.FP8_SCALE_ROW,
                   fp8sm.FP8_SCALE_BLOCK_1x128, fp8sm.FP8_SCALE_BLOCK_128x128):
        n = max(fp8sm.scale_count(256, 384, recipe), 1)
        s = torch.empty(n, dtype=torch.float32)
        fp8sm._check_quant_outputs(x, q, s, 256, 384, recipe)      # exact sizes pass
        with pytest.raises(ValueError):
            fp8sm._check_quant_outputs(x, q.view(-1)[:-1], s, 256, 384, recipe)
        if n > 1:
            with pytest.raises(ValueError):
                fp8sm._check_quant_outputs(x, q, s[:-1], 256, 384, recipe)
        with pytest.raises(ValueError):
            fp8sm._check_quant_outputs(x, q, s.view(torch.int32), 256, 384, recipe)
        with pytest.raises(ValueError):
            fp8sm._check_quant_outputs(x, q.to(torch.int8), s, 256, 384, recipe)
    with pytest.raises(ValueError):   # a column slice is not contiguous
        fp8sm._check_quant_outputs(x, torch.empty(256, 768, dtype=torch.uint8)[:, :384],
                                   torch.empty(256, dtype=torch.float32), 256, 384,
                                   fp8sm.FP8_SCALE_ROW)
