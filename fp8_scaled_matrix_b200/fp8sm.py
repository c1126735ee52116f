"""Thin Python binding over the C ABI in include/fp8sm.h (libfp8sm.so).

Argument marshalling only: torch tensors supply device memory and the
current CUDA stream; every step of the computation runs in the library's
kernels.  There is no fallback: if the library cannot be loaded, or a call
returns an error, an exception is raised.

Names match the C entry points (fp8_quantize, fp8_scaled_mm,
fp8_grouped_scaled_mm, fp8_get_device_status, fp8_last_error, ...).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8sm.so")

# enums (include/fp8sm.h)
FP8_OK, FP8_ERR_VALUE, FP8_ERR_UNSUPPORTED, FP8_ERR_CUDA, FP8_ERR_TIMEOUT = 0, 1, 2, 3, 4
FP8_SCALE_TENSOR, FP8_SCALE_ROW, FP8_SCALE_BLOCK_1x128, FP8_SCALE_BLOCK_128x128 = 0, 1, 2, 3
FP8_MM_TENSOR_TENSOR, FP8_MM_ROW_ROW, FP8_MM_1x128_128x128, FP8_MM_1x128_128x1 = 0, 1, 2, 3
FP8_OUT_BF16, FP8_OUT_F32 = 0, 1

QUANT_RECIPES = {"tensor": FP8_SCALE_TENSOR, "row": FP8_SCALE_ROW,
                 "1x128": FP8_SCALE_BLOCK_1x128, "128x128": FP8_SCALE_BLOCK_128x128}
MM_RECIPES = {"tensor": FP8_MM_TENSOR_TENSOR, "row": FP8_MM_ROW_ROW,
              "1x128_128x128": FP8_MM_1x128_128x128, "1x128_128x1": FP8_MM_1x128_128x1}

EXPORTED = ["fp8_version", "fp8_last_error", "fp8_quantize_workspace_bytes",
            "fp8_quantize", "fp8_scaled_mm", "fp8_grouped_scaled_mm",
            "fp8_get_device_status", "fp8_debug_timeout_probe",
            "fp8_quantize_noalloc", "fp8_quantize_transposed",
            "fp8_grouped_scaled_mm_blockwise", "fp8_scaled_mm_quantized",
            "fp8_mx_scale_bytes", "fp8_quantize_mx", "fp8_scaled_mm_mx",
            "fp8_scaled_mm_mx_quantized", "fp8_grouped_scaled_mm_mx",
            "fp8_grouped_padded_tokens", "fp8_quantize_transposed_grouped",
            "fp8_grouped_scaled_mm_wgrad", "fp8_quantize_batched",
            "fp8_quantize_transposed_batched", "fp8_scaled_mm_quantized_dual",
            "fp8_tensor_amax", "fp8_quantize_tensor_with_amax"]


class Fp8Error(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"[status {status}] {msg}")
        self.status = status


class Fp8ValueError(Fp8Error, ValueError):
    pass


class Fp8Unsupported(Fp8Error, NotImplementedError):
    pass


class Fp8Timeout(Fp8Error):
    pass


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libfp8sm.so (raises if it is missing; there is no other path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m fp8_scaled_matrix_b200.build` "
            "(there is no fallback implementation)")
    L = ctypes.CDLL(path)
    P, I64, I32, U32, SZ = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                           ctypes.c_uint32, ctypes.c_size_t)
    E = ctypes.c_int
    L.fp8_version.restype = ctypes.c_int
    L.fp8_version.argtypes = []
    L.fp8_last_error.restype = ctypes.c_char_p
    L.fp8_last_error.argtypes = []
    L.fp8_quantize_workspace_bytes.restype = SZ
    L.fp8_quantize_workspace_bytes.argtypes = [E, I64, I64]
    L.fp8_quantize.restype = E
    L.fp8_quantize.argtypes = [P, I64, I64, I64, E, P, P, P, SZ, P]
    L.fp8_scaled_mm.restype = E
    L.fp8_scaled_mm.argtypes = [P, P, I64, I64, I64, P, P, E, P, E, P, P]
    L.fp8_mx_scale_bytes.restype = SZ
    L.fp8_mx_scale_bytes.argtypes = [I64, I64]
    L.fp8_quantize_mx.restype = E
    L.fp8_quantize_mx.argtypes = [P, I64, I64, I64, P, P, P]
    L.fp8_scaled_mm_mx.restype = E
    L.fp8_scaled_mm_mx.argtypes = [P, P, I64, I64, I64, P, P, P, E, P, P]
    L.fp8_scaled_mm_mx_quantized.restype = E
    L.fp8_scaled_mm_mx_quantized.argtypes = [P, P, I64, I64, I64, P, P, P, P, P, P]
    L.fp8_scaled_mm_quantized.restype = E
    L.fp8_scaled_mm_quantized.argtypes = [P, P, I64, I64, I64, P, P, E, P, P, P, P]
    L.fp8_grouped_scaled_mm.restype = E
    L.fp8_grouped_scaled_mm.argtypes = [P, P, I64, I64, I64, I32, P, P, P, E, P, P]
    L.fp8_tensor_amax.restype = E
    L.fp8_tensor_amax.argtypes = [P, I64, I64, I64, P, P]
    L.fp8_quantize_tensor_with_amax.restype = E
    L.fp8_quantize_tensor_with_amax.argtypes = [P, I64, I64, I64, P, P, P, P]
    L.fp8_scaled_mm_quantized_dual.restype = E
    L.fp8_scaled_mm_quantized_dual.argtypes = [P, P, I64, I64, I64, P, P, E, P, P, P, P, P, P]
    L.fp8_quantize_batched.restype = E
    L.fp8_quantize_batched.argtypes = [P, I32, I64, I64, I64, E, P, P, P]
    L.fp8_quantize_transposed_batched.restype = E
    L.fp8_quantize_transposed_batched.argtypes = [P, I32, I64, I64, I64, E, P, P, P]
    L.fp8_grouped_padded_tokens.restype = I64
    L.fp8_grouped_padded_tokens.argtypes = [I64, I32]
    L.fp8_quantize_transposed_grouped.restype = E
    L.fp8_quantize_transposed_grouped.argtypes = [P, I64, I64, I64, P, I32, P, P, P]
    L.fp8_grouped_scaled_mm_wgrad.restype = E
    L.fp8_grouped_scaled_mm_wgrad.argtypes = [P, P, I64, I64, I64, I32, P, P, P, E, P, P]
    L.fp8_grouped_scaled_mm_mx.restype = E
    L.fp8_grouped_scaled_mm_mx.argtypes = [P, P, I64, I64, I64, I32, P, P, P, E, P, P]
    L.fp8_grouped_scaled_mm_blockwise.restype = E
    L.fp8_grouped_scaled_mm_blockwise.argtypes = [P, P, I64, I64, I64, I32, P, P, P, E, P, P]
    L.fp8_get_device_status.restype = E
    L.fp8_get_device_status.argtypes = [P]
    L.fp8_debug_timeout_probe.restype = E
    L.fp8_debug_timeout_probe.argtypes = [U32, P]
    L.fp8_quantize_noalloc.restype = E
    L.fp8_quantize_noalloc.argtypes = [P, I64, I64, I64, E, P, P, P]
    L.fp8_quantize_transposed.restype = E
    L.fp8_quantize_transposed.argtypes = [P, I64, I64, I64, E, P, P, P]
    _lib = L
    return L


def _check(status: int):
    if status == FP8_OK:
        return
    msg = load_library().fp8_last_error().decode(errors="replace")
    cls = {FP8_ERR_VALUE: Fp8ValueError, FP8_ERR_UNSUPPORTED: Fp8Unsupported,
           FP8_ERR_TIMEOUT: Fp8Timeout}.get(status, Fp8Error)
    raise cls(status, msg)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must live in CUDA device memory")


def _check_quant_outputs(x: torch.Tensor, out: torch.Tensor, scales: torch.Tensor,
                         rows: int, cols: int, recipe: int) -> None:
    """Caller-passed outputs of a quantization: contiguous, of the right
    dtype, on x's device and large enough for what the library writes (the
    codes, rows x cols bytes, and the recipe's scales); the library writes
    through the raw pointers, so a smaller buffer would be overrun."""
    if (out.dtype != torch.uint8 or not out.is_contiguous() or out.device != x.device
            or out.numel() < rows * cols):
        raise ValueError(f"out must be a contiguous uint8 tensor on {x.device} with at "
                         f"least {rows * cols} elements")
    need = max(scale_count(rows, cols, recipe), 1)
    if (scales.dtype != torch.float32 or not scales.is_contiguous()
            or scales.device != x.device or scales.numel() < need):
        raise ValueError(f"scales must be a contiguous float32 tensor on {x.device} with at "
                         f"least {need} elements")


def fp8_version() -> int:
    return load_library().fp8_version()


def fp8_last_error() -> str:
    return load_library().fp8_last_error().decode(errors="replace")


def scale_count(rows: int, cols: int, recipe: int) -> int:
    if recipe == FP8_SCALE_TENSOR:
        return 1
    if recipe == FP8_SCALE_ROW:
        return rows
    if recipe == FP8_SCALE_BLOCK_1x128:
        return (cols // 128) * rows
    return (cols // 128) * ((rows + 127) // 128)


def fp8_quantize_workspace_bytes(recipe: int, rows: int, cols: int) -> int:
    return load_library().fp8_quantize_workspace_bytes(recipe, rows, cols)


def fp8_quantize(x: torch.Tensor, recipe: int, out: Optional[torch.Tensor] = None,
                 scales: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None,
                 stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Quantize a 2-D bf16 CUDA tensor (row stride x.stride(0)).

    Returns (codes uint8 (rows, cols), scales float32).  `out`, `scales` and
    `workspace` may be passed to avoid allocations."""
    L = load_library()
    _need_cuda(x)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 tensor with unit column stride")
    rows, cols = x.shape
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(max(scale_count(rows, cols, recipe), 1),
                             dtype=torch.float32, device=x.device)
    _need_cuda(out, scales, workspace)
    _check_quant_outputs(x, out, scales, rows, cols, recipe)
    ws_bytes = L.fp8_quantize_workspace_bytes(recipe, rows, cols)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=x.device)
    if workspace is not None and (workspace.device != x.device or not workspace.is_contiguous()):
        raise ValueError(f"workspace must be a contiguous tensor on {x.device}")
    # the row stride only matters when there is more than one non-empty row
    ld = x.stride(0) if (rows > 1 and cols > 0) else cols
    _check(L.fp8_quantize(_ptr(x), rows, cols, ld, recipe, _ptr(out),
                          _ptr(scales), _ptr(workspace),
                          0 if workspace is None else workspace.numel() * workspace.element_size(),
                          _stream(stream)))
    return out, scales


def fp8_quantize_noalloc(x: torch.Tensor, recipe: int, out: torch.Tensor,
                         scales: torch.Tensor, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Quantize like fp8_quantize without any allocation, for callers that
    may not allocate device memory (for example a plugin inside a host
    application that owns every allocation, or a service whose memory plan
    is fixed at start-up).  The caller passes the output buffers; the library
    uses its own fixed scratch, shared by all calls (order calls on one
    stream: concurrent calls race on it)."""
    L = load_library()
    _need_cuda(x, out, scales)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 tensor with unit column stride")
    rows, cols = x.shape
    _check_quant_outputs(x, out, scales, rows, cols, recipe)
    ld = x.stride(0) if (rows > 1 and cols > 0) else cols
    _check(L.fp8_quantize_noalloc(_ptr(x), rows, cols, ld, recipe, _ptr(out),
                                  _ptr(scales), _stream(stream)))
    return out, scales


def fp8_quantize_transposed(x: torch.Tensor, recipe: int, out: Optional[torch.Tensor] = None,
                            scales: Optional[torch.Tensor] = None,
                            stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Quantize x^T (x: 2-D bf16 CUDA tensor (rows, cols), rows % 128 == 0)
    with the 1x128 or 128x128 recipe, as fp8_quantize(x.t()) would.

    Returns (codes uint8 (cols, rows), scales float32 in the recipe's layout
    for a (cols, rows) matrix)."""
    L = load_library()
    _need_cuda(x)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 tensor with unit column stride")
    rows, cols = x.shape
    if out is None:
        out = torch.empty((cols, rows), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(max(scale_count(cols, rows, recipe), 1),
                             dtype=torch.float32, device=x.device)
    ld = x.stride(0) if (rows > 1 and cols > 0) else cols
    _check(L.fp8_quantize_transposed(_ptr(x), rows, cols, ld, recipe, _ptr(out),
                                     _ptr(scales), _stream(stream)))
    return out, scales


def fp8_scaled_mm(a: torch.Tensor, b: torch.Tensor, scale_a: torch.Tensor,
                  scale_b: torch.Tensor, recipe: int,
                  bias: Optional[torch.Tensor] = None, out_dtype=torch.bfloat16,
                  out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out = (a * scale_a) @ (b * scale_b)^T (+ bias); a (M,K), b (N,K) uint8 e4m3 codes."""
    L = load_library()
    _need_cuda(a, b, scale_a, scale_b, bias)
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K:
        raise ValueError("a and b must share K")
    for t in (a, b):
        if t.dtype not in (torch.uint8, torch.float8_e4m3fn) or not t.is_contiguous():
            raise ValueError("a and b must be contiguous e4m3 (uint8 codes)")
    if bias is not None and (bias.dtype != torch.bfloat16 or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous bf16 tensor")
    od = FP8_OUT_F32 if out_dtype == torch.float32 else FP8_OUT_BF16
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=a.device)
    _check(L.fp8_scaled_mm(_ptr(a), _ptr(b), M, N, K, _ptr(scale_a), _ptr(scale_b),
                           recipe, _ptr(bias), od, _ptr(out), _stream(stream)))
    return out


def fp8_scaled_mm_quantized(a: torch.Tensor, b: torch.Tensor, scale_a: torch.Tensor,
                            scale_b: torch.Tensor, recipe: int,
                            bias: Optional[torch.Tensor] = None,
                            out: Optional[torch.Tensor] = None,
                            out_scales: Optional[torch.Tensor] = None,
                            stream=None):
    """fp8_scaled_mm whose result is quantized in 1x128 groups along n.

    Returns (codes (M, N) uint8 e4m3, scales (N/128, M) fp32).
    """
    L = load_library()
    _need_cuda(a, b, scale_a, scale_b, bias)
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K:
        raise ValueError("a and b must share K")
    for t in (a, b):
        if t.dtype not in (torch.uint8, torch.float8_e4m3fn) or not t.is_contiguous():
            raise ValueError("a and b must be contiguous e4m3 (uint8 codes)")
    if bias is not None and (bias.dtype != torch.bfloat16 or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous bf16 tensor")
    if out is None:
        out = torch.empty((M, N), dtype=torch.uint8, device=a.device)
    if out_scales is None:
        out_scales = torch.empty((N // 128, M), dtype=torch.float32, device=a.device)
    if out.numel() < M * N or out_scales.numel() < (N // 128) * M:
        raise ValueError("out or out_scales too small")
    _check(L.fp8_scaled_mm_quantized(_ptr(a), _ptr(b), M, N, K, _ptr(scale_a),
                                     _ptr(scale_b), recipe, _ptr(bias), _ptr(out),
                                     _ptr(out_scales), _stream(stream)))
    return out, out_scales


def fp8_mx_scale_bytes(rows: int, cols: int) -> int:
    return int(load_library().fp8_mx_scale_bytes(rows, cols))


def fp8_quantize_mx(x: torch.Tensor, out: Optional[torch.Tensor] = None,
                    scales: Optional[torch.Tensor] = None,
                    stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """MXFP8 quantization of a 2-D bf16 CUDA tensor: returns (codes uint8
    (rows, cols), E8M0 scale bytes uint8 in the scale-factor tile layout)."""
    L = load_library()
    _need_cuda(x)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 tensor with unit column stride")
    rows, cols = x.shape
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    nbytes = fp8_mx_scale_bytes(rows, cols)
    if scales is None:
        scales = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    if out.numel() < rows * cols or scales.numel() < nbytes:
        raise ValueError("out or scales too small")
    _check(L.fp8_quantize_mx(_ptr(x), rows, cols, x.stride(0), _ptr(out), _ptr(scales),
                             _stream(stream)))
    return out, scales[:nbytes] if scales.numel() > nbytes else scales


def fp8_scaled_mm_mx(a: torch.Tensor, b: torch.Tensor, scale_a: torch.Tensor,
                     scale_b: torch.Tensor, bias: Optional[torch.Tensor] = None,
                     out_dtype=torch.bfloat16, out: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """MXFP8 GEMM: a (M,K), b (N,K) e4m3 codes; scale_a, scale_b E8M0 bytes
    in the scale-factor tile layout (as fp8_quantize_mx returns them)."""
    L = load_library()
    _need_cuda(a, b, scale_a, scale_b, bias)
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K:
        raise ValueError("a and b must share K")
    for t in (a, b):
        if t.dtype not in (torch.uint8, torch.float8_e4m3fn) or not t.is_contiguous():
            raise ValueError("a and b must be contiguous e4m3 (uint8 codes)")
    if (scale_a.numel() < fp8_mx_scale_bytes(M, K) or
            scale_b.numel() < fp8_mx_scale_bytes(N, K)):
        raise ValueError("scale tiles too small")
    if bias is not None and (bias.dtype != torch.bfloat16 or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous bf16 tensor")
    od = FP8_OUT_F32 if out_dtype == torch.float32 else FP8_OUT_BF16
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=a.device)
    _check(L.fp8_scaled_mm_mx(_ptr(a), _ptr(b), M, N, K, _ptr(scale_a), _ptr(scale_b),
                              _ptr(bias), od, _ptr(out), _stream(stream)))
    return out


def fp8_scaled_mm_mx_quantized(a: torch.Tensor, b: torch.Tensor, scale_a: torch.Tensor,
                               scale_b: torch.Tensor, bias: Optional[torch.Tensor] = None,
                               out: Optional[torch.Tensor] = None,
                               out_scales: Optional[torch.Tensor] = None,
                               stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """MXFP8 GEMM with MXFP8 output: returns (codes (M, N) uint8, E8M0 scale
    bytes in the scale-factor tile layout) -- the A operand of a next
    fp8_scaled_mm_mx."""
    L = load_library()
    _need_cuda(a, b, scale_a, scale_b, bias)
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K:
        raise ValueError("a and b must share K")
    for t in (a, b):
        if t.dtype not in (torch.uint8, torch.float8_e4m3fn) or not t.is_contiguous():
            raise ValueError("a and b must be contiguous e4m3 (uint8 codes)")
    if bias is not None and (bias.dtype != torch.bfloat16 or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous bf16 tensor")
    if out is None:
        out = torch.empty((M, N), dtype=torch.uint8, device=a.device)
    nbytes = fp8_mx_scale_bytes(M, N)
    if out_scales is None:
        out_scales = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=a.device)
    if out.numel() < M * N or out_scales.numel() < nbytes:
        raise ValueError("out or out_scales too small")
    _check(L.fp8_scaled_mm_mx_quantized(_ptr(a), _ptr(b), M, N, K, _ptr(scale_a),
                                        _ptr(scale_b), _ptr(bias), _ptr(out),
                                        _ptr(out_scales), _stream(stream)))
    return out, out_scales[:nbytes] if out_scales.numel() > nbytes else out_scales


def fp8_grouped_scaled_mm(a: torch.Tensor, b_experts: torch.Tensor,
                          scale_a: torch.Tensor, scale_b: torch.Tensor,
                          offs: torch.Tensor, out_dtype=torch.bfloat16,
                          out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Grouped rowwise GEMM: rows [offs[g-1], offs[g]) of a times expert g."""
    L = load_library()
    _need_cuda(a, b_experts, scale_a, scale_b, offs)
    if offs is None:
        raise ValueError("offs is required")
    if offs.dtype != torch.int32:
        raise ValueError("offs must be int32")
    M, K = a.shape
    E, N, K2 = b_experts.shape
    if K2 != K or offs.numel() != E:
        raise ValueError("shape mismatch")
    od = FP8_OUT_F32 if out_dtype == torch.float32 else FP8_OUT_BF16
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=a.device)
    _check(L.fp8_grouped_scaled_mm(_ptr(a), _ptr(b_experts), M, N, K, E, _ptr(scale_a),
                                   _ptr(scale_b), _ptr(offs), od, _ptr(out),
                                   _stream(stream)))
    return out


def fp8_grouped_scaled_mm_blockwise(a: torch.Tensor, b_experts: torch.Tensor,
                                    scale_a: torch.Tensor, scale_b: torch.Tensor,
                                    offs: torch.Tensor, out_dtype=torch.bfloat16,
                                    out: Optional[torch.Tensor] = None,
                                    stream=None) -> torch.Tensor:
    """Grouped GEMM with 1x128 (a) / per-expert 128x128 (b_experts) scales."""
    L = load_library()
    _need_cuda(a, b_experts, scale_a, scale_b, offs)
    if offs.dtype != torch.int32:
        raise ValueError("offs must be int32")
    M, K = a.shape
    E, N, K2 = b_experts.shape
    if K2 != K or offs.numel() != E:
        raise ValueError("shape mismatch")
    od = FP8_OUT_F32 if out_dtype == torch.float32 else FP8_OUT_BF16
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=a.device)
    _check(L.fp8_grouped_scaled_mm_blockwise(_ptr(a), _ptr(b_experts), M, N, K, E,
                                             _ptr(scale_a), _ptr(scale_b), _ptr(offs), od,
                                             _ptr(out), _stream(stream)))
    return out


def fp8_get_device_status(stream=None) -> int:
    """Synchronize and return (and clear) the device status word."""
    return load_library().fp8_get_device_status(_stream(stream))


def check_device_status(stream=None):
    _check(fp8_get_device_status(stream))


def fp8_debug_timeout_probe(limit_us: int, stream=None):
    _check(load_library().fp8_debug_timeout_probe(limit_us, _stream(stream)))


def fp8_grouped_scaled_mm_mx(a: torch.Tensor, b_experts: torch.Tensor,
                             scale_a: torch.Tensor, scale_b: torch.Tensor,
                             offs: torch.Tensor, out_dtype=torch.bfloat16,
                             out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Grouped MXFP8 GEMM: rows [offs[g-1], offs[g]) of a times expert g;
    scale_a A's scale-factor tiles, scale_b the experts' tile sets in order."""
    L = load_library()
    _need_cuda(a, b_experts, scale_a, scale_b, offs)
    if offs.dtype != torch.int32:
        raise ValueError("offs must be int32")
    M, K = a.shape
    E, N, K2 = b_experts.shape
    if K2 != K or offs.numel() != E:
        raise ValueError("shape mismatch")
    if (scale_a.numel() < fp8_mx_scale_bytes(M, K) or
            scale_b.numel() < E * fp8_mx_scale_bytes(N, K)):
        raise ValueError("scale tiles too small")
    od = FP8_OUT_F32 if out_dtype == torch.float32 else FP8_OUT_BF16
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=a.device)
    _check(L.fp8_grouped_scaled_mm_mx(_ptr(a), _ptr(b_experts), M, N, K, E, _ptr(scale_a),
                                      _ptr(scale_b), _ptr(offs), od, _ptr(out),
                                      _stream(stream)))
    return out


def fp8_grouped_padded_tokens(tokens: int, E: int) -> int:
    return int(load_library().fp8_grouped_padded_tokens(tokens, E))


def fp8_quantize_transposed_grouped(x: torch.Tensor, offs: torch.Tensor,
                                    out: Optional[torch.Tensor] = None,
                                    scales: Optional[torch.Tensor] = None,
                                    stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-expert 1x128 quantization of x^T (x: tokens x cols bf16), each
    group of tokens padded to a multiple of 128: returns (codes (cols, P),
    scales (P/128, cols)), P = fp8_grouped_padded_tokens(tokens, E)."""
    L = load_library()
    _need_cuda(x, offs)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 tensor with unit column stride")
    if offs.dtype != torch.int32:
        raise ValueError("offs must be int32")
    T, cols = x.shape
    E = offs.numel()
    P = fp8_grouped_padded_tokens(T, E)
    if out is None:
        out = torch.empty((cols, P), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((P // 128, cols), dtype=torch.float32, device=x.device)
    if out.numel() < cols * P or scales.numel() < (P // 128) * cols:
        raise ValueError("out or scales too small")
    _check(L.fp8_quantize_transposed_grouped(_ptr(x), T, cols, x.stride(0), _ptr(offs), E,
                                             _ptr(out), _ptr(scales), _stream(stream)))
    return out, scales


def fp8_grouped_scaled_mm_wgrad(a_t: torch.Tensor, b_t: torch.Tensor, scale_a: torch.Tensor,
                                scale_b: torch.Tensor, offs: torch.Tensor, tokens: int,
                                out_dtype=torch.bfloat16, out: Optional[torch.Tensor] = None,
                                stream=None) -> torch.Tensor:
    """Per-expert weight gradient: out[g] = dY_g^T @ X_g from the padded
    transposed codes of fp8_quantize_transposed_grouped; returns (E, M, N)."""
    L = load_library()
    _need_cuda(a_t, b_t, scale_a, scale_b, offs)
    if offs.dtype != torch.int32:
        raise ValueError("offs must be int32")
    E = offs.numel()
    M, P = a_t.shape
    N = b_t.shape[0]
    if b_t.shape[1] != P or P != fp8_grouped_padded_tokens(tokens, E):
        raise ValueError("operands must have the padded width of fp8_quantize_transposed_grouped")
    od = FP8_OUT_F32 if out_dtype == torch.float32 else FP8_OUT_BF16
    if out is None:
        out = torch.empty((E, M, N), dtype=out_dtype, device=a_t.device)
    _check(L.fp8_grouped_scaled_mm_wgrad(_ptr(a_t), _ptr(b_t), M, N, tokens, E, _ptr(scale_a),
                                         _ptr(scale_b), _ptr(offs), od, _ptr(out),
                                         _stream(stream)))
    return out


def fp8_quantize_batched(x: torch.Tensor, recipe: int, out: Optional[torch.Tensor] = None,
                         scales: Optional[torch.Tensor] = None,
                         stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """128x128 quantization of each matrix of a contiguous (B, rows, cols)
    bf16 stack in one launch: returns (codes (B, rows, cols), scales
    (B, cols/128, ceil(rows/128)))."""
    L = load_library()
    _need_cuda(x)
    if x.dtype != torch.bfloat16 or x.dim() != 3 or not x.is_contiguous():
        raise ValueError("x must be a contiguous (B, rows, cols) bf16 tensor")
    B, rows, cols = x.shape
    if out is None:
        out = torch.empty((B, rows, cols), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((B, cols // 128, (rows + 127) // 128), dtype=torch.float32,
                             device=x.device)
    _check(L.fp8_quantize_batched(_ptr(x), B, rows, cols, cols, recipe, _ptr(out), _ptr(scales),
                                  _stream(stream)))
    return out, scales


def fp8_quantize_transposed_batched(x: torch.Tensor, recipe: int,
                                    out: Optional[torch.Tensor] = None,
                                    scales: Optional[torch.Tensor] = None,
                                    stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """1x128 / 128x128 quantization of each matrix's transpose for a
    contiguous (B, rows, cols) bf16 stack: returns (codes (B, cols, rows),
    scales, each matrix's fp8_quantize_transposed layout in order)."""
    L = load_library()
    _need_cuda(x)
    if x.dtype != torch.bfloat16 or x.dim() != 3 or not x.is_contiguous():
        raise ValueError("x must be a contiguous (B, rows, cols) bf16 tensor")
    B, rows, cols = x.shape
    per = scale_count(cols, rows, recipe)
    if out is None:
        out = torch.empty((B, cols, rows), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((B, per), dtype=torch.float32, device=x.device)
    _check(L.fp8_quantize_transposed_batched(_ptr(x), B, rows, cols, cols, recipe, _ptr(out),
                                             _ptr(scales), _stream(stream)))
    return out, scales


def fp8_scaled_mm_quantized_dual(a: torch.Tensor, b: torch.Tensor, scale_a: torch.Tensor,
                                 scale_b: torch.Tensor, recipe: int,
                                 bias: Optional[torch.Tensor] = None,
                                 out: Optional[torch.Tensor] = None,
                                 out_scales: Optional[torch.Tensor] = None,
                                 out_t: Optional[torch.Tensor] = None,
                                 out_t_scales: Optional[torch.Tensor] = None, stream=None):
    """fp8_scaled_mm writing both e4m3 forms of its result: 1x128 groups along
    n, and the transpose with 1x128 groups along m.

    Returns (codes (M, N), scales (N/128, M), transposed codes (N, M),
    transposed scales (M/128, N)); uint8 e4m3 codes, fp32 scales."""
    L = load_library()
    _need_cuda(a, b, scale_a, scale_b, bias)
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K:
        raise ValueError("a and b must share K")
    for t in (a, b):
        if t.dtype not in (torch.uint8, torch.float8_e4m3fn) or not t.is_contiguous():
            raise ValueError("a and b must be contiguous e4m3 (uint8 codes)")
    if bias is not None and (bias.dtype != torch.bfloat16 or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous bf16 tensor")
    dev = a.device
    if out is None:
        out = torch.empty((M, N), dtype=torch.uint8, device=dev)
    if out_scales is None:
        out_scales = torch.empty((N // 128, M), dtype=torch.float32, device=dev)
    if out_t is None:
        out_t = torch.empty((N, M), dtype=torch.uint8, device=dev)
    if out_t_scales is None:
        out_t_scales = torch.empty((M // 128, N), dtype=torch.float32, device=dev)
    if (out.numel() < M * N or out_t.numel() < M * N or
            out_scales.numel() < (N // 128) * M or out_t_scales.numel() < (M // 128) * N):
        raise ValueError("an output buffer is too small")
    _check(L.fp8_scaled_mm_quantized_dual(_ptr(a), _ptr(b), M, N, K, _ptr(scale_a),
                                          _ptr(scale_b), recipe, _ptr(bias), _ptr(out),
                                          _ptr(out_scales), _ptr(out_t), _ptr(out_t_scales),
                                          _stream(stream)))
    return out, out_scales, out_t, out_t_scales


# ----------------------------------------- tensorwise over row shards (ranks)

def _check_shard(x: torch.Tensor):
    _need_cuda(x)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 tensor with unit column stride")
    rows, cols = x.shape
    return rows, cols, (x.stride(0) if (rows > 1 and cols > 0) else cols)


def fp8_tensor_amax(x: torch.Tensor, out: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """max |x| of a bf16 shard, as a (1,) float32 device tensor."""
    L = load_library()
    rows, cols, ld = _check_shard(x)
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    _check(L.fp8_tensor_amax(_ptr(x), rows, cols, ld, _ptr(out), _stream(stream)))
    return out


def fp8_quantize_tensor_with_amax(x: torch.Tensor, amax: torch.Tensor,
                                  out: Optional[torch.Tensor] = None,
                                  scale: Optional[torch.Tensor] = None,
                                  stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Tensorwise cast of a shard with the scale of a given amax (device
    float, e.g. all-reduced over the ranks).  Returns (codes, scale (1,))."""
    L = load_library()
    rows, cols, ld = _check_shard(x)
    _need_cuda(amax)
    if amax.dtype != torch.float32 or amax.numel() < 1:
        raise ValueError("amax must be a float32 device tensor")
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty(1, dtype=torch.float32, device=x.device)
    _check(L.fp8_quantize_tensor_with_amax(_ptr(x), rows, cols, ld, _ptr(amax), _ptr(out),
                                           _ptr(scale), _stream(stream)))
    return out, scale


def allreduce_amax(amax: torch.Tensor, group=None) -> torch.Tensor:
    """The one exchange of the sharded tensorwise quantization: max over the
    ranks of the process group (in place), when one is initialised.  The
    group's backend must reduce tensors on amax's device (NCCL for CUDA)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return amax


def fp8_quantize_tensorwise_sharded(x: torch.Tensor, group=None,
                                    stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Tensorwise quantization of this rank's row shard of a tensor with the
    scale of the whole tensor: shard amax, all-reduce(MAX) over the group,
    cast.  Returns (codes, scale (1,)), the scale equal on every rank."""
    amax = fp8_tensor_amax(x, stream=stream)
    if stream is None:
        allreduce_amax(amax, group)
    else:
        with torch.cuda.stream(stream):   # the collective is ordered on that stream
            allreduce_amax(amax, group)
    return fp8_quantize_tensor_with_amax(x, amax, stream=stream)
