"""Shared helpers for the parity tests: move workload tensors between the
oracle (numpy bit patterns) and the CUDA path (torch device tensors)."""
import numpy as np
import torch

import oracle
from fp8_scaled_matrix_b200 import workloads as W

QUANT_GROUP = {"tensor": oracle.GROUP_TENSOR, "row": oracle.GROUP_ROW,
               "1x128": oracle.GROUP_1x128, "128x128": oracle.GROUP_128x128}
MM = {"tensor": oracle.MM_TENSOR_TENSOR, "row": oracle.MM_ROW_ROW,
      "1x128_128x128": oracle.MM_1x128_128x128, "1x128_128x1": oracle.MM_1x128_128x1}
# (A quantize group, B quantize group) of each GEMM recipe
OPERAND_GROUPS = {"tensor": ("tensor", "tensor"), "row": ("row", "row"),
                  "1x128_128x128": ("1x128", "128x128"),
                  "1x128_128x1": ("1x128", "1x128")}


def to_dev(t, dev="cuda"):
    return t.to(dev)


def codes_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.uint8).numpy()


def out_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def check_gemm(out, ref, mag, what=""):
    ok = oracle.within_tolerance(out, ref, mag)
    if not ok.all():
        bad = np.argwhere(~ok)
        i, j = bad[0]
        raise AssertionError(
            f"{what}: {bad.shape[0]} of {ok.size} elements out of tolerance; first at "
            f"({i},{j}) out={out[i, j]!r} ref={ref[i, j]!r} mag={mag[i, j]!r}")


def sample_rows(M: int, n: int = 48, seed: int = 0, tile: int = 128) -> np.ndarray:
    """Rows straddling tile boundaries plus seeded random rows."""
    fixed = {0, 1, M - 1, M - 2}
    for b in range(tile, M, tile * max(1, (M // tile) // 8)):
        fixed.update({b - 1, b})
    rng = np.random.default_rng(seed)
    extra = rng.choice(M, size=min(M, n), replace=False)
    rows = sorted(r for r in fixed.union(int(x) for x in extra) if 0 <= r < M)
    return np.array(rows, dtype=np.int64)
