"""The seeded synthetic inputs (CPU): every workload builds with the shapes,
recipe and FLOP count its description states, the same seed gives the same
tensors, and the MoE group split has the stated structure (chunks of 16 rows,
16 experts, cumulative end offsets ending at the token count)."""
import numpy as np
import pytest
import torch

from fp8_scaled_matrix_b200 import workloads as W

# (index, scale_down) -> (recipe, M, N, K) of the reduced case
EXPECT = {
    0: ("tensor", 256, 256, 256),
    1: ("row", 4096, 4096, 4096),
    2: ("1x128_128x128", 128, 5120, 8192),     # 16640 / 128, down to a multiple of 16
    3: ("1x128_128x1", 128, 5120, 8192),
    5: ("grad_input", 128, 8192, 5120),
    6: ("grad_weight", 5120, 8192, 128),
    8: ("chain", 128, 5120, 8192),
    9: ("mxfp8", 128, 5120, 8192),
    10: ("chain_mx", 128, 5120, 8192),
    14: ("chain_train", 128, 5120, 8192),
}


@pytest.mark.parametrize("idx", sorted(EXPECT))
def test_shapes_recipes_and_flops(idx):
    sd = 1 if idx in (0, 1) else 128
    wl = W.make_workload(idx, 0, scale_down=sd)
    recipe, M, N, K = EXPECT[idx]
    assert (wl.recipe, wl.M, wl.N, wl.K) == (recipe, M, N, K)
    assert wl.a.dtype == torch.bfloat16 and wl.b.dtype == torch.bfloat16
    per_gemm = 2 * M * N * K
    if recipe == "chain_train":
        assert wl.flops == 6 * per_gemm
        T, D, F = M, K, N
        assert T % 128 == 0
        assert wl.a.shape == (T, D) and wl.b.shape == (F, D)
        assert wl.extra["b2"].shape == (D, F) and wl.extra["dy"].shape == (T, D)
    elif recipe in ("chain", "chain_mx"):
        assert wl.flops == per_gemm + 2 * M * wl.extra["b2"].shape[0] * N
    else:
        assert wl.flops == per_gemm


def test_same_seed_same_tensors():
    a = W.make_workload(2, 1, scale_down=128)
    b = W.make_workload(2, 1, scale_down=128)
    assert a.seed == b.seed == 1102
    assert torch.equal(a.a.view(torch.int16), b.a.view(torch.int16))
    assert torch.equal(a.b.view(torch.int16), b.b.view(torch.int16))
    c = W.make_workload(2, 0, scale_down=128)
    assert not torch.equal(a.b.view(torch.int16)[:10], c.b.view(torch.int16)[:10])


def test_rowwise_outliers_and_distributions():
    wl = W.make_workload(1, 0)
    a = wl.a.float()
    # 0.1 % of A's entries scaled by 50: about that many lie beyond 6 sigma of N(0,1)
    n_out = int((a.abs() > 6.0).sum())
    assert 0.6 * 16777 < n_out <= 16777
    assert abs(float(wl.b.float().std()) - 0.02) < 1e-3
    assert wl.bias is not None and abs(float(wl.bias.float().std()) - 0.01) < 2e-3


@pytest.mark.parametrize("idx", [4, 12, 13])
def test_moe_group_split(idx):
    wl = W.make_workload(idx, 0, scale_down=8)
    offs = wl.offs.numpy().astype(np.int64)
    assert wl.offs.dtype == torch.int32 and offs.size == 16
    sizes = np.diff(np.concatenate([[0], offs]))
    assert (sizes >= 0).all() and (sizes % 16 == 0).all()
    tokens = wl.K if idx == 13 else wl.M
    assert offs[-1] == tokens == 32768 // 8
    # ranks drawn from p(r) ~ r^-1.2: the largest group holds the most chunks
    assert sizes.max() > 2 * np.median(sizes[sizes > 0])
