"""Seeded synthetic inputs for the FP8 scaled GEMM workloads.

Only random numbers and shapes live here: no quantization, no scaling, no
GEMM arithmetic.  Both the CUDA path (through the bindings) and the CPU oracle
(in tests and the CPU-baseline leg of bench.py) are fed the same tensors from
this module.

Every tensor is drawn on the CPU from a ``torch.Generator`` in fp32 and then
rounded to bf16 (round-to-nearest-even), in the order listed for each
workload; the seed of workload ``i`` (0-based, in the order below) is
``1000 + i`` (``+100`` for the second (N, K) shape of the blockwise pair).

Workloads (shapes and distributions from the pages' benchmark and test
descriptions; no public dataset is involved):
  0 tensorwise  M=N=K=256, A,B ~ N(0,1)
  1 rowwise     M=N=K=4096, A ~ N(0,1) with 0.1% of entries x50 (outliers),
                W ~ N(0, 0.02^2), bias ~ N(0, 0.01^2)
  2 blockwise 1x128_128x128  M=16640, (N,K) in {(5120,8192), (8192,5120)},
                A ~ N(0,1), W ~ N(0, 0.02^2)
  3 blockwise 1x128_128x1    M=16640, same (N,K) pair,
                L ~ N(0, 1e-3^2) (M,K), R ~ N(0,1) stored (N,K)
  4 grouped     E=16, W ~ N(0, 0.02^2) (16,4096,4096), A ~ N(0,1) (32768,4096),
                group sizes: 2048 chunks of 16 rows, each chunk given to an
                expert drawn from p(r) ~ r^-1.2 over ranks r=1..16, ranks mapped
                to experts by a seeded permutation; offs = cumulative ends
  5 grad_input  the training GEMM grad_input = grad_output @ weight of the
                blockwise benchmark's linear layer (16640 tokens, 8192 in,
                5120 out): dY ~ N(0,1) (16640, 5120), W ~ N(0, 0.02^2)
                (5120, 8192) as stored; GEMM M=16640, N=8192, K=5120
  6 grad_weight grad_weight = grad_output_t @ input of the same layer:
                dY ~ N(0, 1e-3^2) (16640, 5120), X ~ N(0,1) (16640, 8192);
                GEMM M=5120, N=8192, K=16640
  7 grouped blockwise  the tensors of workload 4 (same seed), quantized with
                1x128 activation groups and per-expert 128x128 weight tiles
  8 linear chain  two blockwise (1x128_128x128) linears back to back, the
                first one's output quantized in its GEMM epilogue and fed to
                the second as its 1x128 activation: 16640 tokens, 8192 -> 5120
                -> 8192; X ~ N(0,1) (16640, 8192), W1 ~ N(0, 0.02^2)
                (5120, 8192), W2 ~ N(0, 0.02^2) (8192, 5120) as stored
  9 mxfp8       the tensors of workload 2 (same seeds, both (N, K) shapes),
                quantized MXFP8 (E8M0 scale per 32 elements of K)
 10 linear chain, MXFP8  the tensors of workload 8, every operand MXFP8 and
                the first GEMM writing MXFP8
 11 grouped MXFP8  the tensors of workload 4 (same seed), MXFP8 throughout
 12 grouped grad_input  the MoE layer's backward dX_g = dY_g @ W_g with the
                1x128_128x128 recipe: dY ~ N(0,1) (32768, 4096) (drawn as
                workload 4's activations, same seed and group split), W =
                workload 4's experts (16, 4096 out, 4096 in); GEMM M=32768,
                N=4096 (in), K=4096 (out)
 13 grouped grad_weight  the MoE layer's per-expert weight gradient
                dW_g = dY_g^T @ X_g with the 1x128_128x1 recipe over each
                group's tokens: dY ~ N(0, 1e-3^2) (32768, 4096 out), X ~ N(0,1)
                (32768, 4096 in), workload 4's group split; GEMM M=4096 (out),
                N=4096 (in), K=32768 tokens in 16 groups
 14 linear chain training step  workload 8's chain forward and backward
                with blockwise scaling throughout: X ~ N(0,1) (16640, 8192),
                W1 ~ N(0, 0.02^2) (5120, 8192), W2 ~ N(0, 0.02^2) (8192, 5120),
                dY2 ~ N(0, 1e-3^2) (16640, 8192) the gradient arriving at the
                chain's output; six GEMMs of 16640 x 5120 x 8192 each:
                Y1 = X W1^T, Y2 = Y1 W2^T, dY1 = dY2 W2, dX = dY1 W1 (all
                1x128_128x128), dW1 = dY1^T X, dW2 = dY2^T Y1 (1x128_128x1,
                contracting over the tokens); T must be a multiple of 128
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np
import torch

WORKLOAD_NAMES = [
    "tensorwise_256",
    "rowwise_4096",
    "blockwise_1x128_128x128",
    "blockwise_1x128_128x1",
    "grouped_e16",
    "grad_input_1x128_128x128",
    "grad_weight_1x128_128x1",
    "grouped_e16_blockwise",
    "linear_chain_1x128_128x128",
    "mxfp8",
    "linear_chain_mxfp8",
    "grouped_e16_mxfp8",
    "grouped_e16_grad_input",
    "grouped_e16_grad_weight",
    "linear_chain_train_1x128",
]


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def randn_bf16(shape, std: float, g: torch.Generator,
               outlier_frac: float = 0.0, outlier_mult: float = 1.0) -> torch.Tensor:
    """N(0, std^2) in fp32, optional outliers (a seeded random subset of exactly
    round(frac * numel) entries multiplied by ``outlier_mult``), then bf16."""
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if outlier_frac > 0.0:
        n = int(round(outlier_frac * x.numel()))
        idx = torch.randperm(x.numel(), generator=g)[:n]
        x.view(-1)[idx] *= outlier_mult
    return x.to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a CPU bf16 tensor (no copy of the values' meaning)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def zipf_group_sizes(total_rows: int, E: int, chunk: int, s: float,
                     g: torch.Generator) -> torch.Tensor:
    """Group sizes (multiples of ``chunk``) summing to ``total_rows``."""
    assert total_rows % chunk == 0
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    p = ranks.pow(-s)
    p = p / p.sum()
    n_chunks = total_rows // chunk
    chunk_rank = torch.multinomial(p, n_chunks, replacement=True, generator=g)
    perm = torch.randperm(E, generator=g)
    expert = perm[chunk_rank]
    return torch.bincount(expert, minlength=E).to(torch.int64) * chunk


def offsets_from_sizes(sizes) -> torch.Tensor:
    """Cumulative end offsets, int32."""
    sizes = torch.as_tensor(sizes, dtype=torch.int64)
    return torch.cumsum(sizes, 0).to(torch.int32)


@dataclass
class Workload:
    name: str
    # tensor | row | 1x128_128x128 | 1x128_128x1 | grouped | grouped_blockwise |
    # grad_input | grad_weight | chain | mxfp8 | chain_mx | grouped_mx |
    # grouped_grad_input | grouped_grad_weight | chain_train
    recipe: str
    M: int
    N: int
    K: int
    # GEMM sizes M, N, K; the bf16 operands as a caller holds them (CPU):
    #   a  (M, K); grad_weight: (K, M) (grad_output, tokens x out)
    #   b  (N, K) or (E, N, K); grad_input: (K, N) (the weight as stored);
    #      grad_weight: (K, N) (the layer input, tokens x in);
    #      grouped_grad_input: (E, K, N) (the experts as stored, out x in);
    #   grouped_grad_weight: a (K, M) = dY (tokens x out), b (K, N) = X
    #      (tokens x in), K = tokens split by offs
    a: torch.Tensor
    b: torch.Tensor
    bias: Optional[torch.Tensor] = None   # bf16 (N,) CPU
    offs: Optional[torch.Tensor] = None   # int32 (E,) CPU
    E: int = 0
    seed: int = 0
    extra: Dict = field(default_factory=dict)

    @property
    def flops(self) -> int:
        f = 2 * self.M * self.N * self.K
        if self.recipe == "chain_train":   # six GEMMs of the same size
            return 6 * f
        if "b2" in self.extra:   # the chain's second GEMM: (M, N) @ b2^T
            n2, k2 = self.extra["b2"].shape
            f += 2 * self.M * n2 * k2
        return f


def make_workload(index: int, shape_index: int = 0, scale_down: int = 1) -> Workload:
    """Build workload ``index`` (see module doc).  ``scale_down`` > 1 divides M
    (and, for the grouped case, the token count) to make a smaller case with
    the same distributions; sizes stay multiples of 16."""
    name = WORKLOAD_NAMES[index]
    if index == 7:  # workload 4's tensors, blockwise-scaled
        wl = make_workload(4, shape_index, scale_down)
        wl.name, wl.recipe = name, "grouped_blockwise"
        return wl
    if index == 13:
        ref = make_workload(4, shape_index, scale_down)
        T, D = ref.a.shape
        E = ref.E
        seed = 1000 + index + 100 * shape_index
        g = generator(seed)
        dy = randn_bf16((T, D), 1e-3, g)
        x = randn_bf16((T, D), 1.0, g)
        return Workload(name, "grouped_grad_weight", D, D, T, dy, x, offs=ref.offs, E=E,
                        seed=seed)
    if index == 12:  # workload 4's tensors as (dY, W) of the backward
        wl = make_workload(4, shape_index, scale_down)
        E, Nout, Kin = wl.b.shape
        wl.name, wl.recipe = name, "grouped_grad_input"
        wl.N, wl.K = Kin, Nout
        return wl
    if index == 11:  # workload 4's tensors, MXFP8
        wl = make_workload(4, shape_index, scale_down)
        wl.name, wl.recipe = name, "grouped_mx"
        return wl
    if index == 10:  # workload 8's tensors, MXFP8 throughout
        wl = make_workload(8, shape_index, scale_down)
        wl.name, wl.recipe = name, "chain_mx"
        return wl
    if index == 9:  # workload 2's tensors, MXFP8
        wl = make_workload(2, shape_index, scale_down)
        wl.name, wl.recipe = name, "mxfp8"
        return wl
    seed = 1000 + index + 100 * shape_index
    g = generator(seed)
    if index == 0:
        M = N = K = 256
        a = randn_bf16((M, K), 1.0, g)
        b = randn_bf16((N, K), 1.0, g)
        return Workload(name, "tensor", M, N, K, a, b, seed=seed)
    if index == 1:
        M = N = K = 4096
        M //= scale_down
        a = randn_bf16((M, K), 1.0, g, outlier_frac=0.001, outlier_mult=50.0)
        b = randn_bf16((N, K), 0.02, g)
        bias = randn_bf16((N,), 0.01, g)
        return Workload(name, "row", M, N, K, a, b, bias=bias, seed=seed)
    if index in (2, 3):
        NK = [(5120, 8192), (8192, 5120)][shape_index]
        M = 16640 // scale_down
        M -= M % 16
        N, K = NK
        if index == 2:
            a = randn_bf16((M, K), 1.0, g)
            b = randn_bf16((N, K), 0.02, g)
            return Workload(name, "1x128_128x128", M, N, K, a, b, seed=seed)
        a = randn_bf16((M, K), 1e-3, g)
        b = randn_bf16((N, K), 1.0, g)
        return Workload(name, "1x128_128x1", M, N, K, a, b, seed=seed)
    if index == 4:
        E, N, K = 16, 4096, 4096
        T = 32768 // scale_down
        b = randn_bf16((E, N, K), 0.02, g)
        a = randn_bf16((T, K), 1.0, g)
        sizes = zipf_group_sizes(T, E, 16, 1.2, g)
        offs = offsets_from_sizes(sizes)
        return Workload(name, "grouped", T, N, K, a, b, offs=offs, E=E, seed=seed)
    if index in (5, 6):
        T, K_in, N_out = 16640 // scale_down, 8192, 5120
        T -= T % 128
        if index == 5:
            dy = randn_bf16((T, N_out), 1.0, g)
            w = randn_bf16((N_out, K_in), 0.02, g)
            return Workload(name, "grad_input", T, K_in, N_out, dy, w, seed=seed)
        dy = randn_bf16((T, N_out), 1e-3, g)
        x = randn_bf16((T, K_in), 1.0, g)
        return Workload(name, "grad_weight", N_out, K_in, T, dy, x, seed=seed)
    if index == 8:
        T, D, F = 16640 // scale_down, 8192, 5120
        T -= T % 16
        x = randn_bf16((T, D), 1.0, g)
        w1 = randn_bf16((F, D), 0.02, g)
        w2 = randn_bf16((D, F), 0.02, g)
        return Workload(name, "chain", T, F, D, x, w1, seed=seed, extra={"b2": w2})
    if index == 14:
        T, D, F = 16640 // scale_down, 8192, 5120
        T = max(128, T - T % 128)
        x = randn_bf16((T, D), 1.0, g)
        w1 = randn_bf16((F, D), 0.02, g)
        w2 = randn_bf16((D, F), 0.02, g)
        dy2 = randn_bf16((T, D), 1e-3, g)
        return Workload(name, "chain_train", T, F, D, x, w1, seed=seed,
                        extra={"b2": w2, "dy": dy2})
    raise ValueError(f"unknown workload {index}")


def small_case(recipe: str, M: int, N: int, K: int, seed: int,
               a_std: float = 1.0, b_std: float = 0.02, bias: bool = False,
               E: int = 0, group_sizes: Optional[List[int]] = None) -> Workload:
    """A parity-test case of arbitrary (ragged) size with the workloads'
    distributions."""
    g = generator(seed)
    if recipe == "grouped":
        assert group_sizes is not None and len(group_sizes) == E
        b = randn_bf16((E, N, K), b_std, g)
        a = randn_bf16((M, K), a_std, g)
        offs = offsets_from_sizes(group_sizes)
        assert int(offs[-1]) == M
        return Workload("small_grouped", recipe, M, N, K, a, b, offs=offs, E=E, seed=seed)
    a = randn_bf16((M, K), a_std, g)
    b = randn_bf16((N, K), b_std, g)
    bb = randn_bf16((N,), 0.01, g) if bias else None
    return Workload(f"small_{recipe}", recipe, M, N, K, a, b, bias=bb, seed=seed)
