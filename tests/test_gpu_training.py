"""The training GEMMs of "improve fp8 blockwise gemm perf" (grad_input =
grad_output @ weight with the 1x128_128x128 recipe; grad_weight =
grad_output_t @ input with the 1x128_128x1 recipe) and the transposed
quantizer they need, against the oracle.

The transposed quantizer must equal the oracle's quantization of the
transposed matrix bit for bit; the GEMMs that consume its output must meet
the same per-element tolerance as the forward GEMM."""
import numpy as np
import pytest
import torch

import oracle
from fp8_scaled_matrix_b200 import fp8sm
from fp8_scaled_matrix_b200 import workloads as W
from helpers import MM, QUANT_GROUP, check_gemm, codes_np, out_f64, sample_rows

pytestmark = pytest.mark.gpu

QR = {"1x128": fp8sm.FP8_SCALE_BLOCK_1x128, "128x128": fp8sm.FP8_SCALE_BLOCK_128x128}


def oracle_quantize_t(x: torch.Tensor, group: str):
    """The oracle's quantization of x^T (x a CPU bf16 tensor)."""
    return oracle.quantize(np.ascontiguousarray(W.bf16_bits(x).T), QUANT_GROUP[group])


@pytest.mark.parametrize("group", ["1x128", "128x128"])
@pytest.mark.parametrize("rows,cols,pad", [
    (128, 8, 0),          # one row block, one 8-column chunk
    (256, 128, 0),
    (384, 200, 0),        # ragged column tile
    (1024, 1032, 24),     # several tiles, ragged last tile, strided input
    (128, 4096, 0),
])
def test_quantize_transposed_parity(group, rows, cols, pad):
    g = W.generator(rows * 7 + cols + pad)
    # a few entries far out, so that the groups' scales differ
    full = W.randn_bf16((rows, cols + pad), 1.0, g, outlier_frac=0.002, outlier_mult=50.0)
    x = full[:, :cols]
    xd = full.cuda()[:, :cols]
    q, s = fp8sm.fp8_quantize_transposed(xd, QR[group])
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    oq, osc = oracle_quantize_t(x.contiguous(), group)
    assert q.shape == (cols, rows)
    assert np.array_equal(codes_np(q), oq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), osc.view(np.uint32))


@pytest.mark.parametrize("group", ["1x128", "128x128"])
@pytest.mark.parametrize("rows,cols", [(16384, 2048), (12288, 1544)])
def test_quantize_transposed_parity_many_tiles_per_cta(group, rows, cols):
    """Enough 128 x 128 tiles that every persistent CTA walks its two-buffer
    tile ring several times (buffer reuse, phase flips), with a ragged last
    column tile in the second case; bit-exact against the oracle."""
    g = W.generator(rows + 3 * cols)
    x = W.randn_bf16((rows, cols), 1.0, g, outlier_frac=0.001, outlier_mult=50.0)
    q, s = fp8sm.fp8_quantize_transposed(x.cuda(), QR[group])
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    oq, osc = oracle_quantize_t(x, group)
    assert np.array_equal(codes_np(q), oq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), osc.view(np.uint32))


def test_quantize_transposed_matches_forward_quantize_of_transpose():
    """Same codes and scales as fp8_quantize applied to a materialised x^T."""
    g = W.generator(77)
    x = W.randn_bf16((512, 640), 1.0, g).cuda()
    for group in ("1x128", "128x128"):
        q1, s1 = fp8sm.fp8_quantize_transposed(x, QR[group])
        q2, s2 = fp8sm.fp8_quantize(x.t().contiguous(), QR[group])
        torch.cuda.synchronize()
        assert torch.equal(q1, q2)
        assert torch.equal(s1.view(torch.int32), s2.view(torch.int32))


def _grad_input(go, w, out_dtype):
    qa, sa = fp8sm.fp8_quantize(go.cuda(), fp8sm.FP8_SCALE_BLOCK_1x128)
    qb, sb = fp8sm.fp8_quantize_transposed(w.cuda(), fp8sm.FP8_SCALE_BLOCK_128x128)
    out = fp8sm.fp8_scaled_mm(qa, qb, sa, sb, fp8sm.FP8_MM_1x128_128x128, out_dtype=out_dtype)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    return qa, sa, qb, sb, out


def _grad_weight(go, x, out_dtype):
    qa, sa = fp8sm.fp8_quantize_transposed(go.cuda(), fp8sm.FP8_SCALE_BLOCK_1x128)
    qb, sb = fp8sm.fp8_quantize_transposed(x.cuda(), fp8sm.FP8_SCALE_BLOCK_1x128)
    out = fp8sm.fp8_scaled_mm(qa, qb, sa, sb, fp8sm.FP8_MM_1x128_128x1, out_dtype=out_dtype)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    return qa, sa, qb, sb, out


@pytest.mark.parametrize("M,N_out,K_in", [(256, 384, 512), (300, 256, 1040)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_grad_input_parity(M, N_out, K_in, out_dtype):
    g = W.generator(M + N_out + K_in)
    go = W.randn_bf16((M, N_out), 1.0, g)
    w = W.randn_bf16((N_out, K_in), 0.02, g)
    qa, sa, qb, sb, out = _grad_input(go, w, out_dtype)
    oqa, osa = oracle.quantize(W.bf16_bits(go), QUANT_GROUP["1x128"])
    oqb, osb = oracle_quantize_t(w, "128x128")
    assert np.array_equal(codes_np(qa), oqa) and np.array_equal(codes_np(qb), oqb)
    ref, mag = oracle.scaled_mm(oqa, oqb, osa, osb, MM["1x128_128x128"])
    check_gemm(out_f64(out), ref, mag, f"grad_input {M}x{N_out}x{K_in}")
    # the same product in exact arithmetic (the dequantized operands)
    exact = go.double().numpy() @ w.double().numpy()
    err = out_f64(out) - exact
    assert 10 * np.log10((exact ** 2).sum() / (err ** 2).sum()) >= 20.0


@pytest.mark.parametrize("M,N_out,K_in", [(384, 256, 272), (256, 144, 512)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_grad_weight_parity(M, N_out, K_in, out_dtype):
    g = W.generator(3 * M + N_out + K_in)
    go = W.randn_bf16((M, N_out), 1e-3, g)
    x = W.randn_bf16((M, K_in), 1.0, g)
    qa, sa, qb, sb, out = _grad_weight(go, x, out_dtype)
    oqa, osa = oracle_quantize_t(go, "1x128")
    oqb, osb = oracle_quantize_t(x, "1x128")
    assert np.array_equal(codes_np(qa), oqa) and np.array_equal(codes_np(qb), oqb)
    ref, mag = oracle.scaled_mm(oqa, oqb, osa, osb, MM["1x128_128x1"])
    check_gemm(out_f64(out), ref, mag, f"grad_weight {M}x{N_out}x{K_in}")


@pytest.mark.parametrize("which", ["grad_input", "grad_weight"])
def test_training_gemm_full_size_sampled(which):
    """The linear layer of the blockwise benchmark (16640 tokens, 8192 in,
    5120 out): grad_input (16640 x 8192, K = 5120) and grad_weight
    (5120 x 8192, K = 16640), checked on sampled output rows."""
    g = W.generator(4242 if which == "grad_input" else 4343)
    T, K_in, N_out = 16640, 8192, 5120
    if which == "grad_input":
        go = W.randn_bf16((T, N_out), 1.0, g)
        w = W.randn_bf16((N_out, K_in), 0.02, g)
        qa, sa, qb, sb, out = _grad_input(go, w, torch.bfloat16)
        oqa, osa = oracle.quantize(W.bf16_bits(go), QUANT_GROUP["1x128"])
        oqb, osb = oracle_quantize_t(w, "128x128")
        recipe = "1x128_128x128"
    else:
        go = W.randn_bf16((T, N_out), 1e-3, g)
        x = W.randn_bf16((T, K_in), 1.0, g)
        qa, sa, qb, sb, out = _grad_weight(go, x, torch.bfloat16)
        oqa, osa = oracle_quantize_t(go, "1x128")
        oqb, osb = oracle_quantize_t(x, "1x128")
        recipe = "1x128_128x1"
    assert np.array_equal(codes_np(qb), oqb)
    rows = sample_rows(out.shape[0], 24, seed=5)
    assert np.array_equal(codes_np(qa)[rows], oqa[rows])
    ref, mag = oracle.scaled_mm(oqa, oqb, osa, osb, MM[recipe], rows=rows)
    check_gemm(out_f64(out)[rows], ref, mag, f"{which} full size")
