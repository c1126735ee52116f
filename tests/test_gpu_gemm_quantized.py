"""The GEMM whose epilogue quantizes its own result (fp8_scaled_mm_quantized),
and the chain of two linears it enables.

Two checks per case.  (1) Against the oracle, independently: the oracle
quantizes the same seeded inputs and computes the fp64 GEMM; the dequantized
kernel output (code * scale) must be within the GEMM tolerance plus half an
e4m3 step of it.  (2) A property of the kernel's own output: its codes and
scales are exactly the 1x128 quantization (the scale and cast steps of
"per-token scaling for fp8 linear", Highlights) of the fp32 result that the
same GEMM writes when asked for fp32 output -- the oracle's fp32-input
quantizer applied to that fp32 result must reproduce them bit for bit.  (2) is
what makes the fused quantize bit-exact; the rounding of the fp32 GEMM itself
differs from the fp64 reference, so codes cannot be compared with an oracle
quantize of the fp64 result."""
import numpy as np
import pytest
import torch

import oracle
from fp8_scaled_matrix_b200 import fp8sm
from fp8_scaled_matrix_b200 import workloads as W
from helpers import MM, OPERAND_GROUPS, QUANT_GROUP, sample_rows

pytestmark = pytest.mark.gpu

MMR = {"tensor": fp8sm.FP8_MM_TENSOR_TENSOR, "row": fp8sm.FP8_MM_ROW_ROW,
       "1x128_128x128": fp8sm.FP8_MM_1x128_128x128, "1x128_128x1": fp8sm.FP8_MM_1x128_128x1}


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Value of each e4m3 code (OCP FP8 E4M3: bias 7, no infinities)."""
    c = codes.astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    v = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    return sign * v


def operands(recipe, M, N, K, seed, bias):
    b_std = 0.02 if recipe != "1x128_128x1" else 1.0
    a_std = 1.0 if recipe != "1x128_128x1" else 1e-3
    wl = W.small_case(recipe, M, N, K, seed=seed, a_std=a_std, b_std=b_std, bias=bias)
    ga, gb = OPERAND_GROUPS[recipe]
    qa, sa = oracle.quantize(W.bf16_bits(wl.a), QUANT_GROUP[ga])
    qb, sb = oracle.quantize(W.bf16_bits(wl.b), QUANT_GROUP[gb])
    return wl, qa, sa, qb, sb


def run_both(qa, sa, qb, sb, recipe, bias):
    a, b = torch.from_numpy(qa).cuda(), torch.from_numpy(qb).cuda()
    sad, sbd = torch.from_numpy(sa).cuda(), torch.from_numpy(sb).cuda()
    bd = None if bias is None else bias.cuda()
    y = fp8sm.fp8_scaled_mm(a, b, sad, sbd, MMR[recipe], bias=bd, out_dtype=torch.float32)
    q, s = fp8sm.fp8_scaled_mm_quantized(a, b, sad, sbd, MMR[recipe], bias=bd)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    return y.cpu().numpy(), q.cpu().numpy(), s.cpu().numpy()


def check_exact(y, q, s, what):
    """q, s (scales (N/128, M)) are the 1x128 quantization of the fp32 y: the
    oracle's fp32-input quantizer is run on the kernel's own fp32 result and
    must give the same codes and scales bit for bit."""
    M, N = y.shape
    q_want, s_want = oracle.quantize_f32(np.ascontiguousarray(y.astype(np.float32)),
                                         oracle.GROUP_1x128)
    s = np.ascontiguousarray(s).reshape(-1)[:s_want.size]
    bad_s = np.argwhere(s_want.view(np.uint32) != s.view(np.uint32))
    assert bad_s.size == 0, f"{what}: {len(bad_s)} scales differ, first {bad_s[0]}"
    bad = np.argwhere(q_want != q)
    assert bad.size == 0, (f"{what}: {len(bad)} codes differ, first {bad[0]} "
                           f"kernel={q[tuple(bad[0])]:#x} want={q_want[tuple(bad[0])]:#x}")


def check_against_fp64(q, s, ref, mag, what):
    M, N = q.shape
    scale = s.reshape(N // 128, M).T.repeat(128, axis=1).astype(np.float64)
    deq = e4m3_decode(q) * scale
    # the GEMM tolerance for the fp32 value y, then the rounding of y to e4m3:
    # half a step, 2^-4 |y| for normal codes and 2^-10 scale below them
    gemm_tol = 1e-2 * np.abs(ref) + 1e-3 * mag
    tol = gemm_tol + 2.0 ** -4 * (np.abs(ref) + gemm_tol) + scale * 2.0 ** -9
    err = np.abs(deq - ref)
    bad = np.argwhere(err > tol)
    assert bad.size == 0, (f"{what}: {len(bad)} elements out of tolerance, first "
                           f"{bad[0]} deq={deq[tuple(bad[0])]} ref={ref[tuple(bad[0])]}")


CASES = [
    # recipe, M, N, K, bias
    ("tensor", 300, 256, 528, True),
    ("tensor", 1, 128, 16, False),
    ("row", 129, 512, 4096, True),
    ("row", 300, 384, 528, False),           # last tile half empty along n
    ("row", 4096, 4096, 256, True),          # last wave split into 128-wide items
    ("row", 7, 128, 32, True),
    ("1x128_128x128", 260, 384, 384, True),
    ("1x128_128x128", 1100, 2304, 1024, False),
    ("1x128_128x1", 130, 512, 256, False),
    ("1x128_128x1", 64, 128, 128, True),
    ("1x128_128x1", 2304, 4352, 512, False),
]


@pytest.mark.parametrize("recipe,M,N,K,bias", CASES)
def test_quantized_output_parity(recipe, M, N, K, bias):
    seed = M * 17 + N * 5 + K + 3
    wl, qa, sa, qb, sb = operands(recipe, M, N, K, seed, bias)
    y, q, s = run_both(qa, sa, qb, sb, recipe, wl.bias)
    what = f"{recipe} {M}x{N}x{K}"
    check_exact(y, q, s, what)
    rows = sample_rows(M, n=64, seed=seed)
    bias_bits = None if wl.bias is None else W.bf16_bits(wl.bias)
    ref, mag = oracle.scaled_mm(qa, qb, sa, sb, MM[recipe], bias_bits=bias_bits, rows=rows)
    check_against_fp64(q[rows], s.reshape(N // 128, M)[:, rows].copy(), ref, mag, what)


@pytest.mark.parametrize("recipe", ["row", "1x128_128x128"])
def test_quantized_output_zero_groups(recipe):
    """Rows of a that are all zero give all-zero groups (no bias): code 0 with
    the floor scale 1e-12/448; rows that are not zero are unaffected."""
    M, N, K = 200, 256, 256
    wl, qa, sa, qb, sb = operands(recipe, M, N, K, 11, False)
    qa[:3] = 0
    qa[150] = 0
    y, q, s = run_both(qa, sa, qb, sb, recipe, None)
    check_exact(y, q, s, f"{recipe} zero rows")
    s2 = s.reshape(N // 128, M)
    floor = np.float32(np.float32(1e-12) / np.float32(448.0))
    for r in (0, 1, 2, 150):
        assert (q[r] == 0).all()
        assert (s2[:, r] == floor).all()


def test_quantized_output_constant_group():
    """A group whose values are all equal maps to code 0x7e (448) exactly."""
    M, N, K = 64, 128, 128
    a = torch.zeros(M, K, dtype=torch.uint8, device="cuda")
    b = torch.zeros(N, K, dtype=torch.uint8, device="cuda")
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    bias = torch.full((N,), -3.0, dtype=torch.bfloat16, device="cuda")
    q, s = fp8sm.fp8_scaled_mm_quantized(a, b, one, one, fp8sm.FP8_MM_TENSOR_TENSOR,
                                         bias=bias)
    torch.cuda.synchronize()
    assert (q.cpu() == 0xFE).all()          # -448
    assert torch.equal(s.cpu(), torch.full((1, M), float(np.float32(3.0) / np.float32(448.0)),
                                              dtype=torch.float32))


QR = {"row": fp8sm.FP8_SCALE_ROW, "1x128": fp8sm.FP8_SCALE_BLOCK_1x128,
      "128x128": fp8sm.FP8_SCALE_BLOCK_128x128}


@pytest.mark.parametrize("idx,shape_index", [(1, 0), (2, 0), (3, 1)])
def test_quantized_output_full_size_sampled(idx, shape_index):
    """Workload shapes (rowwise 4096^3 with bias; blockwise 16640x5120x8192 and
    16640x8192x5120): the quantized output against the oracle's quantizer on
    sampled rows of the same kernel schedule's fp32 result."""
    wl = W.make_workload(idx, shape_index)
    ga, gb = OPERAND_GROUPS[wl.recipe]
    a, b = wl.a.cuda(), wl.b.cuda()
    qa, sa = fp8sm.fp8_quantize(a, QR[ga])
    qb, sb = fp8sm.fp8_quantize(b, QR[gb])
    del a, b
    bd = None if wl.bias is None else wl.bias.cuda()
    q, s = fp8sm.fp8_scaled_mm_quantized(qa, qb, sa, sb, MMR[wl.recipe], bias=bd)
    y = fp8sm.fp8_scaled_mm(qa, qb, sa, sb, MMR[wl.recipe], bias=bd, out_dtype=torch.float32)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    rows = torch.from_numpy(sample_rows(wl.M, n=96, seed=idx)).cuda()
    ys = y.index_select(0, rows).cpu().numpy()
    qs = q.index_select(0, rows).cpu().numpy()
    ss = s.index_select(1, rows).cpu().numpy()
    check_exact(ys, qs, ss, f"{wl.name} full size")


def test_linear_chain_against_oracle():
    """Two blockwise linears chained through the quantized output (the
    linear-chain workload at full width, sampled rows): X -> GPU quantize ->
    GEMM1 quantized -> GEMM2, against the oracle's chain on the same inputs
    (quantize, fp64 GEMM1 rounded to fp32, 1x128 quantize, fp64 GEMM2); and the
    chain's SQNR against the unquantized fp64 product (>= 20 dB, the MoE
    handler's output threshold)."""
    wl = W.make_workload(8)
    f = fp8sm
    x, w1, w2 = wl.a.cuda(), wl.b.cuda(), wl.extra["b2"].cuda()
    qx, sx = f.fp8_quantize(x, f.FP8_SCALE_BLOCK_1x128)
    q1, s1 = f.fp8_quantize(w1, f.FP8_SCALE_BLOCK_128x128)
    q2, s2 = f.fp8_quantize(w2, f.FP8_SCALE_BLOCK_128x128)
    r = f.FP8_MM_1x128_128x128
    y1q, y1s = f.fp8_scaled_mm_quantized(qx, q1, sx, s1, r)
    out = f.fp8_scaled_mm(y1q, q2, y1s, s2, r, out_dtype=torch.float32)
    torch.cuda.synchronize()
    f.check_device_status()
    rows = sample_rows(wl.M, 40, seed=8)
    G = oracle.GROUP_128x128
    oqx, osx = oracle.quantize(W.bf16_bits(wl.a), oracle.GROUP_1x128)
    oq1, os1 = oracle.quantize(W.bf16_bits(wl.b), G)
    oq2, os2 = oracle.quantize(W.bf16_bits(wl.extra["b2"]), G)
    y1, _ = oracle.scaled_mm(oqx, oq1, osx, os1, oracle.MM_1x128_128x128, rows=rows)
    oy1q, oy1s = oracle.quantize_f32(y1.astype(np.float32), oracle.GROUP_1x128)
    ref, mag = oracle.scaled_mm(oy1q, oq2, oy1s, os2, oracle.MM_1x128_128x128)
    got = out.cpu().numpy().astype(np.float64)[rows]
    ok = oracle.within_tolerance(got, ref, mag)
    assert ok.all(), f"chain: {int((~ok).sum())} of {ok.size} out of tolerance"
    xs = wl.a.double().numpy()[rows]
    exact = (xs @ wl.b.double().numpy().T) @ wl.extra["b2"].double().numpy().T
    err = got - exact
    sqnr = 10 * np.log10((exact ** 2).sum() / (err ** 2).sum())
    assert sqnr >= 20.0, sqnr


def test_linear_chain_backward_grad_input_against_oracle():
    """The chain's backward through the grad_input GEMMs ("improve fp8 blockwise
    gemm perf": grad_input = grad_output @ weight, 1x128_128x128): dY2 ->
    dY1 = dY2 @ W2 with dY1 quantized 1x128 in that GEMM's epilogue -> dX =
    dY1 @ W1, each weight quantized transposed (128x128); sampled rows against
    the oracle's chain (1x128 quantize, fp64 GEMM rounded to fp32, 1x128
    quantize, fp64 GEMM) and SQNR >= 20 dB against the unquantized product."""
    wl = W.make_workload(8)          # X (T, 8192), W1 (5120, 8192), W2 (8192, 5120)
    f = fp8sm
    g = W.generator(88)
    T = wl.M
    dy2 = W.randn_bf16((T, 8192), 1.0, g)
    w1, w2 = wl.b, wl.extra["b2"]
    r = f.FP8_MM_1x128_128x128
    qd, sd = f.fp8_quantize(dy2.cuda(), f.FP8_SCALE_BLOCK_1x128)
    q2t, s2t = f.fp8_quantize_transposed(w2.cuda(), f.FP8_SCALE_BLOCK_128x128)   # W2^T (5120, 8192)
    q1t, s1t = f.fp8_quantize_transposed(w1.cuda(), f.FP8_SCALE_BLOCK_128x128)   # W1^T (8192, 5120)
    dy1q, dy1s = f.fp8_scaled_mm_quantized(qd, q2t, sd, s2t, r)                  # (T, 5120)
    dx = f.fp8_scaled_mm(dy1q, q1t, dy1s, s1t, r, out_dtype=torch.float32)       # (T, 8192)
    torch.cuda.synchronize()
    f.check_device_status()
    rows = sample_rows(T, 32, seed=18)
    G = oracle.GROUP_128x128
    oqd, osd = oracle.quantize(W.bf16_bits(dy2), oracle.GROUP_1x128)
    oq2t, os2t = oracle.quantize(np.ascontiguousarray(W.bf16_bits(w2).T), G)
    oq1t, os1t = oracle.quantize(np.ascontiguousarray(W.bf16_bits(w1).T), G)
    y1, _ = oracle.scaled_mm(oqd, oq2t, osd, os2t, oracle.MM_1x128_128x128, rows=rows)
    oy1q, oy1s = oracle.quantize_f32(y1.astype(np.float32), oracle.GROUP_1x128)
    ref, mag = oracle.scaled_mm(oy1q, oq1t, oy1s, os1t, oracle.MM_1x128_128x128)
    got = dx.cpu().numpy().astype(np.float64)[rows]
    ok = oracle.within_tolerance(got, ref, mag)
    assert ok.all(), f"backward chain: {int((~ok).sum())} of {ok.size} out of tolerance"
    exact = (dy2.double().numpy()[rows] @ w2.double().numpy()) @ w1.double().numpy()
    err = got - exact
    assert 10 * np.log10((exact ** 2).sum() / (err ** 2).sum()) >= 20.0


# ------------------------------------------- both e4m3 forms from one GEMM
# fp8_scaled_mm_quantized_dual writes the 1x128-along-n form (for the next
# grad_input GEMM) and the transposed 1x128-along-m form (for the grad_weight
# GEMM, 1x128_128x1 with the tokens as K) of the same fp32 result.

def run_dual(qa, sa, qb, sb, bias):
    a, b = torch.from_numpy(qa).cuda(), torch.from_numpy(qb).cuda()
    sad, sbd = torch.from_numpy(sa).cuda(), torch.from_numpy(sb).cuda()
    bd = None if bias is None else bias.cuda()
    r = fp8sm.FP8_MM_1x128_128x128
    y = fp8sm.fp8_scaled_mm(a, b, sad, sbd, r, bias=bd, out_dtype=torch.float32)
    q, s, qt, st = fp8sm.fp8_scaled_mm_quantized_dual(a, b, sad, sbd, r, bias=bd)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    return tuple(t.cpu().numpy() for t in (y, q, s, qt, st))


DUAL_CASES = [
    # M, N, K, bias  (M, N, K multiples of 128)
    (128, 128, 128, False),
    (256, 384, 384, True),           # last tile half empty along n
    (1024, 2304, 1024, False),
    (384, 640, 256, True),
    (2304, 4352, 512, False),        # last wave split into 128-wide items
]


@pytest.mark.parametrize("M,N,K,bias", DUAL_CASES)
def test_dual_output_parity(M, N, K, bias):
    seed = M * 13 + N * 7 + K
    wl, qa, sa, qb, sb = operands("1x128_128x128", M, N, K, seed, bias)
    y, q, s, qt, st = run_dual(qa, sa, qb, sb, wl.bias)
    what = f"dual {M}x{N}x{K}"
    check_exact(y, q, s, what + " rows")
    check_exact(np.ascontiguousarray(y.T), qt, st, what + " transposed")
    bias_bits = None if wl.bias is None else W.bf16_bits(wl.bias)
    ref, mag = oracle.scaled_mm(qa, qb, sa, sb, MM["1x128_128x128"], bias_bits=bias_bits)
    check_against_fp64(q, s, ref, mag, what + " rows")
    check_against_fp64(qt, st, np.ascontiguousarray(ref.T), np.ascontiguousarray(mag.T),
                       what + " transposed")


def test_dual_output_rejects_other_recipes_and_shapes():
    z = torch.zeros(128, 128, dtype=torch.uint8, device="cuda")
    one = torch.ones(1, 128, device="cuda")
    with pytest.raises(fp8sm.Fp8Unsupported):
        fp8sm.fp8_scaled_mm_quantized_dual(z, z, one, one, fp8sm.FP8_MM_ROW_ROW)
    a = torch.zeros(100, 128, dtype=torch.uint8, device="cuda")
    with pytest.raises(fp8sm.Fp8ValueError):
        fp8sm.fp8_scaled_mm_quantized_dual(a, z, torch.ones(1, 100, device="cuda"),
                                           torch.ones(1, 1, device="cuda"),
                                           fp8sm.FP8_MM_1x128_128x128)


def test_dual_output_full_size_sampled():
    """The blockwise workload (16640 x 5120 x 8192): both forms against the
    same kernel schedule's fp32 result, on sampled rows and sampled columns."""
    wl = W.make_workload(2, 0)
    a, b = wl.a.cuda(), wl.b.cuda()
    qa, sa = fp8sm.fp8_quantize(a, fp8sm.FP8_SCALE_BLOCK_1x128)
    qb, sb = fp8sm.fp8_quantize(b, fp8sm.FP8_SCALE_BLOCK_128x128)
    del a, b
    r = fp8sm.FP8_MM_1x128_128x128
    q, s, qt, st = fp8sm.fp8_scaled_mm_quantized_dual(qa, qb, sa, sb, r)
    y = fp8sm.fp8_scaled_mm(qa, qb, sa, sb, r, out_dtype=torch.float32)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    rows = torch.from_numpy(sample_rows(wl.M, n=64, seed=5)).cuda()
    check_exact(y.index_select(0, rows).cpu().numpy(), q.index_select(0, rows).cpu().numpy(),
                s.index_select(1, rows).cpu().numpy(), "dual full size rows")
    cols = torch.from_numpy(sample_rows(wl.N, n=64, seed=6)).cuda()
    check_exact(y.index_select(1, cols).t().contiguous().cpu().numpy(),
                qt.index_select(0, cols).cpu().numpy(),
                st.index_select(1, cols).cpu().numpy(), "dual full size transposed")


def test_linear_chain_backward_with_grad_weight_against_oracle():
    """A chain of two blockwise linears, X (T, D) -> W1 (F, D) -> W2 (D, F),
    taken backward: dY1 = dY2 @ W2 (1x128_128x128) writes both e4m3 forms of
    dY1; dX = dY1 @ W1 from the 1x128-along-F form (1x128_128x128) and
    dW1 = dY1^T @ X from the 1x128-along-T form (1x128_128x1, K = T), the
    recipes of "improve fp8 blockwise gemm perf".  Against the oracle's chain
    (1x128 quantize, fp64 GEMM rounded to fp32, quantize both ways, fp64
    GEMMs) and SQNR >= 20 dB against the unquantized products."""
    T, D, F = 2048, 1024, 640
    g = W.generator(4242)
    x = W.randn_bf16((T, D), 1.0, g)
    w1 = W.randn_bf16((F, D), 0.02, g)
    w2 = W.randn_bf16((D, F), 0.02, g)
    dy2 = W.randn_bf16((T, D), 1.0, g)
    f = fp8sm
    qd, sd = f.fp8_quantize(dy2.cuda(), f.FP8_SCALE_BLOCK_1x128)
    q2t, s2t = f.fp8_quantize_transposed(w2.cuda(), f.FP8_SCALE_BLOCK_128x128)  # W2^T (F, D)
    q1t, s1t = f.fp8_quantize_transposed(w1.cuda(), f.FP8_SCALE_BLOCK_128x128)  # W1^T (D, F)
    qxt, sxt = f.fp8_quantize_transposed(x.cuda(), f.FP8_SCALE_BLOCK_1x128)     # X^T (D, T)
    dy1q, dy1s, dy1tq, dy1ts = f.fp8_scaled_mm_quantized_dual(
        qd, q2t, sd, s2t, f.FP8_MM_1x128_128x128)
    dx = f.fp8_scaled_mm(dy1q, q1t, dy1s, s1t, f.FP8_MM_1x128_128x128, out_dtype=torch.float32)
    dw1 = f.fp8_scaled_mm(dy1tq, qxt, dy1ts, sxt, f.FP8_MM_1x128_128x1, out_dtype=torch.float32)
    torch.cuda.synchronize()
    f.check_device_status()
    G = oracle.GROUP_128x128
    oqd, osd = oracle.quantize(W.bf16_bits(dy2), oracle.GROUP_1x128)
    oq2t, os2t = oracle.quantize(np.ascontiguousarray(W.bf16_bits(w2).T), G)
    oq1t, os1t = oracle.quantize(np.ascontiguousarray(W.bf16_bits(w1).T), G)
    oqxt, osxt = oracle.quantize(np.ascontiguousarray(W.bf16_bits(x).T), oracle.GROUP_1x128)
    y1, _ = oracle.scaled_mm(oqd, oq2t, osd, os2t, oracle.MM_1x128_128x128)
    y1 = y1.astype(np.float32)
    oy1q, oy1s = oracle.quantize_f32(y1, oracle.GROUP_1x128)
    oy1tq, oy1ts = oracle.quantize_f32(np.ascontiguousarray(y1.T), oracle.GROUP_1x128)
    rows = sample_rows(T, 48, seed=42)
    ref_dx, mag_dx = oracle.scaled_mm(oy1q, oq1t, oy1s, os1t, oracle.MM_1x128_128x128, rows=rows)
    ref_dw, mag_dw = oracle.scaled_mm(oy1tq, oqxt, oy1ts, osxt, oracle.MM_1x128_128x1)
    got_dx = dx.cpu().numpy().astype(np.float64)[rows]
    got_dw = dw1.cpu().numpy().astype(np.float64)
    for got, ref, mag, what in ((got_dx, ref_dx, mag_dx, "dX"), (got_dw, ref_dw, mag_dw, "dW1")):
        ok = oracle.within_tolerance(got, ref, mag)
        assert ok.all(), f"backward {what}: {int((~ok).sum())} of {ok.size} out of tolerance"
    dy1_exact = dy2.double().numpy() @ w2.double().numpy()
    for got, exact in ((got_dx, dy1_exact[rows] @ w1.double().numpy()),
                       (got_dw, dy1_exact.T @ x.double().numpy())):
        err = got - exact
        assert 10 * np.log10((exact ** 2).sum() / (err ** 2).sum()) >= 20.0
