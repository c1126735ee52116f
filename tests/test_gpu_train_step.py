"""The two-linear chain's training step as bench.py times it (forward and
backward, blockwise scaled, the chain workload at full size: 16640 tokens,
8192 -> 5120 -> 8192), checked against the oracle's chain on samples the oracle
computes one by one:

  Y2  and dX  on sampled token rows (each row needs its own row of Y1 / dY1);
  dW1 on sampled rows of one 128-wide block of dY1's features, and dW2 on
      sampled rows of one 128-wide block of Y1's features (each needs that
      block of Y1 / dY1 for every token, quantized along the tokens).

The oracle's chain: 1x128 / 128x128 quantize of the bf16 inputs, fp64 GEMM
rounded to fp32, that result quantized 1x128 along the features (next
forward / grad_input operand) and along the tokens (grad_weight operand),
fp64 GEMMs.  Plus SQNR >= 20 dB of each output against the unquantized fp64
products."""
import numpy as np
import pytest
import torch

import bench
import oracle
from fp8_scaled_matrix_b200 import fp8sm
from fp8_scaled_matrix_b200 import workloads as W
from helpers import check_gemm, sample_rows

pytestmark = pytest.mark.gpu

G1, G128 = oracle.GROUP_1x128, oracle.GROUP_128x128
R, R1 = oracle.MM_1x128_128x128, oracle.MM_1x128_128x1


def block_of(q, s, blk):
    """Rows [128 blk, 128 blk + 128) of a 128x128-quantized (N, K) operand:
    its codes and its (K/128, 1) column of tile scales."""
    kb = q.shape[1] // 128
    s2 = s.reshape(kb, q.shape[0] // 128)
    return (np.ascontiguousarray(q[128 * blk:128 * (blk + 1)]),
            np.ascontiguousarray(s2[:, blk]))


def sqnr_db(got, exact):
    err = got - exact
    return 10 * np.log10((exact ** 2).sum() / (err ** 2).sum())


@pytest.fixture(scope="module")
def step_and_workload():
    wl = W.make_workload(14, 0)
    st = bench.TrainStep(wl, torch.device("cuda", 0))
    st.quantize()
    st.gemm()
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    outs = {k: t.float().cpu().numpy().astype(np.float64)
            for k, t in zip(("y2", "dx", "dw1", "dw2"), st.outputs())}
    del st
    torch.cuda.empty_cache()
    return wl, outs


@pytest.fixture(scope="module")
def oracle_inputs(step_and_workload):
    wl, _ = step_and_workload
    xb, w1b = W.bf16_bits(wl.a), W.bf16_bits(wl.b)
    w2b, db = W.bf16_bits(wl.extra["b2"]), W.bf16_bits(wl.extra["dy"])
    o = {}
    o["qx"], o["sx"] = oracle.quantize(xb, G1)
    o["qd"], o["sd"] = oracle.quantize(db, G1)
    o["qw1"], o["sw1"] = oracle.quantize(w1b, G128)
    o["qw2"], o["sw2"] = oracle.quantize(w2b, G128)
    o["qw1t"], o["sw1t"] = oracle.quantize(np.ascontiguousarray(w1b.T), G128)
    o["qw2t"], o["sw2t"] = oracle.quantize(np.ascontiguousarray(w2b.T), G128)
    return o


def test_train_step_forward_y2(step_and_workload, oracle_inputs):
    wl, outs = step_and_workload
    o = oracle_inputs
    rows = sample_rows(wl.M, 32, seed=140)
    y1, _ = oracle.scaled_mm(o["qx"], o["qw1"], o["sx"], o["sw1"], R, rows=rows)
    y1q, y1s = oracle.quantize_f32(y1.astype(np.float32), G1)
    ref, mag = oracle.scaled_mm(y1q, o["qw2"], y1s, o["sw2"], R)
    check_gemm(outs["y2"][rows], ref, mag, "train step Y2")
    exact = (wl.a.double().numpy()[rows] @ wl.b.double().numpy().T) @ \
        wl.extra["b2"].double().numpy().T
    assert sqnr_db(outs["y2"][rows], exact) >= 20.0


def test_train_step_grad_input_dx(step_and_workload, oracle_inputs):
    wl, outs = step_and_workload
    o = oracle_inputs
    rows = sample_rows(wl.M, 32, seed=141)
    dy1, _ = oracle.scaled_mm(o["qd"], o["qw2t"], o["sd"], o["sw2t"], R, rows=rows)
    d1q, d1s = oracle.quantize_f32(dy1.astype(np.float32), G1)
    ref, mag = oracle.scaled_mm(d1q, o["qw1t"], d1s, o["sw1t"], R)
    check_gemm(outs["dx"][rows], ref, mag, "train step dX")
    exact = (wl.extra["dy"].double().numpy()[rows] @ wl.extra["b2"].double().numpy()) @ \
        wl.b.double().numpy()
    assert sqnr_db(outs["dx"][rows], exact) >= 20.0


def test_train_step_grad_weight_dw1(step_and_workload, oracle_inputs):
    """dW1 = dY1^T X on sampled rows of dY1's feature block 17 (and its edges)."""
    wl, outs = step_and_workload
    o = oracle_inputs
    blk = 17
    qb, sb = block_of(o["qw2t"], o["sw2t"], blk)
    dy1_blk, _ = oracle.scaled_mm(o["qd"], qb, o["sd"], sb, R)          # (T, 128)
    dtq, dts = oracle.quantize_f32(np.ascontiguousarray(dy1_blk.astype(np.float32).T), G1)
    qxt, sxt = oracle.quantize(np.ascontiguousarray(W.bf16_bits(wl.a).T), G1)
    local = np.array([0, 1, 63, 64, 126, 127, 40, 99])
    ref, mag = oracle.scaled_mm(dtq, qxt, dts, sxt, R1, rows=local)
    got = outs["dw1"][128 * blk + local]
    check_gemm(got, ref, mag, "train step dW1")
    dy1_exact = wl.extra["dy"].double().numpy() @ \
        wl.extra["b2"].double().numpy()[:, 128 * blk + local]
    assert sqnr_db(got, dy1_exact.T @ wl.a.double().numpy()) >= 20.0


def test_train_step_grad_weight_dw2(step_and_workload, oracle_inputs):
    """dW2 = dY2^T Y1 on sampled rows, columns of Y1's feature block 29."""
    wl, outs = step_and_workload
    o = oracle_inputs
    blk = 29
    qb, sb = block_of(o["qw1"], o["sw1"], blk)
    y1_blk, _ = oracle.scaled_mm(o["qx"], qb, o["sx"], sb, R)           # (T, 128)
    ytq, yts = oracle.quantize_f32(np.ascontiguousarray(y1_blk.astype(np.float32).T), G1)
    qdt, sdt = oracle.quantize(np.ascontiguousarray(W.bf16_bits(wl.extra["dy"]).T), G1)
    rows = sample_rows(wl.K, 12, seed=142)
    ref, mag = oracle.scaled_mm(qdt, ytq, sdt, yts, R1, rows=rows)      # (rows, 128)
    got = outs["dw2"][rows][:, 128 * blk:128 * (blk + 1)]
    check_gemm(got, ref, mag, "train step dW2")
    y1_exact = wl.a.double().numpy() @ wl.b.double().numpy()[128 * blk:128 * (blk + 1)].T
    exact = wl.extra["dy"].double().numpy()[:, rows].T @ y1_exact
    assert sqnr_db(got, exact) >= 20.0
