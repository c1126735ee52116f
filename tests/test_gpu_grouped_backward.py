"""The MoE layer's grad_input on the GPU: for each expert g,
dX[rows of g] = dY[rows of g] @ W_g, the backward of
out = grouped_mm(x, weight.transpose(-2, -1)) ("Add _grouped_mm dispatch
handler to Float8Tensor") with the 1x128_128x128 recipe that "improve fp8
blockwise gemm perf" uses for grad_input.  The contraction runs along the
expert weight's output dimension, so each expert's weight is quantized
transposed (W_g^T, 128x128 tiles) and the grouped blockwise GEMM consumes
it.  Checked against the oracle: dY quantized 1x128, each materialised W_g^T
quantized 128x128, and the dense 1x128_128x128 GEMM applied group by group."""
import numpy as np
import pytest
import torch

import oracle
from fp8_scaled_matrix_b200 import fp8sm
from fp8_scaled_matrix_b200 import workloads as W
from helpers import MM, check_gemm, out_f64, sample_rows

pytestmark = pytest.mark.gpu


def gpu_grad_input(dy, w, offs):
    """dy (M, N) bf16 CUDA, w (E, N, K) bf16 CUDA -> grad_input (M, K)."""
    E, N, K = w.shape
    qdy, sdy = fp8sm.fp8_quantize(dy, fp8sm.FP8_SCALE_BLOCK_1x128)
    qs, ss = [], []
    for e in range(E):
        q, s = fp8sm.fp8_quantize_transposed(w[e], fp8sm.FP8_SCALE_BLOCK_128x128)
        qs.append(q)
        ss.append(s)
    out = fp8sm.fp8_grouped_scaled_mm_blockwise(qdy, torch.stack(qs), sdy, torch.stack(ss),
                                                offs, out_dtype=torch.float32)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    return out


def oracle_grad_input(dy, w, ends, rows=None):
    qa, sa = oracle.quantize(W.bf16_bits(dy), oracle.GROUP_1x128)     # sa (N/128, M)
    M, N = dy.shape
    E, _, K = w.shape
    sa2 = sa.reshape(N // 128, M)
    want = np.arange(M) if rows is None else np.asarray(rows)
    outs, mags = [], []
    start = 0
    for g, end in enumerate(ends):
        sel = want[(want >= start) & (want < end)]
        if sel.size:
            qb, sb = oracle.quantize(np.ascontiguousarray(W.bf16_bits(w[g]).T),
                                     oracle.GROUP_128x128)
            ref, mag = oracle.scaled_mm(np.ascontiguousarray(qa[start:end]), qb,
                                        np.ascontiguousarray(sa2[:, start:end]).reshape(-1), sb,
                                        MM["1x128_128x128"], rows=sel - start)
            outs.append(ref)
            mags.append(mag)
        start = int(end)
    return np.concatenate(outs), np.concatenate(mags)


@pytest.mark.parametrize("sizes,N,K", [
    ([5, 0, 17, 130], 256, 384),
    ([300], 384, 256),
    ([1, 255, 129, 0, 2], 128, 640),
])
def test_grouped_grad_input_parity(sizes, N, K):
    E = len(sizes)
    g = W.generator(sum(sizes) + 11 * N + K)
    dy = W.randn_bf16((sum(sizes), N), 1.0, g)
    w = W.randn_bf16((E, N, K), 0.02, g)
    ends = np.cumsum(sizes).astype(np.int32)
    out = gpu_grad_input(dy.cuda(), w.cuda(), torch.as_tensor(ends).cuda())
    ref, mag = oracle_grad_input(dy, w, ends)
    check_gemm(out_f64(out), ref, mag, f"grouped grad_input {sizes}")


def test_grouped_grad_input_full_size_sampled():
    """The MoE workload's experts and group split (16 x 4096 x 4096, 32768
    rows), dY of the same shape as the routed activations."""
    wl = W.make_workload(12, 0)
    out = gpu_grad_input(wl.a.cuda(), wl.b.cuda(), wl.offs.cuda())
    ends = wl.offs.numpy()
    rows = set(sample_rows(wl.M, 32, seed=21).tolist())
    for e in ends[:-1]:
        rows.update({int(e) - 1, int(e)})
    rows = np.array(sorted(r for r in rows if 0 <= r < wl.M))
    ref, mag = oracle_grad_input(wl.a, wl.b, ends, rows=rows)
    check_gemm(out_f64(out)[rows], ref, mag, "grouped grad_input full size")
