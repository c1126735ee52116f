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


# -------------------------------------------------- weight gradient per expert

def padded_t_bits(x: torch.Tensor, start: int, end: int) -> np.ndarray:
    """Group [start, end) of x (tokens x cols), transposed and padded with zero
    tokens to a multiple of 128: the definition of the per-expert layout."""
    n = end - start
    pad = -(-n // 128) * 128
    out = np.zeros((x.shape[1], pad), np.uint16)
    out[:, :n] = W.bf16_bits(x[start:end]).T
    return out


def oracle_wgrad_group(dy, x, start, end, rows=None):
    qa, sa = oracle.quantize(padded_t_bits(dy, start, end), oracle.GROUP_1x128)
    qb, sb = oracle.quantize(padded_t_bits(x, start, end), oracle.GROUP_1x128)
    return (qa, sa, qb, sb), oracle.scaled_mm(qa, qb, sa, sb, MM["1x128_128x1"], rows=rows)


def gpu_wgrad(dy, x, offs_np, out_dtype=torch.float32):
    offs = torch.as_tensor(offs_np, dtype=torch.int32).cuda()
    qa, sa = fp8sm.fp8_quantize_transposed_grouped(dy.cuda(), offs)
    qb, sb = fp8sm.fp8_quantize_transposed_grouped(x.cuda(), offs)
    out = fp8sm.fp8_grouped_scaled_mm_wgrad(qa, qb, sa, sb, offs, dy.shape[0],
                                            out_dtype=out_dtype)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    return qa, sa, qb, sb, out


def test_grouped_transposed_quantize_many_tiles_per_cta():
    """The per-expert padded transposed quantization on enough tiles that every
    persistent CTA reuses its tile buffers several times, with empty, ragged
    and multi-block groups: each group's padded codes and scales bit-exact
    against the oracle's quantization of that group's zero-padded transpose."""
    sizes = [0, 3000, 1, 4096, 0, 5000, 128, 3775]
    T, cols = sum(sizes), 2048
    g = W.generator(9090)
    x = W.randn_bf16((T, cols), 1.0, g, outlier_frac=0.001, outlier_mult=50.0)
    ends = np.cumsum(sizes).astype(np.int32)
    offs = torch.as_tensor(ends, dtype=torch.int32).cuda()
    q, s = fp8sm.fp8_quantize_transposed_grouped(x.cuda(), offs)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    q, s = q.cpu().numpy(), s.cpu().numpy()
    start, pb = 0, 0
    for end in ends:
        n = int(end) - start
        nblk = -(-n // 128)
        if n:
            oq, osc = oracle.quantize(padded_t_bits(x, start, int(end)), oracle.GROUP_1x128)
            cols_ = slice(128 * pb, 128 * (pb + nblk))
            assert np.array_equal(q[:, cols_], oq)
            assert np.array_equal(s[pb:pb + nblk].reshape(-1).view(np.uint32), osc.view(np.uint32))
        start, pb = int(end), pb + nblk


@pytest.mark.parametrize("sizes,M,N", [
    ([5, 0, 17, 130], 256, 272),
    ([0, 0, 64, 0], 128, 256),
    ([300], 128, 512),
    ([1, 255, 129, 0, 2, 384], 384, 160),
])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_grouped_wgrad_parity(sizes, M, N, out_dtype):
    E = len(sizes)
    T = sum(sizes)
    g = W.generator(T * 7 + M + N)
    dy = W.randn_bf16((T, M), 1e-3, g)
    x = W.randn_bf16((T, N), 1.0, g)
    ends = np.cumsum(sizes).astype(np.int32)
    qa, sa, qb, sb, out = gpu_wgrad(dy, x, ends, out_dtype)
    qa, sa, qb, sb = (t.cpu().numpy() for t in (qa, sa, qb, sb))
    start, pb = 0, 0
    for e, end in enumerate(ends):
        n = int(end) - start
        nblk = -(-n // 128)
        if n == 0:
            assert (out[e] == 0).all(), f"empty group {e} must give a zero gradient"
            continue
        (oqa, osa, oqb, osb), (ref, mag) = oracle_wgrad_group(dy, x, start, int(end))
        # the quantized per-group blocks are the oracle's bit for bit
        cols = slice(128 * pb, 128 * (pb + nblk))
        assert np.array_equal(qa[:, cols], oqa) and np.array_equal(qb[:, cols], oqb)
        assert np.array_equal(sa[pb:pb + nblk].reshape(-1).view(np.uint32), osa.view(np.uint32))
        assert np.array_equal(sb[pb:pb + nblk].reshape(-1).view(np.uint32), osb.view(np.uint32))
        check_gemm(out_f64(out[e]), ref, mag, f"wgrad group {e} of {sizes}")
        start, pb = int(end), pb + nblk


def test_grouped_wgrad_full_size_sampled():
    """The MoE layer's weight gradient on the MoE workload's split (16 experts,
    32768 tokens, 4096 outputs x 4096 inputs): three experts checked on
    sampled rows (the largest, a small one and the last)."""
    wl = W.make_workload(13, 0)
    dy, x = wl.a, wl.b
    ends = wl.offs.numpy()
    _, _, _, _, out = gpu_wgrad(dy, x, ends)
    sizes = np.diff(np.concatenate([[0], ends]))
    pick = {int(np.argmax(sizes)), len(ends) - 1}
    nz = [e for e in range(len(ends)) if sizes[e] > 0]
    pick.add(int(min(nz, key=lambda e: sizes[e])))
    for e in sorted(pick):
        start = int(ends[e - 1]) if e else 0
        rows = sample_rows(wl.M, 24, seed=e)
        _, (ref, mag) = oracle_wgrad_group(dy, x, start, int(ends[e]), rows=rows)
        check_gemm(out_f64(out[e])[rows], ref, mag, f"wgrad expert {e} full size")


def test_grouped_wgrad_malformed_offs_reports_value_error():
    T, M, N, E = 64, 128, 64, 3
    offs = torch.tensor([40, 20, 64], dtype=torch.int32, device="cuda")
    dy = torch.zeros(T, M, dtype=torch.bfloat16, device="cuda")
    fp8sm.fp8_quantize_transposed_grouped(dy, offs)
    torch.cuda.synchronize()
    assert fp8sm.fp8_get_device_status() == fp8sm.FP8_ERR_VALUE
    P = fp8sm.fp8_grouped_padded_tokens(T, E)
    sentinel = torch.full((E, M, N), 7.0, device="cuda")
    fp8sm.fp8_grouped_scaled_mm_wgrad(
        torch.zeros(M, P, dtype=torch.uint8, device="cuda"),
        torch.zeros(N, P, dtype=torch.uint8, device="cuda"),
        torch.ones(P // 128, M, device="cuda"), torch.ones(P // 128, N, device="cuda"),
        offs, T, out_dtype=torch.float32, out=sentinel)
    assert fp8sm.fp8_get_device_status() == fp8sm.FP8_ERR_VALUE
    assert (sentinel.cpu() == 7.0).all()
