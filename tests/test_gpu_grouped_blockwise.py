"""Grouped (MoE) GEMM with blockwise scales (1x128 activations, each
expert's 128x128 weight scales) against the oracle: the oracle's grouped
result is its dense 1x128_128x128 GEMM applied group by group to the rows of
that group and that expert's weights (the definition of the grouped GEMM)."""
import numpy as np
import pytest
import torch

import oracle
from fp8_scaled_matrix_b200 import fp8sm
from fp8_scaled_matrix_b200 import workloads as W
from helpers import MM, check_gemm, out_f64, sample_rows

pytestmark = pytest.mark.gpu


def oracle_operands(a, b):
    """a (M, K) bf16, b (E, N, K) bf16 -> oracle codes/scales in the layouts the
    blockwise grouped entry point takes."""
    qa, sa = oracle.quantize(W.bf16_bits(a), oracle.GROUP_1x128)        # sa (K/128, M)
    E, N, K = b.shape
    qbs, sbs = [], []
    for e in range(E):
        q, s = oracle.quantize(W.bf16_bits(b[e].contiguous()), oracle.GROUP_128x128)
        qbs.append(q)
        sbs.append(s)                                                  # (K/128, ceil(N/128))
    return qa, sa, np.stack(qbs), np.stack(sbs)


def oracle_grouped(qa, sa, qb, sb, offs, rows=None):
    M, K = qa.shape
    KB = K // 128
    sa2 = sa.reshape(KB, M)
    start = 0
    outs, mags = [], []
    want = np.arange(M) if rows is None else np.asarray(rows)
    for e, end in enumerate(offs):
        sel = want[(want >= start) & (want < end)]
        if sel.size:
            a_rows = np.ascontiguousarray(qa[start:end])
            s_rows = np.ascontiguousarray(sa2[:, start:end]).reshape(-1)
            ref, mag = oracle.scaled_mm(a_rows, np.ascontiguousarray(qb[e]), s_rows,
                                        np.ascontiguousarray(sb[e]).reshape(-1),
                                        MM["1x128_128x128"], rows=sel - start)
            outs.append(ref)
            mags.append(mag)
        start = end
    return np.concatenate(outs), np.concatenate(mags)


def run_gpu(qa, sa, qb, sb, offs, out_dtype):
    out = fp8sm.fp8_grouped_scaled_mm_blockwise(
        torch.from_numpy(qa).cuda(), torch.from_numpy(np.ascontiguousarray(qb)).cuda(),
        torch.from_numpy(np.ascontiguousarray(sa)).cuda(),
        torch.from_numpy(np.ascontiguousarray(sb)).cuda(),
        torch.as_tensor(offs, dtype=torch.int32).cuda(), out_dtype=out_dtype)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    return out


@pytest.mark.parametrize("sizes,N,K", [
    ([5, 0, 17, 130], 272, 256),
    ([0, 0, 64, 0], 256, 128),
    ([300], 512, 384),
    ([1, 255, 129, 0, 2], 528, 640),
])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_grouped_blockwise_parity(sizes, N, K, out_dtype):
    E = len(sizes)
    g = W.generator(sum(sizes) * 3 + N + K)
    a = W.randn_bf16((sum(sizes), K), 1.0, g)
    b = W.randn_bf16((E, N, K), 0.02, g)
    offs = np.cumsum(sizes).astype(np.int32)
    qa, sa, qb, sb = oracle_operands(a, b)
    out = run_gpu(qa, sa, qb, sb, offs, out_dtype)
    if sum(sizes) == 0:
        return
    ref, mag = oracle_grouped(qa, sa, qb, sb, offs)
    check_gemm(out_f64(out), ref, mag, f"grouped blockwise {sizes}")


def test_grouped_blockwise_full_size_sampled():
    """The MoE workload's shape and group split (16 experts, 32768 routed rows,
    N = K = 4096) with blockwise scales, GPU quantization end to end, checked
    on sampled rows (including group edges)."""
    wl = W.make_workload(4, 0)
    a, b = wl.a.cuda(), wl.b.cuda()
    E, N, K = wl.b.shape
    qa, sa = fp8sm.fp8_quantize(a, fp8sm.FP8_SCALE_BLOCK_1x128)
    qbs, sbs = [], []
    for e in range(E):
        q, s = fp8sm.fp8_quantize(b[e], fp8sm.FP8_SCALE_BLOCK_128x128)
        qbs.append(q)
        sbs.append(s)
    qb, sb = torch.stack(qbs), torch.stack(sbs)
    offs = wl.offs.cuda()
    out = fp8sm.fp8_grouped_scaled_mm_blockwise(qa, qb, sa, sb, offs)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    oqa, osa, oqb, osb = oracle_operands(wl.a, wl.b)
    assert np.array_equal(qa.cpu().numpy(), oqa)
    assert np.array_equal(qb.cpu().numpy(), oqb)
    ends = wl.offs.numpy()
    rows = set(sample_rows(wl.M, 40, seed=11).tolist())
    for e in ends[:-1]:
        rows.update({int(e) - 1, int(e)})
    rows = np.array(sorted(r for r in rows if 0 <= r < wl.M))
    ref, mag = oracle_grouped(oqa, osa, oqb, osb, ends, rows=rows)
    check_gemm(out_f64(out)[rows], ref, mag, "grouped blockwise full size")


def test_grouped_blockwise_malformed_offs_reports_value_error():
    E, N, K, M = 3, 32, 128, 20
    sentinel = torch.full((M, N), 7.0, device="cuda")
    fp8sm.fp8_grouped_scaled_mm_blockwise(
        torch.zeros(M, K, dtype=torch.uint8, device="cuda"),
        torch.zeros(E, N, K, dtype=torch.uint8, device="cuda"),
        torch.ones(M, device="cuda"), torch.ones(E, 1, device="cuda"),
        torch.tensor([10, 5, 20], dtype=torch.int32, device="cuda"),
        out_dtype=torch.float32, out=sentinel)
    assert fp8sm.fp8_get_device_status() == fp8sm.FP8_ERR_VALUE
    assert (sentinel.cpu() == 7.0).all()
