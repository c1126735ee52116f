"""Grouped (MoE) MXFP8 GEMM against the oracle: the oracle's grouped result is
its dense MXFP8 GEMM applied group by group to that group's rows (their codes
and plain E8M0 scales) and that expert's weights (the definition of the
grouped GEMM).  Groups start at arbitrary rows, so the kernel's gather of A's
scale words from the scale-factor tiles is exercised at every offset."""
import numpy as np
import pytest
import torch

import oracle
from fp8_scaled_matrix_b200 import fp8sm
from fp8_scaled_matrix_b200 import workloads as W
from helpers import check_gemm, out_f64, sample_rows

pytestmark = pytest.mark.gpu


def oracle_operands(a, b):
    """a (M, K) bf16, b (E, N, K) bf16 -> oracle codes and plain scales."""
    qa, ea = oracle.mx_quantize(W.bf16_bits(a))
    per = [oracle.mx_quantize(W.bf16_bits(b[e].contiguous())) for e in range(b.shape[0])]
    return qa, ea, np.stack([q for q, _ in per]), np.stack([e for _, e in per])


def oracle_grouped(qa, ea, qb, eb, offs, rows=None):
    M = qa.shape[0]
    want = np.arange(M) if rows is None else np.asarray(rows)
    outs, mags = [], []
    start = 0
    for g, end in enumerate(offs):
        sel = want[(want >= start) & (want < end)]
        if sel.size:
            ref, mag = oracle.mx_scaled_mm(np.ascontiguousarray(qa[start:end]), qb[g],
                                           np.ascontiguousarray(ea[start:end]), eb[g],
                                           rows=sel - start)
            outs.append(ref)
            mags.append(mag)
        start = int(end)
    return np.concatenate(outs), np.concatenate(mags)


def gpu_tiles(qa, ea, qb, eb):
    """The entry point's scale layouts, from the oracle's plain scales: A's
    tiles, then each expert's tile set in order."""
    ta = oracle.mx_scales_to_tiles(ea)
    tb = np.concatenate([oracle.mx_scales_to_tiles(eb[g]) for g in range(eb.shape[0])])
    return (torch.from_numpy(qa).cuda(), torch.from_numpy(np.ascontiguousarray(qb)).cuda(),
            torch.from_numpy(ta).cuda(), torch.from_numpy(tb).cuda())


@pytest.mark.parametrize("sizes,N,K", [
    ([5, 0, 17, 130], 272, 256),
    ([0, 0, 64, 0], 256, 96),
    ([300], 512, 384),
    ([1, 255, 129, 0, 2], 528, 160),
    ([40, 100, 33, 7, 200, 64, 1, 90], 256, 4096),
])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_grouped_mx_parity(sizes, N, K, out_dtype):
    E = len(sizes)
    g = W.generator(sum(sizes) * 5 + N + K)
    a = W.randn_bf16((sum(sizes), K), 1.0, g)
    b = W.randn_bf16((E, N, K), 0.02, g)
    offs = np.cumsum(sizes).astype(np.int32)
    qa, ea, qb, eb = oracle_operands(a, b)
    out = fp8sm.fp8_grouped_scaled_mm_mx(*gpu_tiles(qa, ea, qb, eb),
                                         torch.as_tensor(offs).cuda(), out_dtype=out_dtype)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    if sum(sizes) == 0:
        return
    ref, mag = oracle_grouped(qa, ea, qb, eb, offs)
    check_gemm(out_f64(out), ref, mag, f"grouped mx {sizes}")


def test_grouped_mx_full_size_sampled():
    """The MoE workload (16 experts, 32768 routed rows, N = K = 4096), MXFP8
    quantized on the GPU (the experts in one call on the (E N, K) view),
    checked on sampled rows including every group edge."""
    wl = W.make_workload(4, 0)
    E, N, K = wl.b.shape
    qa, sa = fp8sm.fp8_quantize_mx(wl.a.cuda())
    qb, sb = fp8sm.fp8_quantize_mx(wl.b.cuda().reshape(E * N, K))
    out = fp8sm.fp8_grouped_scaled_mm_mx(qa, qb.view(E, N, K), sa, sb, wl.offs.cuda())
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    oqa, oea, oqb, oeb = oracle_operands(wl.a, wl.b)
    ends = wl.offs.numpy()
    rows = set(sample_rows(wl.M, 40, seed=13).tolist())
    for e in ends[:-1]:
        rows.update({int(e) - 1, int(e)})
    rows = np.array(sorted(r for r in rows if 0 <= r < wl.M))
    ref, mag = oracle_grouped(oqa, oea, oqb, oeb, ends, rows=rows)
    check_gemm(out_f64(out)[rows], ref, mag, "grouped mx full size")


def test_grouped_mx_malformed_offs_reports_value_error():
    E, N, K, M = 3, 32, 128, 20
    sentinel = torch.full((M, N), 7.0, device="cuda")
    fp8sm.fp8_grouped_scaled_mm_mx(
        torch.zeros(M, K, dtype=torch.uint8, device="cuda"),
        torch.zeros(E, N, K, dtype=torch.uint8, device="cuda"),
        torch.zeros(fp8sm.fp8_mx_scale_bytes(M, K), dtype=torch.uint8, device="cuda"),
        torch.zeros(E * fp8sm.fp8_mx_scale_bytes(N, K), dtype=torch.uint8, device="cuda"),
        torch.tensor([10, 5, 20], dtype=torch.int32, device="cuda"),
        out_dtype=torch.float32, out=sentinel)
    assert fp8sm.fp8_get_device_status() == fp8sm.FP8_ERR_VALUE
    assert (sentinel.cpu() == 7.0).all()
