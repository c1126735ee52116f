"""Grouped (MoE) rowwise GEMM parity, empty groups, malformed offs."""
import numpy as np
import pytest
import torch

import oracle
from fp8_scaled_matrix_b200 import fp8sm
from fp8_scaled_matrix_b200 import workloads as W
from helpers import check_gemm, codes_np, out_f64, sample_rows

pytestmark = pytest.mark.gpu


def oracle_grouped_operands(wl):
    qa, sa = oracle.quantize(W.bf16_bits(wl.a), oracle.GROUP_ROW)
    E, N, K = wl.b.shape
    qb, sb = oracle.quantize(W.bf16_bits(wl.b.reshape(E * N, K)), oracle.GROUP_ROW)
    return qa, sa, qb.reshape(E, N, K), sb.reshape(E, N)


def run_gpu(qa, sa, qb, sb, offs, out_dtype):
    out = fp8sm.fp8_grouped_scaled_mm(
        torch.from_numpy(qa).cuda(), torch.from_numpy(np.ascontiguousarray(qb)).cuda(),
        torch.from_numpy(sa).cuda(), torch.from_numpy(np.ascontiguousarray(sb)).cuda(),
        torch.as_tensor(offs, dtype=torch.int32).cuda(), out_dtype=out_dtype)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("sizes,N,K", [
    ([5, 0, 17, 130], 272, 256),
    ([0, 0, 64, 0], 256, 128),
    ([300], 512, 384),
    ([16] * 12, 48, 64),
    ([1, 255, 129, 0, 2], 528, 160),
])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_grouped_parity(sizes, N, K, out_dtype):
    E = len(sizes)
    M = sum(sizes)
    wl = W.small_case("grouped", M, N, K, seed=M + N + K, E=E, group_sizes=sizes)
    qa, sa, qb, sb = oracle_grouped_operands(wl)
    out = run_gpu(qa, sa, qb, sb, wl.offs.numpy(), out_dtype)
    fp8sm.check_device_status()
    ref, mag = oracle.grouped_scaled_mm(qa, qb, sa, sb, wl.offs.numpy())
    check_gemm(out_f64(out), ref, mag, f"grouped {sizes}")


def test_grouped_matches_dense_per_group():
    sizes = [130, 0, 77]
    wl = W.small_case("grouped", sum(sizes), 256, 256, seed=9, E=3, group_sizes=sizes)
    qa, sa, qb, sb = oracle_grouped_operands(wl)
    out = out_f64(run_gpu(qa, sa, qb, sb, wl.offs.numpy(), torch.float32))
    start = 0
    for e, sz in enumerate(sizes):
        if sz:
            d = fp8sm.fp8_scaled_mm(torch.from_numpy(qa[start:start + sz]).cuda(),
                                    torch.from_numpy(qb[e]).cuda(),
                                    torch.from_numpy(sa[start:start + sz].copy()).cuda(),
                                    torch.from_numpy(sb[e].copy()).cuda(),
                                    fp8sm.FP8_MM_ROW_ROW, out_dtype=torch.float32)
            torch.cuda.synchronize()
            assert np.array_equal(out_f64(d), out[start:start + sz])
        start += sz


@pytest.mark.parametrize("offs", [[10, 5, 20], [5, 10, 19], [-1, 10, 20], [5, 10, 21]])
def test_grouped_malformed_offs_reports_value_error(offs):
    E, N, K, M = 3, 32, 64, 20
    qa = np.zeros((M, K), np.uint8)
    qb = np.zeros((E, N, K), np.uint8)
    sentinel = torch.full((M, N), 7.0, device="cuda")
    fp8sm.fp8_grouped_scaled_mm(
        torch.from_numpy(qa).cuda(), torch.from_numpy(qb).cuda(),
        torch.ones(M, device="cuda"), torch.ones(E, N, device="cuda"),
        torch.tensor(offs, dtype=torch.int32, device="cuda"),
        out_dtype=torch.float32, out=sentinel)
    st = fp8sm.fp8_get_device_status()
    assert st == fp8sm.FP8_ERR_VALUE
    assert (sentinel.cpu() == 7.0).all()          # nothing written
    assert fp8sm.fp8_get_device_status() == fp8sm.FP8_OK   # read clears


def test_grouped_full_size_sampled():
    """The MoE workload (E=16, 32768 x 4096 x 4096, Zipf group sizes) as
    bench.py launches it: GPU quantize of tokens and experts, then the grouped
    GEMM; sampled rows (group and tile edges) against the oracle."""
    wl = W.make_workload(4)
    E, N, K = wl.b.shape
    a = wl.a.cuda()
    w = wl.b.cuda().reshape(E * N, K)
    qa, sa = fp8sm.fp8_quantize(a, fp8sm.FP8_SCALE_ROW)
    qw, sw = fp8sm.fp8_quantize(w, fp8sm.FP8_SCALE_ROW)
    offs = wl.offs.cuda()
    out = fp8sm.fp8_grouped_scaled_mm(qa, qw.view(E, N, K), sa, sw.view(E, N), offs)
    torch.cuda.synchronize()
    fp8sm.check_device_status()
    ends = wl.offs.numpy().astype(np.int64)
    edges = set()
    for e in ends:
        edges.update({int(e) - 1, int(e), int(e) + 1})
    rows = np.array(sorted(r for r in edges.union(sample_rows(wl.M, 24, seed=4).tolist())
                           if 0 <= r < wl.M), dtype=np.int64)
    oqa, osa, oqb, osb = oracle_grouped_operands(wl)
    ref, mag = oracle.grouped_scaled_mm(oqa, oqb, osa, osb, wl.offs.numpy(), rows=rows)
    check_gemm(out_f64(out)[rows], ref, mag, "grouped full size")
