"""Pins for the oracle's dynamic quantizer (all four group kinds).

Pinned against: hand-worked rows (tests/golden/quant_handworked.json),
torch's own fp8 cast on the scaled values, and invariants the definition
fixes (the largest element of every non-zero group lands on +-448; a group's
scale is exactly amax/448 in fp32; all-zero groups use the epsilon guard;
dequantized values sit within half an e4m3 step of the input; the scale
layouts index the right group).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from fp8_scaled_matrix_b200 import workloads as W


def _bits(vals):
    return W.bf16_bits(torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16))


def test_handworked_rows(golden_dir):
    fx = json.load(open(os.path.join(golden_dir, "quant_handworked.json")))
    for row in fx["rows"]:
        x = _bits([row["x"]])
        for group in (oracle.GROUP_ROW, oracle.GROUP_TENSOR):
            q, s = oracle.quantize(x, group)
            assert [f"0x{c:02X}" for c in q[0]] == row["codes"], row["note"]
            if row["scale"] == "eps/448":
                assert s[0] == np.float32(oracle.EPS) / np.float32(448.0)
            else:
                assert s[0] == np.float32(row["scale"])
    sat = fx["saturation"]
    q = oracle.cast_with_inverse(_bits([sat["x"]]), sat["inverse"])
    assert [f"0x{c:02X}" for c in q[0]] == sat["codes"]


def _torch_reference_cast(x_bits, inv):
    """Cast x*inv through torch's fp8 conversion (clamped to +-448)."""
    f = torch.from_numpy(x_bits.astype(np.uint32) << 16).view(torch.float32)
    y = f * torch.tensor(inv, dtype=torch.float32)
    return y.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _groups(rows, cols, group):
    """Yield (row slice, col slice, scale index) for every group."""
    if group == oracle.GROUP_TENSOR:
        yield slice(0, rows), slice(0, cols), 0
    elif group == oracle.GROUP_ROW:
        for r in range(rows):
            yield slice(r, r + 1), slice(0, cols), r
    elif group == oracle.GROUP_1x128:
        for kb in range(cols // 128):
            for r in range(rows):
                yield slice(r, r + 1), slice(kb * 128, kb * 128 + 128), kb * rows + r
    else:
        RB = (rows + 127) // 128
        for kb in range(cols // 128):
            for rb in range(RB):
                yield (slice(rb * 128, min(rows, rb * 128 + 128)),
                       slice(kb * 128, kb * 128 + 128), kb * RB + rb)


@pytest.mark.parametrize("group,rows,cols", [
    (oracle.GROUP_TENSOR, 37, 200),
    (oracle.GROUP_ROW, 67, 264),
    (oracle.GROUP_1x128, 45, 384),
    (oracle.GROUP_128x128, 300, 256),   # ragged last row block
])
def test_invariants_random(group, rows, cols):
    g = W.generator(7 + group)
    x = W.randn_bf16((rows, cols), 1.0, g, outlier_frac=0.01, outlier_mult=50.0)
    xb = W.bf16_bits(x)
    q, s = oracle.quantize(xb, group)
    xf = x.float().numpy()
    n_groups = 0
    for rs, cs, si in _groups(rows, cols, group):
        n_groups += 1
        blk = xf[rs, cs]
        amax = np.float32(np.abs(blk).max())
        # scale is exactly amax/448 in fp32
        assert s[si] == np.float32(amax) / np.float32(448.0)
        inv = np.float32(448.0) / np.float32(amax)
        # cast agrees with torch's fp8 conversion of x*inv
        want = _torch_reference_cast(xb[rs, cs], inv)
        assert np.array_equal(q[rs, cs], want)
        # the largest element lands on +-448
        codes = q[rs, cs]
        assert ((codes & 0x7F) == 0x7E).any()
        assert ((codes & 0x7F) <= 0x7E).all()
        # dequantized values are within half an e4m3 step (relative 2^-4,
        # absolute 2^-10 in the subnormal range) of x, in units of the scale
        dq = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()
        y = blk.astype(np.float64) * float(inv)
        assert (np.abs(dq - y) <= np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10) + 1e-12).all()
    assert n_groups == oracle.scale_count(rows, cols, group)


def test_all_zero_groups_use_eps():
    x = np.zeros((3, 256), dtype=np.uint16)
    for group in range(4):
        q, s = oracle.quantize(x, group)
        assert (q == 0).all()
        assert (s == np.float32(oracle.EPS) / np.float32(448.0)).all()


def test_negative_zero_and_single_element_groups():
    x = _bits([[-0.0], [3.0], [-5.0]])
    q, s = oracle.quantize(x, oracle.GROUP_ROW)
    assert list(q[:, 0]) == [0x80, 0x7E, 0xFE]
    assert s[1] == np.float32(3.0) / np.float32(448.0)


def test_layouts_pick_the_right_group():
    """Put a distinct magnitude in every group and check each scale slot."""
    rows, cols = 256, 384
    x = torch.zeros(rows, cols)
    for r in range(rows):
        for kb in range(3):
            x[r, kb * 128 + (r % 128)] = float(1 + (r % 7) + 10 * kb)
    xb = W.bf16_bits(x.to(torch.bfloat16))
    _, s = oracle.quantize(xb, oracle.GROUP_1x128)
    for r in range(rows):
        for kb in range(3):
            assert s[kb * rows + r] == np.float32(1 + (r % 7) + 10 * kb) / np.float32(448)
    _, s = oracle.quantize(xb, oracle.GROUP_128x128)
    for rb in range(2):
        for kb in range(3):
            assert s[kb * 2 + rb] == np.float32(7 + 10 * kb) / np.float32(448)
    _, s = oracle.quantize(xb, oracle.GROUP_ROW)
    assert s[5] == np.float32(26) / np.float32(448)


def test_bad_arguments_rejected():
    with pytest.raises(ValueError):
        oracle.quantize(np.zeros((2, 100), dtype=np.uint16), oracle.GROUP_1x128)
