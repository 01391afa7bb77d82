"""Pins of two oracle functions against facts fixed outside them.

* oracle_quantize_nvfp4_s2, NVFP4 with a caller-given global scale per group
  (josch15366/Qwen3.8-Flash-Next-NVFP4-LocalHessian-Experts, introduction:
  gate and up share one weight_scale_2, which a caller holding them apart
  must pass itself): the hand-worked example, closed forms of a saturated
  block and of s2 = 0, rejection of invalid scales, and the gate/up split
  (each half quantized with RN32(max(amax_gate, amax_up) / 2688), formed
  here in numpy, reproduces the fused slab).
* census, the summary figures of a set of tensors (dabsLabs/Qwen3.8-Flash-
  Next-NVFP4, metric table and "What makes this build different"): values
  worked by hand.
"""
import math

import numpy as np
import pytest

from conftest import read_golden
from test_oracle_nvfp4 import bits_of, to_bf16_bits, unpack_codes


def test_worked_example_with_a_given_scale(orc):
    # The golden example has s2 = 1; given s2 = 1 the blocks come out the
    # same with or without the element that set the group amax.
    for keep_amax in (True, False):
        x = np.zeros((1, 1, 48), np.float32)
        x[0, 0, 0] = 2688 if keep_amax else 0
        x[0, 0, 16], x[0, 0, 17] = 3, 1
        x[0, 0, 32], x[0, 0, 33] = 4, 3
        codes, scales, m4 = orc.quantize_nvfp4_s2(bits_of(x), np.ones(1, np.float32), mode=1)
        vals = unpack_codes(codes)[0, 0]
        for row in read_golden("nvfp4_worked.txt"):
            b, sc, M, c0, c1 = int(row[1]), int(row[3], 16), int(row[5]), int(row[7]), int(row[9])
            if b == 0 and not keep_amax:
                assert scales[0, 0, 0] == 0 and np.all(vals[:16] == 0)
                continue
            assert scales[0, 0, b] == sc, row
            assert m4[0, b] == (1 if M == 4 else 0), row
            assert vals[16 * b] == c0 and vals[16 * b + 1] == c1, row


def test_scale_below_the_group_amax_saturates(orc):
    # s2 = 2^-12, x0 = 6: t6 = 6 / (6 * 2^-12) = 4096 and t4 = 6144 both
    # saturate to E4M3 448 (0x7E), so the plans coincide (a tie: M=6);
    # d = 448 * 2^-12 and 6 / d = 54.9 saturates to E2M1 6 (code 7); -6 gives
    # code 0xF; 0.5 / d = 4.57 rounds to 4 (code 6).
    x = np.zeros((1, 1, 16), np.float32)
    x[0, 0, :3] = (6.0, -6.0, 0.5)
    codes, scales, m4 = orc.quantize_nvfp4_s2(bits_of(x), np.float32([2.0 ** -12]), mode=1)
    vals = unpack_codes(codes)[0, 0]
    assert scales[0, 0, 0] == 0x7E and m4[0, 0] == 0
    assert list(vals[:3]) == [0x7, 0xF, 0x6] and np.all(vals[3:] == 0)


def test_zero_scale_gives_zero_codes_and_scales(orc):
    x = np.random.default_rng(3).normal(0, 0.1, (2, 4, 32)).astype(np.float32)
    codes, scales, m4 = orc.quantize_nvfp4_s2(to_bf16_bits(x), np.zeros(2, np.float32), mode=1)
    assert not codes.any() and not scales.any() and not m4.any()


@pytest.mark.parametrize("bad", [-1.0, float("nan"), float("inf")])
def test_invalid_scale_is_rejected(orc, bad):
    x = np.zeros((1, 1, 16), np.uint16)
    with pytest.raises(RuntimeError):
        orc.quantize_nvfp4_s2(x, np.float32([bad]), mode=1)


@pytest.mark.parametrize("mode", [0, 1])
def test_gate_and_up_apart_with_the_shared_scale_reproduce_the_fused_slab(orc, mode):
    rng = np.random.default_rng(11)
    E, I, H = 3, 8, 64
    x = rng.normal(0, 0.02, (E, 2 * I, H)).astype(np.float32)
    x[1, I + 2, 5] = 0.4            # expert 1: the amax sits in up
    x[2, 3, 7] = -0.3               # expert 2: in gate
    xb = to_bf16_bits(x)
    c, s, s2, m4 = orc.quantize_nvfp4(xb, mode=mode)
    xf = (xb.astype(np.uint32) << 16).view(np.float32)
    amax = np.maximum(np.abs(xf[:, :I]).max(axis=(1, 2)), np.abs(xf[:, I:]).max(axis=(1, 2)))
    shared = (amax.astype(np.float32) / np.float32(2688.0)).astype(np.float32)
    assert np.array_equal(shared.view(np.uint32), s2.view(np.uint32))
    cg, sg, mg = orc.quantize_nvfp4_s2(np.ascontiguousarray(xb[:, :I]), shared, mode=mode)
    cu, su, mu = orc.quantize_nvfp4_s2(np.ascontiguousarray(xb[:, I:]), shared, mode=mode)
    assert np.array_equal(np.concatenate([cg, cu], axis=1), c)
    assert np.array_equal(np.concatenate([sg, su], axis=1), s)
    nb = I * H // 16
    assert np.array_equal(np.concatenate([mg, mu], axis=1), m4.reshape(E, 2 * nb))
    # separate scales per half (the convention the pages rule out) differ
    # wherever the halves' amax differ
    own = (np.abs(xf[:, :I]).max(axis=(1, 2)).astype(np.float32) / np.float32(2688.0)).astype(np.float32)
    cg2, _, _ = orc.quantize_nvfp4_s2(np.ascontiguousarray(xb[:, :I]), own, mode=mode)
    assert not np.array_equal(cg2[1], cg[1])


def test_census_values_worked_by_hand(orc):
    # rel = sqrt(err) / sqrt(ref) = 0.5, 0.5, 0 -> mean 1/3, max 0.5;
    # SSE against RTN: (1 + 4 + 0) / (2 + 8 + 0) - 1 = -0.5; M=4: 3 of 12
    r = orc.census([1.0, 4.0, 0.0], [4.0, 16.0, 1.0], err_rtn=[2.0, 8.0, 0.0], m4_blocks=3, blocks=12)
    assert r["n_tensors"] == 3
    assert r["mean_relerr"] == pytest.approx(1.0 / 3.0, rel=1e-15)
    assert r["max_relerr"] == 0.5
    assert r["sum_sq_err"] == 5.0 and r["sum_sq_ref"] == 21.0
    assert r["sse_vs_rtn"] == -0.5
    assert r["m4_fraction"] == 0.25


def test_census_of_one_tensor_and_of_an_unmatched_error(orc):
    r = orc.census([9.0], [16.0])
    assert r["mean_relerr"] == r["max_relerr"] == 0.75 and r["sse_vs_rtn"] is None
    r = orc.census([1.0, 0.0], [0.0, 0.0])       # an all-zero tensor that was not reproduced
    assert math.isinf(r["max_relerr"]) and r["m4_fraction"] == 0.0
