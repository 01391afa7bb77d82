"""Pins of the oracle's FP8 -> MX requantization (oracle_requant_fp8_mx).

The conversion starts from block-FP8 weights (MJPansa/Qwen3.8-Flash-Next-
MXFP4-FP8-R12, "Quantization and layer selection"); the block shape and the
fp32 intermediate are readings.  Pinned by a hand-worked block, by the
special case where every dequantized value is exactly a bf16 (then the
requantization must equal the already pinned bf16 MX quantizer on those
values), by power-of-two scale changes (codes fixed, scale bytes shifted),
and by rejection of the E4M3 NaN code."""
import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden
from mxfp_block_scaled_b200 import workloads


def test_hand_worked_block():
    q = np.full((1, 32), 0x38, np.uint8)
    q[0, 0] = 0x7E
    s = np.array([[0.1]], np.float32)
    for fmt, sbyte, c0, crest in read_golden("fp8_requant_worked.txt"):
        codes, scales = oracle.requant_fp8_mx(q, s, 128, 128, fmt)
        assert scales[0, 0] == int(sbyte), fmt
        assert codes[0, 0] == int(c0, 16), fmt
        assert np.all(codes[0, 1:] == int(crest, 16)), fmt


def _e4m3_values(q):
    return np.array([oracle.e4m3_value(int(c)) for c in q.reshape(-1)]).reshape(q.shape)


@pytest.mark.parametrize("fmt", ["mxfp8", "mxfp4"])
def test_bf16_exact_case_reduces_to_the_bf16_quantizer(fmt):
    """Scales of the form 1.5 * 2^k: E4M3 (4 significant bits) times 1.5
    (2 bits) needs at most 6 bits, so every dequantized value is an exact
    bf16 and the fp32 step rounds nothing."""
    codes, _ = workloads.block_fp8_source(96, 256, seed=3, brows=32, bcols=64)
    q = codes.numpy()
    k = np.random.default_rng(3).integers(-20, -4, size=(3, 4))
    s = (1.5 * np.exp2(k)).astype(np.float32)
    c1, s1 = oracle.requant_fp8_mx(q, s, 32, 64, fmt)
    w = _e4m3_values(q) * np.repeat(np.repeat(s.astype(np.float64), 32, 0), 64, 1)
    wb = torch.from_numpy(w.astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(wb.float().double().numpy(), w)          # exact in bf16
    c2, s2 = oracle.quantize_mx(workloads.bf16_bits(wb), fmt)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


def test_power_of_two_scale_shifts_only_the_scale_bytes():
    codes, scales = workloads.block_fp8_source(128, 256, seed=5)
    q, s = codes.numpy(), scales.numpy()
    for fmt in ("mxfp8", "mxfp4"):
        c1, b1 = oracle.requant_fp8_mx(q, s, 128, 128, fmt)
        c2, b2 = oracle.requant_fp8_mx(q, s * np.float32(8.0), 128, 128, fmt)
        assert np.array_equal(c1, c2)
        live = b1 > 0                                   # all-zero blocks stay at byte 0
        assert np.array_equal(b2[live].astype(int), b1[live].astype(int) + 3)


def test_nan_source_is_rejected():
    q = np.full((1, 32), 0x38, np.uint8)
    q[0, 7] = 0xFF
    with pytest.raises(RuntimeError):
        oracle.requant_fp8_mx(q, np.ones((1, 1), np.float32), 128, 128, "mxfp8")


def test_dequantized_value_is_rounded_to_fp32_once():
    """Reading of the fp32 intermediate: w = RN32(E4M3(code) * scale).  With
    scale = RN32(1.25 / 1.125), the value 1.125 dequantizes to exactly 1.25
    after that rounding (an E2M1 tie once the block's exponent is 0, kept at
    the even code 2), while the unrounded product lies 2^-24 above the tie
    and would take the odd code 3."""
    from fractions import Fraction as F
    from oracle import micro
    sc = np.float32(np.float32(1.25) / np.float32(1.125))
    q = np.zeros((1, 32), np.uint8)
    q[0, 0] = 0x48                                       # 4.0: w = 4.44, block exponent 0
    q[0, 1] = 0x39                                       # 1.125
    codes, scales = oracle.requant_fp8_mx(q, np.array([[sc]], np.float32), 128, 128, "mxfp4")
    assert scales[0, 0] == 127
    assert codes[0, 0] == 0x6 | (0x2 << 4)               # 4.44 -> 4 (code 6), 1.25 -> 1.0 (code 2)
    assert np.all(codes[0, 1:] == 0)
    exact = F(9, 8) * F(float(sc))
    assert exact - F(5, 4) == F(1, 2 ** 24)
    assert micro.e2m1_encode(np.float32(exact)) == 2     # rounded once: the tie
    assert micro.E2M1_GRID[3] - exact < exact - micro.E2M1_GRID[2]   # unrounded: nearer 1.5
