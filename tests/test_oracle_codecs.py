"""Pins of the oracle's number formats against facts that do not come from
the oracle: hand-derived golden tables, an exact rational restatement of
the formats (oracle/micro.py), and closed forms."""
import math
from fractions import Fraction as F

import numpy as np
import pytest

from conftest import read_golden
from oracle import micro


def _bf16_values(positive_only=False):
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    f = f[np.isfinite(f)]
    if positive_only:
        f = f[f > 0]
    return f


def test_e2m1_decode_matches_golden_grid(orc):
    rows = read_golden("e2m1_grid.txt")
    assert len(rows) == 16
    for code, val in rows:
        v = orc.e2m1_value(int(code))
        assert v == float(val)
        assert math.copysign(1.0, v) == math.copysign(1.0, float(val))


def test_e2m1_round_trip_all_codes(orc):
    for c in range(16):
        assert orc.e2m1_encode(orc.e2m1_value(c)) == c


def test_e2m1_ties_golden(orc):
    for x, code in read_golden("e2m1_ties.txt"):
        # inputs are fp32 values (the kernel rounds an fp32 quotient)
        assert orc.e2m1_encode(float(np.float32(float(x)))) == int(code), x


def test_e2m1_encode_matches_rational_nearest_on_all_bf16(orc):
    vals = _bf16_values()
    # scale into the interesting range too: grid-relative positions
    for scale in (1.0, 2.0 ** -3, 2.0 ** 3):
        with np.errstate(over="ignore"):
            scaled = vals[::7] * np.float32(scale)
        for v in scaled:
            if not np.isfinite(v):
                continue
            assert orc.e2m1_encode(float(v)) == micro.e2m1_encode(v), v


def test_e2m1_encode_at_every_midpoint_and_neighbours(orc):
    grid = [float(g) for g in micro.E2M1_GRID]
    for a, b in zip(grid[:-1], grid[1:]):
        m = np.float32((a + b) / 2)
        for v in (np.nextafter(m, np.float32(-1)), m, np.nextafter(m, np.float32(10))):
            for s in (1, -1):
                x = np.float32(s * v)
                assert orc.e2m1_encode(float(x)) == micro.e2m1_encode(x)


def test_e4m3_decode_golden_points(orc):
    for code, val in read_golden("e4m3_points.txt"):
        v = orc.e4m3_value(int(code, 16))
        if val == "nan":
            assert math.isnan(v)
        else:
            assert v == float(val)
            assert math.copysign(1.0, v) == math.copysign(1.0, float(val))


def test_e4m3_decode_all_codes_match_sorted_value_list(orc):
    for c in range(256):
        if c & 0x7F == 0x7F:
            assert math.isnan(orc.e4m3_value(c))
            continue
        assert F(orc.e4m3_value(c)) == micro.e4m3_value(c)


def test_e4m3_round_trip_and_saturation(orc):
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue
        assert orc.e4m3_encode(orc.e4m3_value(c)) == c
    assert orc.e4m3_encode(448.0) == 0x7E
    assert orc.e4m3_encode(463.99) == 0x7E
    assert orc.e4m3_encode(1e30) == 0x7E
    assert orc.e4m3_encode(-1e30) == 0xFE
    assert orc.e4m3_encode(2.0 ** -10) == 0x00        # tie with 0 -> even code 0
    assert orc.e4m3_encode(3 * 2.0 ** -11) == 0x01    # 0.75 * 2^-9: nearer 2^-9
    assert orc.e4m3_encode(3 * 2.0 ** -10) == 0x02    # 1.5 * 2^-9: tie, even code
    assert orc.e4m3_encode(2.0 ** -6 - 2.0 ** -11) == 0x08  # tie 0x07/0x08 -> even
    assert orc.e4m3_encode(-(2.0 ** -12)) == 0x80


def test_e4m3_encode_matches_rational_nearest_at_midpoints(orc):
    vals = [float(v) for v in micro.E4M3_LIST]
    for a, b in zip(vals[:-1], vals[1:]):
        m = np.float32((a + b) / 2)
        for v in (np.nextafter(m, np.float32(-1)), m, np.nextafter(m, np.float32(1e9))):
            assert orc.e4m3_encode(float(v)) == micro.e4m3_encode(v), v


def test_e4m3_encode_matches_rational_nearest_on_random_fp32(orc):
    rng = np.random.default_rng(1)
    v = np.float32(2.0) ** rng.uniform(-12, 10, 4000).astype(np.float32)
    v *= rng.choice(np.array([-1, 1], np.float32), v.size)
    for x in v.astype(np.float32):
        assert orc.e4m3_encode(float(x)) == micro.e4m3_encode(x), x


def test_ue8m0_values(orc):
    assert orc.ue8m0_value(127) == 1.0
    assert orc.ue8m0_value(0) == 2.0 ** -127
    assert orc.ue8m0_value(254) == 2.0 ** 127
    assert math.isnan(orc.ue8m0_value(255))


def test_mx_exponent_golden(orc):
    for amax, qmax, e in read_golden("mx_exponent.txt"):
        assert orc.mx_exponent(float(amax), float(qmax)) == int(e), (amax, qmax)


@pytest.mark.parametrize("qmax", [448, 6])
def test_mx_exponent_every_bf16_amax(orc, qmax):
    """Every positive finite bf16 amax: the exponent is the smallest integer
    e (clamped to [-127, 127]) with amax <= qmax * 2^e, computed here with
    Python rationals from frexp."""
    Q = F(qmax)
    for a in _bf16_values(positive_only=True):
        A = F(float(a))
        m, ex = math.frexp(float(a) / qmax)
        e = ex - 1                        # log2 candidate from below
        while A > Q * F(2) ** e:
            e += 1
        while e > -200 and A <= Q * F(2) ** (e - 1):
            e -= 1
        e = max(-127, min(127, e))
        assert orc.mx_exponent(float(a), float(qmax)) == e, a
