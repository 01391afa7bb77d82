"""The fp32 form of the exact 4/6 decision that the NVFP4 kernel uses (the
block quantizer's filtered comparison), checked in exact arithmetic on the
CPU.  Every fp32 operation of the kernel's sequence is emulated as
round-to-nearest-even of the exact rational result, and the test asserts:
  - P = D6^2 B6 - D4^2 B4 comes out exact (the argument: 1 <= D4/D6 <= 2, so
    both terms are integer multiples of 2^(2 e6 - 2) below 2^(2 e6 + 20));
  - whenever |dl| > 2^-20 (|v4| + |Q|), the sign of dl is the sign of the
    exact G6/2 - G4/2 and the two are not equal, so the filter never decides
    against the exact comparison;
on random blocks and on tie-rich and near-tie blocks (grid-exact blocks, then
the same blocks with one element moved by one bf16 ulp).  The plans come
from the exact-rational restatement in oracle/micro.py."""
from fractions import Fraction as F

import numpy as np
import torch

from oracle import micro


def rn32(q):
    """Round a rational to the nearest fp32 (ties to even), as a Fraction.
    Normal range only (the fast path keeps every operand there)."""
    if q == 0:
        return F(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if F(2) ** e > a:
        e -= 1
    assert -126 <= e <= 127
    m = a / F(2) ** (e - 23)                    # in [2^23, 2^24)
    n = m.numerator // m.denominator
    r = m - n
    if r > F(1, 2) or (r == F(1, 2) and n % 2 == 1):
        n += 1
    return sign * F(n) * F(2) ** (e - 23)


def plan_sums(xs, s2, M):
    sc, codes, _ = micro.plan(xs, s2, M)
    q = [micro.e2m1_value(c) for c in codes]
    A = sum(F(float(x)) * qi for x, qi in zip(xs, q))
    B = sum(qi * qi for qi in q)
    return sc, F(micro.e4m3_value(sc)), A, B


def filtered_decision(xs, s2):
    """(decided, use4_filter, exact_use4, exact_tie, P_exact_ok) for one block
    on the fast path, or None when the block is not on it."""
    sc6, D6, A6, B6 = plan_sums(xs, s2, 6)
    sc4, D4, A4, B4 = plan_sums(xs, s2, 4)
    if sc6 == 0 or sc4 == 0:
        return None
    s2f = F(float(s2))
    s2h = s2f / 2                               # exact in fp32
    # the kernel's sequence (A and B are exact fp32 values)
    assert rn32(A6) == A6 and rn32(A4) == A4 and rn32(B6) == B6 and rn32(B4) == B4
    u6, u4 = rn32(D6 * B6), rn32(D4 * B4)
    P = rn32(D6 * u6 - rn32(D4 * u4))
    p_exact = P == D6 * D6 * B6 - D4 * D4 * B4
    v4 = rn32(D4 * A4)
    Q = rn32(D6 * A6 - v4)
    dl = rn32(s2h * P - Q)
    thr = rn32(rn32(abs(v4) + abs(Q)) * F(1, 2 ** 20))
    decided = abs(dl) > thr
    g6 = D6 * (D6 * s2h * B6 - A6)
    g4 = D4 * (D4 * s2h * B4 - A4)
    return decided, dl > 0, g4 < g6, g4 == g6, p_exact


def _bf16(v):
    return [np.float32(t) for t in torch.tensor(np.asarray(v, np.float32)).to(torch.bfloat16).float().numpy()]


def _check(blocks, s2):
    decided = 0
    for xs in blocks:
        r = filtered_decision(xs, s2)
        if r is None:
            continue
        d, use4_f, use4_x, tie, p_ok = r
        assert p_ok
        if d:
            decided += 1
            assert not tie
            assert use4_f == use4_x
    return decided


def test_random_blocks():
    rng = np.random.default_rng(31)
    amax_g = 2.625
    s2 = micro.global_scale(np.float32(amax_g))
    blocks = []
    for _ in range(300):
        v = rng.standard_normal(16) * rng.choice([0.05, 0.2, 0.6])
        v[rng.random(16) < 0.05] *= 6
        blocks.append(_bf16(np.clip(v, -amax_g, amax_g)))
    assert _check(blocks, s2) > 250


def test_ties_and_near_ties():
    """Grid-exact blocks make both plans' errors equal (the filter must not
    decide them); moving one element by one bf16 ulp makes them near-ties."""
    rng = np.random.default_rng(32)
    s2 = np.float32(2.0 ** -10)
    ok_scales = [v for v in micro.E4M3_LIST[1:127] if 1.5 * v in micro.E4M3_LIST and 1.5 * v <= 298]
    blocks = []
    for _ in range(150):
        base = float(ok_scales[rng.integers(len(ok_scales))]) * float(s2)
        v = rng.choice([0.0, 1.5, 3.0, 6.0, -1.5, -3.0, -6.0], 16) * base
        v[rng.integers(16)] = 6.0 * base
        xs = _bf16(v)
        blocks.append(xs)
        nz = [i for i in range(16) if xs[i] != 0]
        k = nz[rng.integers(len(nz))]                # a non-zero element: its bits +-1 stay finite
        bits = torch.tensor([float(xs[k])], dtype=torch.float32).to(torch.bfloat16).view(torch.int16)
        moved = (bits + int(rng.choice([-1, 1]))).view(torch.bfloat16).float().item()
        near = list(xs)
        near[k] = np.float32(moved)
        blocks.append(near)
    _check(blocks, s2)
    # the exact ties are present and left to the exact comparison
    ties = sum(1 for xs in blocks[::2] if (r := filtered_decision(xs, s2)) and r[3])
    assert ties > 50
