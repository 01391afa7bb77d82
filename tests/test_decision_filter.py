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
from the exact-rational restatement in oracle/micro.py.

The same emulation covers the weighted scale search's fp32 filter: every
candidate's fp32 weighted error W32 (the kernel's operation order) lies
within half its error bound eps of both the exact weighted error and the
binary64 value the definition forms, a block the filter decides gets the
binary64 argmin, and blocks whose binary64 scores tie are never decided."""
from fractions import Fraction as F

import numpy as np
import torch

from oracle import micro
from exact_fp import rn32


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


# ---- the weighted search's fp32 scores and their bound -------------------
def _wsse32(xs, hs, codes, D, s2):
    """The kernel's fp32 weighted error of one candidate: with the
    candidate's divisor d = RN(D s2), per element e = RN(x - q d) (one FMA),
    then acc = RN(h RN(e e) + acc) in two interleaved partial sums (even /
    odd elements), added at the end."""
    d = rn32(D * F(float(s2)))
    acc = [F(0), F(0)]
    for i, (x, h, c) in enumerate(zip(xs, hs, codes)):
        e = rn32(F(float(x)) - micro.e2m1_value(c) * d)
        acc[i & 1] = rn32(F(float(h)) * rn32(e * e) + acc[i & 1])
    return rn32(acc[0] + acc[1])


def _wsse64(xs, hs, codes, D, s2):
    """The definition's binary64 procedure (Python floats are binary64)."""
    acc = 0.0
    for x, h, c in zip(xs, hs, codes):
        deq = float(micro.e2m1_value(c) * D) * float(s2)     # exact: 4 + 24 bits
        e = float(x) - deq
        acc = acc + float(h) * (e * e)
    return acc


def _weighted_case(xs, hs, s2):
    """One block of the weighted search: checks every candidate's fp32 score
    against its bound and the filter's decision against the binary64 argmin.
    Returns (candidates checked, decided, binary64 argmin was a tie)."""
    # A as the kernel forms it: acc = RN(h RN(x x) + acc) in two partial sums
    acc = [F(0), F(0)]
    for i, (x, h) in enumerate(zip(xs, hs)):
        acc[i & 1] = rn32(F(float(h)) * rn32(F(float(x)) ** 2) + acc[i & 1])
    A = rn32(acc[0] + acc[1])
    if not (F(2) ** -60 <= A <= F(2) ** 100):
        return 0, False, False
    sc6, _, _ = micro.plan(xs, s2, 6)
    sc4, _, _ = micro.plan(xs, s2, 4)
    cands = []
    for sc in range(sc6, sc4 + 1):
        codes, _ = micro.plan_with_scale_code(xs, s2, sc)
        D = F(micro.e4m3_value(sc))
        w32 = _wsse32(xs, hs, codes, D, s2)
        exact = sum(F(float(h)) * (F(float(x)) - micro.e2m1_value(c) * D * F(float(s2))) ** 2
                    for x, h, c in zip(xs, hs, codes))
        w64 = F(_wsse64(xs, hs, codes, D, s2))
        eps = (F(2.0 ** -22 * float(A * w32) ** 0.5) + F(2.0 ** -19) * w32
               + F(2.0 ** -45) * A + F(2.0 ** -100))
        # the constants take about twice the derived error: half of eps must do
        assert abs(w32 - exact) <= eps / 2, (sc, float(w32), float(exact))
        assert abs(w32 - w64) <= eps / 2, (sc, float(w32), float(w64))
        cands.append((sc, w32, eps, w64))
    # the filter: the fp32 argmin (first on equal scores) is kept when every
    # other candidate's W - eps lies above the best's W + eps
    best = min(range(len(cands)), key=lambda i: (cands[i][1], i))
    bw, be = cands[best][1], cands[best][2]
    lb = min((w - e for i, (_, w, e, _) in enumerate(cands) if i != best), default=None)
    decided = lb is None or lb > bw + be
    w64s = [c[3] for c in cands]
    arg64 = min(range(len(cands)), key=lambda i: (w64s[i], i))
    tie64 = w64s.count(w64s[arg64]) > 1
    if decided:
        assert cands[best][0] == cands[arg64][0]
        assert not tie64
    return len(cands), decided, tie64


def test_weighted_fp32_bound_and_filter():
    rng = np.random.default_rng(33)
    s2 = micro.global_scale(np.float32(2.625))
    checked = decided = 0
    for _ in range(60):
        xs = _bf16(np.clip(rng.standard_normal(16) * rng.choice([0.05, 0.3]), -2.625, 2.625))
        hs = [np.float32(v) for v in rng.gamma(0.7, 1.0, 16)]
        n, d, _ = _weighted_case(xs, hs, s2)
        checked += n
        decided += d
    assert checked > 250 and decided > 40


def test_weighted_filter_leaves_ties_to_binary64():
    """One-hot weights on a grid-exact element: several candidates score the
    same, and the filter must hand every such block to the binary64 search."""
    rng = np.random.default_rng(34)
    s2 = np.float32(2.0 ** -10)
    ties = 0
    for _ in range(60):
        base = float(2.0 ** int(rng.integers(-3, 4))) * float(s2)
        v = rng.choice([0.5, 1.0, 1.5, 2.0, 3.0, -1.0, -2.0], 16) * base
        v[rng.integers(16)] = 6.0 * base
        xs = _bf16(v)
        hs = [np.float32(0.0)] * 16
        hs[int(rng.integers(16))] = np.float32(rng.choice([0.25, 1.0, 3.0]))
        _, _, tie = _weighted_case(xs, hs, s2)
        ties += tie
    assert ties > 20
