"""Exact rational micro-oracle for tiny blocks (test infrastructure only).

An independent second statement of the NVFP4 block quantizer and of the
exact squared error that the 4/6 decision compares, in Python
``fractions.Fraction`` arithmetic, used to pin the C oracle on small
inputs.  It shares nothing with ``mxq_oracle.c`` beyond reading the same
pages:

* dabsLabs/Qwen3.8-Flash-Next-NVFP4, "What makes this build different":
  per 16-element block, the amax/6 plan and the four-over-six plan are
  both encoded and the one with the lower exact post-rounding squared
  error is kept (never worse than plain RTN).
* josch15366/Qwen3.8-Flash-Next-NVFP4-LocalHessian-Experts, introduction:
  the global scale is amax / 2688 (= amax / (6 * 448)).

The fp32 steps (RN32 of a quotient or product) are taken with numpy
float32 scalars, which round each operation to nearest even.  Formats are
built here as sorted value lists, not decoded from bit fields: the E2M1
grid is the list {0, 0.5, 1, 1.5, 2, 3, 4, 6}; the E4M3 list is every
m/8 * 2^-6 (m = 0..7) followed by every (1 + m/8) * 2^k for k = -6..8
that does not exceed 448.  For non-negative values the code equals the
position in the sorted list, which is how both formats order their codes.
"""
from fractions import Fraction as F

import numpy as np

E2M1_GRID = [F(0), F(1, 2), F(1), F(3, 2), F(2), F(3), F(4), F(6)]


def _e4m3_list():
    vals = [F(m, 8) * F(1, 64) for m in range(8)]
    for k in range(-6, 9):
        for m in range(8):
            v = (1 + F(m, 8)) * (F(2) ** k)
            if v <= 448:
                vals.append(v)
    return vals


E4M3_LIST = _e4m3_list()
assert len(E4M3_LIST) == 127 and E4M3_LIST[-1] == 448


def _nearest_index(v, grid):
    """Index of the grid value nearest |v|; ties to the even index;
    beyond the last value saturate to it."""
    a = abs(v)
    if a >= grid[-1]:
        return len(grid) - 1
    lo = max(i for i, g in enumerate(grid) if g <= a)
    if grid[lo] == a or lo == len(grid) - 1:
        return lo
    hi = lo + 1
    dl, dh = a - grid[lo], grid[hi] - a
    if dl < dh:
        return lo
    if dh < dl:
        return hi
    return lo if lo % 2 == 0 else hi


def _is_negative(v_float):
    return bool(np.signbit(v_float))


def e2m1_encode(y):
    """y: a float (np.float32 or float).  Code with sign bit 3."""
    idx = _nearest_index(F(float(y)), E2M1_GRID)
    return idx | (8 if _is_negative(y) else 0)


def e2m1_value(code):
    v = E2M1_GRID[code & 7]
    return -v if code & 8 else v


def e4m3_encode(t):
    idx = _nearest_index(F(float(t)), E4M3_LIST)
    return idx | (0x80 if _is_negative(t) else 0)


def e4m3_value(code):
    v = E4M3_LIST[code & 0x7F]
    return -v if code & 0x80 else v


def f32(v):
    return np.float32(v)


def plan_with_scale_code(x, s2, sc):
    """Codes and exact SSE of a block for a given E4M3 scale code.
    x: list of np.float32, s2: np.float32."""
    D = e4m3_value(sc)
    d = f32(f32(float(D)) * s2)
    if D == 0 or d == 0:
        codes = [0] * len(x)
    else:
        codes = [e2m1_encode(f32(xi / d)) for xi in x]
    s2f = F(float(s2))
    sse = sum((F(float(xi)) - e2m1_value(c) * D * s2f) ** 2 for xi, c in zip(x, codes))
    return codes, sse


def plan(x, s2, M):
    """One plan: scale code from t = RN32(amax_b / RN32(M * s2))."""
    if s2 == 0:
        return 0, [0] * len(x), sum(F(float(xi)) ** 2 for xi in x)
    amax_b = max(abs(xi) for xi in x)
    t = f32(amax_b / f32(f32(M) * s2))
    sc = e4m3_encode(t)
    codes, sse = plan_with_scale_code(x, s2, sc)
    return sc, codes, sse


def block_four_six(x, s2):
    """(M, scale_code, codes, sse_chosen, sse_6, sse_4) for one block:
    M=4 only if its exact SSE is strictly lower."""
    sc6, c6, e6 = plan(x, s2, 6)
    sc4, c4, e4 = plan(x, s2, 4)
    if e4 < e6:
        return 4, sc4, c4, e4, e6, e4
    return 6, sc6, c6, e6, e6, e4


def best_scale_sse(x, s2):
    """Brute force: lowest exact SSE over every non-negative finite E4M3
    scale code (the value codes follow from the scale as in every plan)."""
    return min(plan_with_scale_code(x, s2, sc)[1] for sc in range(127))


def global_scale(amax_g):
    return f32(f32(amax_g) / f32(2688.0))
