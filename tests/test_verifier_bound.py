"""The verifier's fp32 arithmetic emulated exactly on the CPU, against the
exact sums the oracle's definition gives.  Per element the kernel forms
e = RN32(x - deq) with one rounding (NVFP4: one FMA of the exact q * D with
-s2; MX: deq = q * 2^e is exact), adds e^2 and x^2 by fp32 FMAs into two
partial sums of 8 terms (even / odd elements of 16), adds the pair once in
fp32 and then in fp64.  So err is within 11 * 2^-24 and ref within 9 * 2^-24
of the exact sums whatever the data, inside the 1e-6 relative agreement
asked of the verifier.  The fp64 additions across blocks are summed exactly
here: they add at most a few times 2^-53 relative.

The constructed tensor at the end has errors of a few fp32 ulps of the
reconstruction: there, rounding deq to fp32 before subtracting would be off
by tens of percent, while the single rounding stays within the bound."""
from fractions import Fraction as F

import numpy as np
import pytest
import torch

import oracle
from oracle import micro
from exact_fp import rn32

U = F(1, 2 ** 24)


def _bf16(shape, scale, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


def _half_sums(xs, deqs, fused_deq=None):
    """One run of 16 elements: the kernel's two interleaved fp32 partials of
    8 terms each, added once.  fused_deq(i) gives the exact value the FMA
    subtracts (NVFP4); otherwise deqs[i] is an exact fp32 value (MX)."""
    e_acc, r_acc = [F(0), F(0)], [F(0), F(0)]
    for i, x in enumerate(xs):
        d = fused_deq(i) if fused_deq else deqs[i]
        e = rn32(x - d)
        e_acc[i & 1] = rn32(e * e + e_acc[i & 1])
        r_acc[i & 1] = rn32(x * x + r_acc[i & 1])
    return rn32(e_acc[0] + e_acc[1]), rn32(r_acc[0] + r_acc[1])


def _check(err_k, ref_k, err_x, ref_x):
    assert abs(err_k - err_x) <= 11 * U * err_x
    assert abs(ref_k - ref_x) <= 9 * U * ref_x


def test_bound_is_inside_the_verifier_tolerance():
    assert float(11 * U) < 1e-6 and float(9 * U) < 1e-6


@pytest.mark.parametrize("seed", [0, 1])
def test_nvfp4_tensor_sums(seed):
    x = _bf16((2, 32, 64), 0.02, seed)
    x[0, 3, 5] = 0.3                                     # an outlier block
    bits = x.view(torch.int16).numpy().view(np.uint16)
    codes, scales, s2, _ = oracle.quantize_nvfp4(bits, mode=1)
    xv = [F(float(v)) for v in x.float().reshape(-1).tolist()]
    for t in range(2):                                  # one tensor per group
        err_k = ref_k = err_x = ref_x = F(0)
        s2f = F(float(s2[t]))
        nb = 32 * 64 // 16
        for b in range(nb):
            gb = t * nb + b
            D = F(micro.e4m3_value(int(scales.reshape(-1)[gb])))
            cb = codes.reshape(-1)[gb * 8:(gb + 1) * 8]
            q = [F(micro.e2m1_value(int(c) >> (4 * h) & 0xF)) for c in cb for h in (0, 1)]
            xs = xv[gb * 16:(gb + 1) * 16]
            e, r = _half_sums(xs, None, fused_deq=lambda i: q[i] * D * s2f)
            err_k += e
            ref_k += r
            err_x += sum((xi - qi * D * s2f) ** 2 for xi, qi in zip(xs, q))
            ref_x += sum(xi * xi for xi in xs)
        _check(err_k, ref_k, err_x, ref_x)
        # and against the oracle's own binary64 sums
        oe, orf = oracle.dequant_relerr(bits[t:t + 1], codes[t:t + 1], scales[t:t + 1], s2[t:t + 1],
                                        "nvfp4", 1, 32, 64, 1)
        assert abs(F(float(oe[0])) - err_x) <= 1e-12 * err_x


@pytest.mark.parametrize("fmt", ["mxfp8", "mxfp4"])
def test_mx_tensor_sums(fmt):
    x = _bf16((32, 64), 1.0, 7)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    codes, scales = oracle.quantize_mx(bits, fmt)
    xv = [F(float(v)) for v in x.float().reshape(-1).tolist()]
    err_k = ref_k = err_x = ref_x = F(0)
    for b in range(32 * 64 // 32):
        sc = F(2) ** (int(scales.reshape(-1)[b]) - 127)
        if fmt == "mxfp8":
            q = [F(micro.e4m3_value(int(c))) for c in codes.reshape(-1)[b * 32:(b + 1) * 32]]
        else:
            q = [F(micro.e2m1_value(int(c) >> (4 * h) & 0xF))
                 for c in codes.reshape(-1)[b * 16:(b + 1) * 16] for h in (0, 1)]
        deq = [qi * sc for qi in q]
        assert all(rn32(d) == d for d in deq)             # exact in fp32
        xs = xv[b * 32:(b + 1) * 32]
        for h in (0, 16):                                 # the two halves of 8 pairs
            e, r = _half_sums(xs[h:h + 16], deq[h:h + 16])
            err_k += e
            ref_k += r
        err_x += sum((xi - d) ** 2 for xi, d in zip(xs, deq))
        ref_x += sum(xi * xi for xi in xs)
    _check(err_k, ref_k, err_x, ref_x)


def test_errors_of_a_few_ulps_need_the_single_rounding():
    """x = 3 stored as q = 1.5, D = 2 with s2 = 1 + 2^-23: the exact error is
    3 * 2^-23 per element.  One rounding of x - q D s2 keeps it exactly;
    rounding deq first gives 2^-21 (a 78 % larger square)."""
    s2 = F(1) + F(1, 2 ** 23)                             # an fp32 value
    assert rn32(s2) == s2
    xs, q, D = [F(3)] * 16, F(3, 2), F(2)
    exact = sum((x - q * D * s2) ** 2 for x in xs)
    e_one, _ = _half_sums(xs, None, fused_deq=lambda i: q * D * s2)
    e_two, _ = _half_sums(xs, [rn32(q * D * s2)] * 16)
    assert abs(e_one - exact) <= 11 * U * exact
    assert (e_two - exact) / exact > F(1, 2)
