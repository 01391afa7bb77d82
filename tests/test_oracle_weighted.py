"""Pins of the oracle's weighted-SSE scale search (oracle_quantize_nvfp4_weighted).

The pages say only that the Local-Hessian build chooses its per-group scales
by a Hessian-weighted search instead of the plain amax / MSE sweep
(josch15366/Qwen3.8-Flash-Next-NVFP4-LocalHessian-Experts, "What is
different about it").  The reading (candidate codes from the amax/6 plan's
to the four-over-six plan's, objective sum h (x - q D s2)^2 in binary64 in a
fixed order, ties to the smaller code) is checked against an exact rational
restatement (oracle/micro.py builds the value codes independently of the C
oracle), plus invariants: never worse than either 4/6 plan, invariant
under power-of-two weight scaling, and a one-hot weight picks the scale
that best reproduces that element."""
from fractions import Fraction as F

import numpy as np
import pytest

import oracle
from oracle import micro


def _blocks(seed, n, std=0.03):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((n, 16)) * std).astype(np.float32)
    x[rng.random((n, 16)) < 0.02] *= 8
    import torch
    xb = torch.from_numpy(x).to(torch.bfloat16)
    bits = xb.view(torch.int16).numpy().view(np.uint16)
    return bits, xb.float().numpy()


def _exact_wsse(xf, h, s2, sc):
    codes, _ = micro.plan_with_scale_code([np.float32(v) for v in xf], s2, sc)
    D, s2f = micro.e4m3_value(sc), F(float(s2))
    return codes, sum(F(float(hi)) * (F(float(xi)) - micro.e2m1_value(c) * D * s2f) ** 2
                      for xi, hi, c in zip(xf, h, codes))


def _candidates(xf, s2):
    sc6, _, _ = micro.plan([np.float32(v) for v in xf], s2, 6)
    sc4, _, _ = micro.plan([np.float32(v) for v in xf], s2, 4)
    return list(range(sc6, sc4 + 1))


def test_matches_the_exact_argmin_away_from_near_ties():
    bits, xf = _blocks(1, 160)
    rng = np.random.default_rng(2)
    h = rng.gamma(0.7, 1.0, size=16).astype(np.float32)
    codes, scales, s2 = oracle.quantize_nvfp4_weighted(bits.reshape(1, 160, 16), h)
    s2v = np.float32(s2[0])
    assert s2v == micro.global_scale(np.abs(xf).max())
    checked = 0
    for b in range(160):
        cands = _candidates(xf[b], s2v)
        vals = [(_exact_wsse(xf[b], h, s2v, sc), sc) for sc in cands]
        best = min(v[0][1] for v in vals)
        best_sc = min(sc for (c, w), sc in vals if w == best)
        others = [w for (c, w), sc in vals if w != best]
        if others and (min(others) - best) <= best * F(1, 10 ** 12):
            continue                       # a near-tie binary64 may decide either way
        checked += 1
        assert scales[0, b, 0] == best_sc, b
        c = dict((sc, cw[0]) for cw, sc in vals)[best_sc]
        packed = [(c[2 * j] & 15) | ((c[2 * j + 1] & 15) << 4) for j in range(8)]
        assert list(codes[0, b]) == packed, b
    assert checked > 150


def test_never_worse_than_either_four_six_plan():
    bits, xf = _blocks(3, 64)
    h = np.random.default_rng(4).uniform(0.0, 5.0, 16).astype(np.float32)
    _, scales, s2 = oracle.quantize_nvfp4_weighted(bits.reshape(1, 64, 16), h)
    s2v = np.float32(s2[0])
    for b in range(64):
        cands = _candidates(xf[b], s2v)
        chosen = _exact_wsse(xf[b], h, s2v, int(scales[0, b, 0]))[1]
        for sc in (cands[0], cands[-1]):
            assert chosen <= _exact_wsse(xf[b], h, s2v, sc)[1] * (1 + F(1, 10 ** 12))


def test_power_of_two_weight_scaling_changes_nothing():
    bits, _ = _blocks(5, 96)
    h = np.random.default_rng(6).uniform(0.1, 3.0, 32).astype(np.float32)
    a = oracle.quantize_nvfp4_weighted(bits.reshape(2, 24, 32), h)
    b = oracle.quantize_nvfp4_weighted(bits.reshape(2, 24, 32), h * np.float32(2.0 ** -7))
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


@pytest.mark.parametrize("k", [0, 5, 15])
def test_one_hot_weight_reproduces_that_element_best(k):
    bits, xf = _blocks(7 + k, 48)
    h = np.zeros(16, np.float32)
    h[k] = 1.0
    _, scales, s2 = oracle.quantize_nvfp4_weighted(bits.reshape(1, 48, 16), h)
    s2v = np.float32(s2[0])
    for b in range(48):
        errs = [(_exact_wsse(xf[b], h, s2v, sc)[1], sc) for sc in _candidates(xf[b], s2v)]
        best = min(e for e, _ in errs)
        assert scales[0, b, 0] == min(sc for e, sc in errs if e == best)


def test_shared_and_per_group_weights_and_rejects_bad_weights():
    bits, _ = _blocks(9, 64)
    h = np.random.default_rng(10).uniform(0.0, 2.0, 32).astype(np.float32)
    a = oracle.quantize_nvfp4_weighted(bits.reshape(2, 16, 32), h)
    b = oracle.quantize_nvfp4_weighted(bits.reshape(2, 16, 32), np.stack([h, h]))
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
    with pytest.raises(RuntimeError):
        oracle.quantize_nvfp4_weighted(bits.reshape(2, 16, 32), -h)
