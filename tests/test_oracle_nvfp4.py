"""Pins of the oracle's NVFP4 quantizer (4/6-optimal block scales and the
shared weight_scale_2) against facts fixed outside the oracle: a
hand-worked example, an exact rational restatement (oracle/micro.py),
brute force over every scale code, closed forms and invariants.

Sources: dabsLabs/Qwen3.8-Flash-Next-NVFP4, "What makes this build
different" (4/6-optimal scales; never worse than plain RTN; stacked
[512, out, in] experts unstacked into gate and up);
josch15366/Qwen3.8-Flash-Next-NVFP4-LocalHessian-Experts, introduction
(input_scale = amax/2688, not amax/6; gate and up share one
weight_scale_2)."""
from fractions import Fraction as F

import numpy as np
import pytest

from conftest import read_golden
from oracle import micro


def bits_of(f32):
    f32 = np.ascontiguousarray(f32, np.float32)
    b = f32.view(np.uint32)
    assert np.all((b & 0xFFFF) == 0), "values must be bf16-exact"
    return (b >> 16).astype(np.uint16)


def to_bf16_bits(a):
    """Round-to-nearest-even fp32 -> bf16 bits (test input preparation)."""
    a = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    r = ((a + 0x7FFF + ((a >> 16) & 1)) >> 16).astype(np.uint16)
    return r


def from_bits(b):
    return (np.asarray(b, np.uint32) << 16).view(np.float32)


def unpack_codes(codes):
    c = np.asarray(codes, np.uint8)
    out = np.empty(c.shape[:-1] + (c.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = c & 0xF
    out[..., 1::2] = c >> 4
    return out


def test_worked_example_golden(orc):
    x = np.zeros((1, 1, 48), np.float32)
    x[0, 0, 0] = 2688
    x[0, 0, 16], x[0, 0, 17] = 3, 1
    x[0, 0, 32], x[0, 0, 33] = 4, 3
    codes, scales, s2, m4 = orc.quantize_nvfp4(bits_of(x), mode=1)
    assert s2[0] == 1.0
    vals = unpack_codes(codes)[0, 0]
    for row in read_golden("nvfp4_worked.txt"):
        b, sc, M, c0, c1 = int(row[1]), int(row[3], 16), int(row[5]), int(row[7]), int(row[9])
        assert scales[0, 0, b] == sc, row
        assert m4[0, b] == (1 if M == 4 else 0), row
        assert vals[16 * b] == c0 and vals[16 * b + 1] == c1, row
        assert np.all(vals[16 * b + 2:16 * b + 16] == 0)


def test_global_scale_closed_form_and_amax_block_scale(orc):
    """s2 = RN32(amax / 2688); under plain RTN the block holding the group
    amax gets scale t = RN32(amax / RN32(6 * s2)), which rounds to E4M3 448."""
    rng = np.random.default_rng(3)
    x = to_bf16_bits(rng.normal(0, 0.02, (4, 32, 64)).astype(np.float32))
    codes, scales, s2, m4 = orc.quantize_nvfp4(x, mode=0)
    xf = from_bits(x)
    for g in range(4):
        amax = np.abs(xf[g]).max()
        assert s2[g] == np.float32(amax) / np.float32(2688)
        blk = np.abs(xf[g]).reshape(-1, 16).max(1)
        i = int(np.argmax(blk))
        assert scales[g].reshape(-1)[i] == 0x7E
    assert not m4.any()


def test_planted_input_scale_bug_is_caught(orc):
    """Negative control: the historical amax/6 global scale must fail the
    closed-form pin above (the amax block no longer reaches scale 448)."""
    rng = np.random.default_rng(3)
    x = to_bf16_bits(rng.normal(0, 0.02, (2, 32, 64)).astype(np.float32))
    _, scales, s2, _ = orc.quantize_nvfp4(x, mode=0, global_div=6.0)
    xf = from_bits(x)
    assert s2[0] != np.float32(np.abs(xf[0]).max()) / np.float32(2688)
    assert scales.max() < 0x7E


def test_gate_up_share_one_weight_scale_2(orc):
    """Fused gate_up [1, 2I, H] is one group: s2 = max(amax_gate, amax_up)/2688,
    and the codes do not depend on where gate ends and up begins."""
    rng = np.random.default_rng(5)
    I, H = 16, 64
    gate = rng.normal(0, 0.01, (I, H)).astype(np.float32)
    up = rng.normal(0, 0.03, (I, H)).astype(np.float32)
    fused = to_bf16_bits(np.concatenate([gate, up])[None])
    c, s, s2, _ = orc.quantize_nvfp4(fused, mode=1)
    xf = from_bits(fused)
    assert s2[0] == np.float32(np.abs(xf).max()) / np.float32(2688)
    # negative control: a separately scaled gate has a different s2 and codes
    cg, sg, s2g, _ = orc.quantize_nvfp4(fused[:, :I], mode=1)
    assert s2g[0] != s2[0]
    assert not np.array_equal(sg[0], s[0, :I])
    # split invariance: re-splitting the same slab at another row gives the
    # same bytes, because blocks are row-local and s2 is shared
    c2, s2b, _, _ = orc.quantize_nvfp4(fused.reshape(1, 2 * I, H), mode=1)
    assert np.array_equal(c2, c) and np.array_equal(s2b, s)


def _random_blocks(rng, n):
    """Tiny groups of one block of 16 with varied magnitude structure."""
    out = []
    for k in range(n):
        kind = k % 5
        if kind == 0:
            v = rng.normal(0, 1, 16)
        elif kind == 1:
            v = rng.normal(0, 1, 16) * np.where(rng.random(16) < 0.1, 10, 1)
        elif kind == 2:
            v = rng.uniform(-1, 1, 16) * 2.0 ** rng.integers(-20, 20)
        elif kind == 3:
            v = rng.standard_t(4, 16)
        else:
            v = np.round(rng.normal(0, 4, 16) * 2) / 2
        out.append(v * 2.0 ** rng.integers(-8, 8))
    return np.array(out, np.float32)


@pytest.mark.parametrize("group_amax_factor", [1.0, 3.0, 37.0, 1e4])
def test_blocks_match_exact_rational_micro_oracle(orc, group_amax_factor):
    """Blocks inside a group whose amax is set by an extra outlier block, so
    block scales span the E4M3 range.  Codes, scale bytes and the M choice
    must equal the exact rational restatement; the chosen error is never
    above the amax/6 plan's (never worse than plain RTN) and never below the
    best error over all 127 scale codes."""
    rng = np.random.default_rng(int(group_amax_factor * 7))
    blocks = _random_blocks(rng, 60)
    amax_blocks = np.abs(blocks).max()
    lead = np.zeros(16, np.float32)
    lead[0] = amax_blocks * group_amax_factor
    x = to_bf16_bits(np.concatenate([lead[None], blocks]).reshape(1, 1, -1))
    codes, scales, s2, m4 = orc.quantize_nvfp4(x, mode=1)
    xf = from_bits(x).reshape(-1, 16)
    assert s2[0] == micro.global_scale(np.abs(xf).max())
    vals = unpack_codes(codes).reshape(-1, 16)
    n4 = 0
    for b in range(xf.shape[0]):
        xb = [np.float32(v) for v in xf[b]]
        M, sc, c, e_ch, e6, e4 = micro.block_four_six(xb, s2[0])
        assert scales.reshape(-1)[b] == sc, b
        assert m4[0, b] == (M == 4), b
        assert list(vals[b]) == c, b
        assert e_ch <= e6
        n4 += M == 4
        if b % 6 == 0:  # brute force is slow: a sample of blocks
            assert micro.best_scale_sse(xb, s2[0]) <= e_ch
    if group_amax_factor < 100:   # tiny block scales leave no room for M=4
        assert n4 > 0


def test_ties_keep_the_amax6_plan(orc):
    """Blocks whose two plans coincide (both scales saturate at 448, or both
    round to the same scale code) must report M=6."""
    x = np.zeros((1, 1, 32), np.float32)
    x[0, 0, 0] = 2688.0            # t6 = 448, t4 = 672 -> 448: same plan
    x[0, 0, 16:32] = 0.0           # all-zero block: both plans give 0 codes
    _, scales, _, m4 = orc.quantize_nvfp4(bits_of(x), mode=1)
    assert scales[0, 0, 0] == 0x7E and m4[0, 0] == 0
    assert scales[0, 0, 1] == 0x00 and m4[0, 1] == 0


def test_rtn_mode_equals_plan6_of_four_six(orc):
    rng = np.random.default_rng(11)
    x = to_bf16_bits(rng.normal(0, 0.02, (3, 16, 128)).astype(np.float32))
    c46, s46, s2a, m4 = orc.quantize_nvfp4(x, mode=1)
    c6, s6, s2b, _ = orc.quantize_nvfp4(x, mode=0)
    assert np.array_equal(s2a, s2b)
    keep = m4.reshape(-1) == 0
    assert np.array_equal(s46.reshape(-1)[keep], s6.reshape(-1)[keep])
    assert np.array_equal(c46.reshape(-1, 8)[keep], c6.reshape(-1, 8)[keep])
    assert not np.array_equal(s46, s6)     # 4/6 changed some blocks


def test_metamorphic_scaling_sign_and_permutation(orc):
    rng = np.random.default_rng(13)
    xf = rng.normal(0, 0.02, (2, 8, 64)).astype(np.float32)
    x = to_bf16_bits(xf)
    c, s, s2, m4 = orc.quantize_nvfp4(x, mode=1)
    # x * 2^k: same codes, scales and M bits; s2 scales by exactly 2^k
    for k in (-3, 5):
        xk = bits_of(from_bits(x) * np.float32(2.0 ** k))
        ck, sk, s2k, m4k = orc.quantize_nvfp4(xk, mode=1)
        assert np.array_equal(ck, c) and np.array_equal(sk, s) and np.array_equal(m4k, m4)
        assert np.array_equal(s2k, s2 * np.float32(2.0 ** k))
    # -x: value codes flip their sign bit; scales and M bits unchanged
    cn, sn, s2n, m4n = orc.quantize_nvfp4(x ^ np.uint16(0x8000), mode=1)
    assert np.array_equal(cn, c ^ np.uint8(0x88))
    assert np.array_equal(sn, s) and np.array_equal(m4n, m4) and np.array_equal(s2n, s2)
    # permutation inside each block permutes the codes, keeps the scale
    perm = rng.permutation(16)
    xp = x.reshape(-1, 16)[:, perm].reshape(x.shape)
    cp, sp, _, m4p = orc.quantize_nvfp4(xp, mode=1)
    assert np.array_equal(sp, s) and np.array_equal(m4p, m4)
    assert np.array_equal(unpack_codes(cp).reshape(-1, 16),
                          unpack_codes(c).reshape(-1, 16)[:, perm])


def test_zero_group_and_degenerate_values(orc):
    x = np.zeros((2, 2, 32), np.uint16)
    x[1] = 0x8000                      # all -0.0
    c, s, s2, m4 = orc.quantize_nvfp4(x, mode=1)
    assert np.all(s2 == 0) and not c.any() and not s.any() and not m4.any()
    # non-finite input is rejected
    x[0, 0, 0] = 0x7F80                # +inf
    with pytest.raises(RuntimeError):
        orc.quantize_nvfp4(x, mode=1)


def test_shapes_rejected(orc):
    with pytest.raises(RuntimeError):
        orc.quantize_nvfp4(np.zeros((1, 2, 24), np.uint16))


def test_exact_decision_values_match_rational_sse(orc):
    """Direct check of the decision quantity: for blocks where the two exact
    errors differ by a hair, the oracle follows the exact comparison."""
    rng = np.random.default_rng(17)
    found = 0
    for trial in range(400):
        v = rng.normal(0, 1, 16).astype(np.float32)
        x = to_bf16_bits(np.concatenate([[8.0] + [0.0] * 15, v]).astype(np.float32).reshape(1, 1, 32))
        _, _, s2, m4 = orc.quantize_nvfp4(x, mode=1)
        xb = [np.float32(t) for t in from_bits(x).reshape(-1, 16)[1]]
        M, _, _, _, e6, e4 = micro.block_four_six(xb, s2[0])
        assert m4[0, 1] == (e4 < e6)
        if e6 != 0 and abs(F(e4 - e6) / e6) < F(1, 50):
            found += 1
    assert found > 0


def test_block_scale_divides_the_amax_once(orc):
    """Reading of the plans' order of operations: t = RN32(amax_b / RN32(M s2)),
    one rounded divisor and one division.  In the second block below (amax_b
    1.0652e-8 in a group of amax 7.2718e-6) that gives t just above an E4M3
    rounding tie, so scale code 51; the other order, RN32(RN32(amax_b / M) /
    s2), lands exactly on the tie and would give the even code 50."""
    amax_g, a = np.float32(7.271766662597656e-06), np.float32(1.0652001947164536e-08)
    xf = np.zeros((1, 1, 32), np.float32)
    xf[0, 0, 0] = amax_g
    xf[0, 0, 16] = a
    x = bits_of(xf)
    _, s, s2, _ = orc.quantize_nvfp4(x, mode=0)
    assert s2[0] == micro.global_scale(amax_g)
    block = [np.float32(v) for v in xf[0, 0, 16:]]
    sc, _, _ = micro.plan(block, s2[0], 6)
    assert s.reshape(-1)[1] == sc == 51
    other = micro.f32(micro.f32(a / micro.f32(6.0)) / s2[0])
    assert micro.e4m3_encode(other) == 50


def test_values_take_the_ieee_quotient_at_e2m1_ties(orc):
    """Reading of the value step: code = E2M1(RN32(x / d)) with the IEEE
    quotient.  With s2 = 2^-10 (group amax 2.625) the second block's scale
    is D = 1.875 and its values lie exactly on every E2M1 tie (0.25 d,
    0.75 d, ..., 5 d), each kept at the even code.  RN32(1 / 1.875) exceeds
    1 / 1.875 by 0.875 * 2^-24 of its value, so a quotient formed as
    x * RN32(1 / d) moves the ties at 1.25, 2.5 and 5 up to odd codes."""
    s2 = np.float32(2.0 ** -10)
    xf = np.zeros((1, 1, 32), np.float32)
    xf[0, 0, 0] = 2.625                                  # group amax: s2 = 2^-10
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    xf[0, 0, 16:24] = np.array([6.0] + ties, np.float32) * np.float32(1.875) * s2
    x = bits_of(xf)
    c, s, s2o, _ = orc.quantize_nvfp4(x, mode=0)
    assert s2o[0] == s2
    assert micro.e4m3_value(int(s.reshape(-1)[1])) == F(15, 8)
    block = [np.float32(v) for v in xf[0, 0, 16:]]
    want, _ = micro.plan_with_scale_code(block, s2, int(s.reshape(-1)[1]))
    got = [(int(b) >> (4 * h)) & 0xF for b in c.reshape(-1)[8:16] for h in (0, 1)]
    assert got == list(want)
    assert got[:8] == [7, 0, 2, 2, 4, 4, 6, 6]           # 6, then every tie at its even code


def test_groups_and_tensors_without_elements(orc):
    """A group with no elements has amax 0, so s2 = 0 and no block; a tensor
    with no elements has both verifier sums 0 and a relative error of 0."""
    for shape in ((3, 0, 32), (2, 8, 0), (0, 4, 16)):
        codes, scales, s2, m4 = orc.quantize_nvfp4(np.zeros(shape, np.uint16), mode=1)
        assert s2.shape == (shape[0],) and np.all(s2 == 0)
        assert codes.size == 0 and scales.size == 0 and m4.size == 0
    err, ref = orc.dequant_relerr(np.zeros((3, 0, 32), np.uint16), np.zeros(1, np.uint8),
                                     np.zeros(1, np.uint8), np.ones(3, np.float32), "nvfp4", 3, 0, 32)
    assert np.all(err == 0) and np.all(ref == 0)
    assert np.all(np.asarray(orc.relerr_from_sums(err, ref)) == 0)
