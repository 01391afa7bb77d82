"""Parity of the CUDA path (through the C ABI) with the CPU oracle on the
same seeded inputs.  Bit-exact on codes, scale bytes, global scales and the
per-block M choice; verifier sums within 1e-6 relative."""
import numpy as np
import pytest
import torch

import oracle
from mxfp_block_scaled_b200 import layers, mxq, workloads

pytestmark = pytest.mark.gpu

RTOL_STATS = 1e-6


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from mxfp_block_scaled_b200 import build
    build.build()
    mxq.load()
    oracle.build()


def bits(t):
    return workloads.bf16_bits(t)


def from_bits_np(b):
    return (np.asarray(b, np.uint32) << 16).view(np.float32)


def to_dev_bf16(bits_np):
    return torch.from_numpy(np.ascontiguousarray(bits_np).view(np.int16)).cuda().view(torch.bfloat16)


def mbits_to_bytes(words, n_blocks):
    w = words.cpu().numpy().view(np.uint32)
    b = np.unpackbits(w.view(np.uint8), bitorder="little")
    return b[:n_blocks]


def check_nvfp4(x_dev, mode="four_six", label=""):
    G, R, C = x_dev.shape
    out = mxq.quantize_nvfp4(x_dev, mode=mode)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    xb = bits(x_dev).reshape(G, R, C)
    c, s, s2, m4 = oracle.quantize_nvfp4(xb, mode=1 if mode == "four_six" else 0)
    gc = out["codes"].cpu().numpy()
    gs = out["scales"].cpu().numpy()
    gs2 = out["s2"].cpu().numpy()
    assert np.array_equal(gs2.view(np.uint32), s2.view(np.uint32)), label + " s2"
    bad = np.nonzero(gs.reshape(-1) != s.reshape(-1))[0]
    assert bad.size == 0, "%s scales differ at blocks %s" % (label, bad[:10])
    badc = np.nonzero((gc.reshape(-1, 8) != c.reshape(-1, 8)).any(1))[0]
    assert badc.size == 0, "%s codes differ at blocks %s" % (label, badc[:10])
    gm = mbits_to_bytes(out["mbits"], G * R * C // 16)
    assert np.array_equal(gm, m4.reshape(-1)), label + " M bits"
    cnt = out["m4_count"].cpu().numpy()[:G]
    if mode == "four_six":
        assert np.array_equal(cnt, m4.reshape(G, -1).sum(1)), label + " m4 count"
    return out, (c, s, s2, m4)


def check_verify(x_dev, codes, scales, s2, fmt, n_tensors, rows, cols, tps=1):
    err, ref, rel = mxq.dequant_relerr(x_dev, codes, scales, s2, fmt, n_tensors, rows, cols, tps)
    torch.cuda.synchronize()
    oe, orf = oracle.dequant_relerr(bits(x_dev), codes.cpu().numpy(), scales.cpu().numpy(),
                                    None if s2 is None else s2.cpu().numpy(), fmt, n_tensors,
                                    rows, cols, tps)
    err, ref, rel = err.cpu().numpy(), ref.cpu().numpy(), rel.cpu().numpy()
    np.testing.assert_allclose(err, oe, rtol=RTOL_STATS, atol=0)
    np.testing.assert_allclose(ref, orf, rtol=RTOL_STATS, atol=0)
    np.testing.assert_allclose(rel, oracle.relerr_from_sums(oe, orf), rtol=RTOL_STATS, atol=0)
    return err, ref, rel


# ---------------------------------------------------------------- NVFP4 --
def test_tiny_moe_layer_four_six_bit_exact_and_verified():
    gu, dn = workloads.tiny_moe_layer(seed=0)
    gu, dn = gu.cuda(), dn.cuda()
    o1, _ = check_nvfp4(gu, label="gate_up")
    o2, (_, _, _, m4) = check_nvfp4(dn, label="down")
    E, R, H = gu.shape
    check_verify(gu, o1["codes"], o1["scales"], o1["s2"], "nvfp4", 2 * E, R // 2, H, tps=2)
    check_verify(dn, o2["codes"], o2["scales"], o2["s2"], "nvfp4", E, dn.shape[1], dn.shape[2])
    assert 0.2 < m4.mean() < 0.7


def test_sse_against_rtn_and_m4_fraction_of_a_layer():
    """The layer figures the pages report beside the relative error:
    SSE(chosen) / SSE(RTN) - 1 (never above 0) and the M=4 fraction, from
    the GPU path against the oracle's own quantize + verify in both modes
    (each error sum within 11 * 2^-24 of the exact one, so 1 + ratio within
    2e-6)."""
    gu, dn = workloads.tiny_moe_layer(seed=0)
    g, d = gu.cuda(), dn.cuda()
    res46 = layers.quantize_routed_layer(g, d, mode="four_six")
    resrtn = layers.quantize_routed_layer(g, d, mode="rtn")
    torch.cuda.synchronize()
    ratio = layers.sse_vs_rtn([res46], [resrtn])
    frac = layers.m4_fraction([res46])
    tot = {0: 0.0, 1: 0.0}
    m4s = blocks = 0
    for x, tps in ((gu, 2), (dn, 1)):
        E, R, C = x.shape
        xb = bits(x)
        for mode in (0, 1):
            c, s, s2, m4 = oracle.quantize_nvfp4(xb, mode=mode)
            oe, _ = oracle.dequant_relerr(xb, c, s, s2, "nvfp4", E * tps, R // tps, C, tps)
            tot[mode] += float(oe.sum())
            if mode == 1:
                m4s += int(m4.sum())
                blocks += m4.size
    want = tot[1] / tot[0] - 1.0
    assert ratio <= 0.0 and want <= 0.0
    assert abs((1.0 + ratio) - (1.0 + want)) <= 2e-6 * (1.0 + want)
    assert frac == m4s / blocks


def test_tiny_moe_layer_rtn():
    gu, _ = workloads.tiny_moe_layer(seed=1)
    check_nvfp4(gu.cuda(), mode="rtn", label="rtn")


@pytest.mark.parametrize("shape", [(3, 5, 48), (1, 1, 16), (2, 70, 256), (5, 3, 32 * 16),
                                   (1, 33, 16 * 33), (7, 64, 64)])
def test_ragged_shapes(shape):
    g = torch.Generator().manual_seed(sum(shape))
    x = (torch.randn(shape, generator=g) * 0.05).to(torch.bfloat16).cuda()
    out, _ = check_nvfp4(x, label=str(shape))
    G, R, C = shape
    check_verify(x, out["codes"], out["scales"], out["s2"], "nvfp4", G, R, C)


def test_degenerate_values():
    G, R, C = 6, 4, 64
    g = torch.Generator().manual_seed(7)
    x = torch.randn((G, R, C), generator=g) * 0.02
    x[0] = 0.0                                     # all-zero group: s2 = 0
    x[1] = -0.0                                    # negative zeros
    x[2] = x[2] * 1e-36                            # tiny: subnormal s2, slow path
    x[3, 0, 0] = 3.0e38                            # huge: s2 outside the fast range
    x[4, :, :16] = 0.0                             # zero blocks inside a normal group
    x[4, 1, 16:32] = 1e-40                         # subnormal bf16 values
    x[5] = torch.round(x[5] * 1000) / 1000         # many exact ties
    x = x.to(torch.bfloat16)
    xb = bits(x)
    xb[1] = 0x8000
    check_nvfp4(to_dev_bf16(xb), label="degenerate")
    check_nvfp4(to_dev_bf16(xb), mode="rtn", label="degenerate rtn")


def _tie_rich_blocks(seed, nblocks):
    """Blocks on grids both plans represent exactly (so the exact 4/6
    decision meets ties G4 == G6 with different scale codes), blocks that
    add an element both plans round to zero (equal non-zero errors), blocks
    exact in the M=4 plan only, and plain random blocks; the first element
    sets the group amax to 2.625, so s2 = 2^-10 exactly."""
    from oracle import micro
    rng = np.random.default_rng(seed)
    s2 = 2.0 ** -10
    scales = [v for v in micro.E4M3_LIST[1:127] if 1.5 * v in micro.E4M3_LIST and 1.5 * v <= 448]
    x = np.zeros((nblocks, 16), np.float32)
    for b in range(nblocks):
        base = np.float32(scales[rng.integers(len(scales))] * s2)
        v = rng.choice([0.0, 1.5, 3.0, 6.0, -1.5, -3.0, -6.0], 16) * base
        v[rng.integers(16)] = 6.0 * base * rng.choice([1, -1])
        if b % 4 == 1:
            v[rng.integers(16)] = base * 2.0 ** -6
        elif b % 4 == 2:
            v = rng.standard_normal(16) * 0.3
        elif b % 4 == 3:
            v[rng.integers(16)] = base * 0.75
        x[b] = v
    x[0] = 0.0
    x[0, 0] = 2.625
    return x


@pytest.mark.parametrize("shape", [(2, 4, 256), (3, 1, 16 * 33)])
def test_exact_decision_at_ties(shape):
    """Ties and near-ties of the two plans' exact errors leave the fp32
    filter undecided and must fall back to the exact decision (M=6 on a
    tie), bit-exact with the oracle on both schedules (single pass: blocks
    per group a multiple of 32; two-pass otherwise)."""
    G, R, C = shape
    nb = R * C // 16
    x = np.stack([_tie_rich_blocks(100 + g, nb).reshape(R, C) for g in range(G)])
    xt = torch.from_numpy(x).to(torch.bfloat16)
    out, (_, _, s2, m4) = check_nvfp4(xt.cuda(), label="ties %s" % (shape,))
    assert np.all(s2 == np.float32(2.0 ** -10))
    assert 0 < m4.sum() < m4.size


@pytest.mark.parametrize("mode", ["rtn", "four_six"])
@pytest.mark.parametrize("G,R", [(1, 1), (8, 32)])
def test_values_on_every_e2m1_tie(G, R, mode):
    """Blocks whose values lie exactly on every E2M1 tie under a block scale
    whose reciprocal is not a binary32 value (D = 1.875 with s2 = 2^-10):
    the quotients must be the correctly rounded ones, so every tie keeps its
    even code.  One group (the cluster kernel) and eight groups of 512
    blocks (the single pass)."""
    s2 = np.float32(2.0 ** -10)
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    vals = np.array([6.0] + ties + [-t for t in ties] + [0.0], np.float32) * np.float32(1.875) * s2
    row = np.zeros(256, np.float32)
    row[0] = 2.625                                       # group amax: s2 = 2^-10
    for b in range(1, 16):
        row[16 * b:16 * b + 16] = np.roll(vals, b)
    x = torch.from_numpy(np.tile(row, (G, R, 1))).to(torch.bfloat16)
    _, (_, s, s2o, _) = check_nvfp4(x.cuda(), mode=mode, label="e2m1 ties")
    assert np.all(s2o == s2)


def test_nonfinite_input_sets_status():
    x = torch.randn((2, 4, 32)).to(torch.bfloat16).cuda()
    x[1, 2, 5] = float("inf")
    out = mxq.quantize_nvfp4(x)
    torch.cuda.synchronize()
    assert int(out["status"].item()) & mxq.DEV_NONFINITE_INPUT
    x[1, 2, 5] = float("nan")
    o2 = mxq.quantize_mx(x.view(8, 32), "mxfp8")
    torch.cuda.synchronize()
    assert int(o2["status"].item()) & mxq.DEV_NONFINITE_INPUT


def test_deterministic_and_canaries():
    gu, _ = workloads.tiny_moe_layer(seed=2)
    gu = gu.cuda()
    G, R, C = gu.shape
    n = G * R * C
    pad = 256
    codes = torch.full((n // 2 + 2 * pad,), 0xA5, dtype=torch.uint8, device="cuda")
    scales = torch.full((n // 16 + 2 * pad,), 0x5A, dtype=torch.uint8, device="cuda")
    s2 = torch.full((G + 64,), -7.0, dtype=torch.float32, device="cuda")
    mb = torch.full(((n // 16) // 32 + 64,), -1, dtype=torch.int32, device="cuda")
    m4 = torch.full((G + 64,), -1, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws, _ = mxq._workspace("quantize_nvfp4", G, R, C, "cuda")
    results = []
    for _ in range(2):
        mxq.mxq_quantize_nvfp4(gu, G, R, C, "four_six", "linear", codes[pad:pad + n // 2],
                               scales[pad:pad + n // 16], s2[:G], mb[:(n // 16) // 32], m4[:G], st, ws)
        torch.cuda.synchronize()
        results.append((codes.clone(), scales.clone(), s2.clone(), mb.clone()))
    for a, b in zip(results[0], results[1]):
        assert torch.equal(a, b)
    assert torch.all(codes[:pad] == 0xA5) and torch.all(codes[pad + n // 2:] == 0xA5)
    assert torch.all(scales[:pad] == 0x5A) and torch.all(scales[pad + n // 16:] == 0x5A)
    assert torch.all(s2[G:] == -7.0) and torch.all(mb[(n // 16) // 32:] == -1) and torch.all(m4[G:] == -1)
    # verifier: bit-identical across runs
    e1 = mxq.dequant_relerr(gu, codes[pad:pad + n // 2], scales[pad:pad + n // 16], s2[:G], "nvfp4",
                            2 * G, R // 2, C, 2)
    e2 = mxq.dequant_relerr(gu, codes[pad:pad + n // 2], scales[pad:pad + n // 16], s2[:G], "nvfp4",
                            2 * G, R // 2, C, 2)
    for a, b in zip(e1, e2):
        assert torch.equal(a, b)


@pytest.mark.parametrize("shape", [(4, 64, 512), (3, 96, 16 * 64)])
def test_m4_count_with_and_without_m_bits(shape):
    """The M=4 count per group is the same whether the M bits are stored
    (counted from them after the quantizer) or not (counted inside it), and
    equals the oracle's."""
    G, R, C = shape
    x, _ = workloads.tiny_moe_layer(seed=11, experts=G, hidden=C, inter=R // 2)
    x = x.cuda()
    a = mxq.quantize_nvfp4(x, with_mbits=True)
    b = mxq.quantize_nvfp4(x, with_mbits=False)
    torch.cuda.synchronize()
    assert int(a["status"].item()) == 0 and int(b["status"].item()) == 0
    assert torch.equal(a["codes"], b["codes"]) and torch.equal(a["scales"], b["scales"])
    _, _, _, m4 = oracle.quantize_nvfp4(bits(x).reshape(G, R, C), mode=1)
    want = m4.reshape(G, -1).sum(1)
    assert np.array_equal(a["m4_count"].cpu().numpy()[:G], want)
    assert np.array_equal(b["m4_count"].cpu().numpy()[:G], want)
    assert np.array_equal(mbits_to_bytes(a["mbits"], G * R * C // 16), m4.reshape(-1))


# ------------------------------------------------------------------- MX --
@pytest.mark.parametrize("fmt", ["mxfp8", "mxfp4"])
def test_shared_expert_mx_bit_exact_dense_and_padded(fmt):
    for padded in (False, True):
        gu, dn = workloads.shared_expert_layer(seed=4, inter=320, hidden=512, pad_from=160,
                                               padded=padded)
        for t in (gu, dn):
            td = t.cuda()
            out = mxq.quantize_mx(td, fmt)
            torch.cuda.synchronize()
            c, s = oracle.quantize_mx(bits(td), fmt)
            assert np.array_equal(out["codes"].cpu().numpy(), c)
            assert np.array_equal(out["scales"].cpu().numpy(), s)
            check_verify(td, out["codes"], out["scales"], None, fmt, 1, *td.shape)
        if padded:
            o = mxq.quantize_mx(gu.cuda(), fmt)
            assert not o["codes"][160:320].any() and not o["scales"][160:320].any()


def _all_bf16_in(lo, hi):
    b = np.arange(0, 0x7F80, dtype=np.uint32)
    f = (b << 16).view(np.float32)
    sel = (f >= lo) & (f <= hi)
    return b[sel].astype(np.uint16)


@pytest.mark.parametrize("fmt,qmax", [("mxfp8", 448.0), ("mxfp4", 6.0)])
def test_every_bf16_value_converts_like_the_oracle(fmt, qmax):
    """Blocks whose first element is qmax (so e = 0) carry every bf16 value
    in [0, qmax] and its negative: the hardware conversion of every such
    input equals the oracle's nearest-even rounding."""
    vals = _all_bf16_in(0.0, qmax)
    vals = np.concatenate([vals, vals | 0x8000])
    per = 31
    nblk = -(-vals.size // per)
    x = np.zeros((nblk, 32), np.uint16)
    qbits = np.float32(qmax).view(np.uint32) >> 16
    x[:, 0] = qbits
    flat = x[:, 1:].reshape(-1)
    flat[:vals.size] = vals
    x[:, 1:] = flat.reshape(nblk, per)
    xd = to_dev_bf16(x)
    out = mxq.quantize_mx(xd, fmt)
    torch.cuda.synchronize()
    c, s = oracle.quantize_mx(x, fmt)
    assert np.all(s == 127)
    assert np.array_equal(out["scales"].cpu().numpy(), s)
    assert np.array_equal(out["codes"].cpu().numpy(), c)


@pytest.mark.parametrize("fmt", ["mxfp8", "mxfp4"])
def test_every_bf16_amax_gives_the_exponent_rule(fmt):
    """One block per positive finite bf16 value (and the subnormals): block
    amax = that value; scale bytes equal the oracle's for all of them."""
    vals = np.arange(1, 0x7F80, dtype=np.uint16)
    x = np.zeros((vals.size, 32), np.uint16)
    x[:, 3] = vals
    x[:, 7] = vals | 0x8000
    xd = to_dev_bf16(x)
    out = mxq.quantize_mx(xd, fmt)
    torch.cuda.synchronize()
    c, s = oracle.quantize_mx(x, fmt)
    assert np.array_equal(out["scales"].cpu().numpy(), s)
    assert np.array_equal(out["codes"].cpu().numpy(), c)


# ---------------------------------------------------------- activations --
@pytest.mark.parametrize("T", [1, 16, 256])
def test_activation_tiles(T):
    a = workloads.activation_tile(T, seed=T).cuda()
    o = mxq.quantize_act(a, "nvfp4")
    torch.cuda.synchronize()
    assert int(o["status"].item()) == 0
    c, s, s2, _ = oracle.quantize_nvfp4(bits(a).reshape(1, T, -1), mode=0)
    assert o["input_scale"].cpu().numpy().view(np.uint32)[0] == s2.view(np.uint32)[0]
    assert np.array_equal(o["codes"].cpu().numpy(), c.reshape(T, -1))
    assert np.array_equal(o["scales"].cpu().numpy(), s.reshape(T, -1))
    for fmt in ("mxfp8", "mxfp4"):
        o = mxq.quantize_act(a, fmt)
        torch.cuda.synchronize()
        c, s = oracle.quantize_mx(bits(a), fmt)
        assert np.array_equal(o["codes"].cpu().numpy(), c)
        assert np.array_equal(o["scales"].cpu().numpy(), s)


def test_activation_input_scale_is_amax_over_2688_not_amax_over_6():
    a = workloads.activation_tile(16, seed=3).cuda()
    o = mxq.quantize_act(a, "nvfp4")
    amax = a.float().abs().max().item()
    got = float(o["input_scale"].item())
    assert got == float(np.float32(amax) / np.float32(2688.0))
    assert abs(got - amax / 6) > 0.1 * amax / 6
