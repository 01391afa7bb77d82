"""GPU parity of three C-ABI entry points with the CPU oracle.

* mxq_quantize_nvfp4_s2, NVFP4 with a caller-given global scale per group
  (josch15366/Qwen3.8-Flash-Next-NVFP4-LocalHessian-Experts, introduction:
  gate and up share one weight_scale_2): gate and up held apart, each
  quantized with the scale they share, equal the fused-slab call byte for
  byte and the oracle; scales the caller got elsewhere (saturating,
  zero, invalid) follow the oracle or set the status word.
* mxq_global_scale_nvfp4, the global scale alone: the quantizer's bits and
  the oracle's, and with mxq_quantize_nvfp4_s2 the quantizer's outputs.
* mxq_census_add, the census of a conversion (dabsLabs/Qwen3.8-Flash-Next-
  NVFP4, metric table and "What makes this build different"): mean and max
  relative error, SSE(chosen) / SSE(RTN) - 1 and the M=4 fraction against the
  oracle's census of its own quantize + verify, within the verifier's
  tolerance (1e-6 relative on each sum); repeated sequences give identical
  bits.
"""
import numpy as np
import pytest
import torch

import oracle
from mxfp_block_scaled_b200 import layers, mxq, workloads
from test_gpu_parity import RTOL_STATS, bits, check_nvfp4, mbits_to_bytes, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from mxfp_block_scaled_b200 import build
    build.build()
    mxq.load()
    oracle.build()


def _run_s2(x_dev, s2_dev, mode="four_six", layout="linear"):
    out = mxq.quantize_nvfp4_s2(x_dev, s2_dev, mode=mode, layout=layout)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("mode", ["four_six", "rtn"])
def test_gate_and_up_apart_equal_the_fused_slab(mode):
    gu, _ = workloads.tiny_moe_layer(seed=3)
    x = gu.cuda()
    E, R, H = x.shape
    I = R // 2
    fused, _ = check_nvfp4(x, mode=mode, label="fused")
    shared = fused["s2"]                                 # RN32(max(amax_gate, amax_up) / 2688)
    gate = _run_s2(x[:, :I].contiguous(), shared, mode)
    up = _run_s2(x[:, I:].contiguous(), shared, mode)
    for o in (gate, up):
        assert int(o["status"].item()) == 0
    codes = torch.cat([gate["codes"], up["codes"]], dim=1)
    scales = torch.cat([gate["scales"], up["scales"]], dim=1)
    assert torch.equal(codes, fused["codes"]) and torch.equal(scales, fused["scales"])
    nb = I * H // 16
    m_fused = mbits_to_bytes(fused["mbits"], E * R * H // 16).reshape(E, 2 * nb)
    mg = mbits_to_bytes(gate["mbits"], E * nb).reshape(E, nb)
    mu = mbits_to_bytes(up["mbits"], E * nb).reshape(E, nb)
    assert np.array_equal(np.concatenate([mg, mu], axis=1), m_fused)
    if mode == "four_six":
        cnt = gate["m4_count"].cpu().numpy()[:E] + up["m4_count"].cpu().numpy()[:E]
        assert np.array_equal(cnt, fused["m4_count"].cpu().numpy()[:E])
    # and against the oracle's caller-given-scale function on each half
    s2 = shared.cpu().numpy()
    for half, o in ((slice(0, I), gate), (slice(I, R), up)):
        c, s, m4 = oracle.quantize_nvfp4_s2(bits(x[:, half].contiguous()), s2,
                                            mode=1 if mode == "four_six" else 0)
        assert np.array_equal(o["codes"].cpu().numpy(), c)
        assert np.array_equal(o["scales"].cpu().numpy(), s)


@pytest.mark.parametrize("shape", [(3, 5, 48), (2, 70, 256), (1, 33, 16 * 33), (4, 64, 512)])
@pytest.mark.parametrize("layout", ["linear", "swizzled_128x4"])
def test_given_scales_match_the_oracle(shape, layout):
    """Scales unrelated to the data: some far below amax / 2688 (blocks
    saturate at 448 and +-6), some far above (tiny codes), one zero."""
    G, R, C = shape
    g = torch.Generator().manual_seed(G * 1000 + R)
    x = (torch.randn(shape, generator=g) * 0.05).to(torch.bfloat16).cuda()
    amax = x.float().abs().amax(dim=(1, 2)).cpu().numpy()
    factors = np.float32([1.0, 1e-3, 50.0, 0.0, 0.37])[np.arange(G) % 5]
    s2 = (amax.astype(np.float32) / np.float32(2688.0) * factors).astype(np.float32)
    out = _run_s2(x, torch.from_numpy(s2).cuda(), layout=layout)
    assert int(out["status"].item()) == 0
    c, s, m4 = oracle.quantize_nvfp4_s2(bits(x), s2, mode=1)
    assert np.array_equal(out["codes"].cpu().numpy(), c)
    if layout == "linear":
        assert np.array_equal(out["scales"].cpu().numpy(), s)
    else:
        from oracle import layout as olay
        want = np.concatenate([olay.to_tiled_128x4(s[k]) for k in range(G)])
        assert np.array_equal(out["scales"].cpu().numpy().reshape(-1)[:want.size], want.reshape(-1))
    assert np.array_equal(mbits_to_bytes(out["mbits"], G * R * C // 16), m4.reshape(-1))


def test_invalid_scale_and_nonfinite_input_set_the_status():
    x = (torch.randn((3, 16, 64)) * 0.1).to(torch.bfloat16).cuda()
    s2 = torch.tensor([1e-4, -1.0, float("nan")], dtype=torch.float32, device="cuda")
    out = _run_s2(x, s2)
    assert int(out["status"].item()) == mxq.DEV_INVALID_SCALE
    # the valid group is still exact
    c, s, _ = oracle.quantize_nvfp4_s2(bits(x[:1].contiguous()), s2[:1].cpu().numpy(), mode=1)
    assert np.array_equal(out["codes"][:1].cpu().numpy(), c)
    xb = bits(x).copy()
    xb[1, 3, 7] = 0x7F80                                   # +Inf
    out = _run_s2(to_dev_bf16(xb), torch.full((3,), 1e-4, dtype=torch.float32, device="cuda"))
    assert int(out["status"].item()) & mxq.DEV_NONFINITE_INPUT


def _oracle_layer(gu, dn, mode):
    """The oracle's quantize + verify of a tiny layer: per stack the
    per-tensor sums and the M=4 blocks."""
    out = []
    for x, tps in ((gu, 2), (dn, 1)):
        E, R, C = x.shape
        xb = bits(x)
        c, s, s2, m4 = oracle.quantize_nvfp4(xb, mode=mode)
        err, ref = oracle.dequant_relerr(xb, c, s, s2, "nvfp4", E * tps, R // tps, C, tps)
        out.append((err, ref, int(m4.sum()), m4.size))
    return out


def test_census_of_a_layer_matches_the_oracle():
    gu, dn = workloads.tiny_moe_layer(seed=0)
    g, d = gu.cuda(), dn.cuda()
    res46 = layers.quantize_routed_layer(g, d, mode="four_six")
    resrtn = layers.quantize_routed_layer(g, d, mode="rtn")
    got = layers.census([res46], [resrtn])
    o46, ortn = _oracle_layer(gu, dn, 1), _oracle_layer(gu, dn, 0)
    want = oracle.census(np.concatenate([o[0] for o in o46]), np.concatenate([o[1] for o in o46]),
                         err_rtn=np.concatenate([o[0] for o in ortn]),
                         m4_blocks=sum(o[2] for o in o46), blocks=sum(o[3] for o in o46))
    assert got["n_tensors"] == want["n_tensors"] == 3 * 8
    assert got["n_tensors_rtn"] == got["n_tensors"]
    for k in ("mean_relerr", "max_relerr", "sum_sq_err", "sum_sq_ref"):
        assert got[k] == pytest.approx(want[k], rel=RTOL_STATS, abs=0), k
    # each error total within 11 * 2^-24 of the exact one: 1 + ratio within 2e-6
    assert abs((1.0 + got["sse_vs_rtn"]) - (1.0 + want["sse_vs_rtn"])) <= 2e-6 * (1.0 + want["sse_vs_rtn"])
    assert got["sse_vs_rtn"] < 0.0
    assert got["blocks"] == sum(o[3] for o in o46)
    assert got["blocks_m4"] == sum(o[2] for o in o46)
    assert got["m4_fraction"] == want["m4_fraction"]


def test_census_is_deterministic_and_accumulates_in_call_order():
    gu, dn = workloads.tiny_moe_layer(seed=2)
    res = layers.quantize_routed_layer(gu.cuda(), dn.cuda(), mode="four_six")
    mx = layers.quantize_routed_layer(gu.cuda(), dn.cuda(), fmt="mxfp8")
    a = layers.census([res, mx])
    b = layers.census([res, mx])
    for k in a:                                          # identical bits, every field
        assert np.float64(a[k]).tobytes() == np.float64(b[k]).tobytes() or a[k] == b[k], k
    one = layers.census([res])
    assert a["n_tensors"] == 2 * one["n_tensors"]
    assert a["blocks"] == one["blocks"] and a["blocks_m4"] == one["blocks_m4"]   # MX adds no blocks
    assert a["max_relerr"] == max(one["max_relerr"], layers.census([mx])["max_relerr"])
    assert np.isnan(a["sse_vs_rtn"])                     # no RTN counterparts were given


@pytest.mark.parametrize("shape", [(8, 256, 256), (3, 5, 48), (2, 70, 256)])
def test_global_scale_alone_matches_the_quantizer_and_the_oracle(shape):
    """mxq_global_scale_nvfp4 (steps a1-a2 alone) writes the bits
    mxq_quantize_nvfp4 writes, and RN32(amax_g / 2688) of the oracle; with
    mxq_quantize_nvfp4_s2 it reproduces mxq_quantize_nvfp4 byte for byte."""
    G, R, C = shape
    g = torch.Generator().manual_seed(G * 31 + R)
    x = (torch.randn(shape, generator=g) * 0.05).to(torch.bfloat16).cuda()
    s2, st = mxq.global_scale_nvfp4(x)
    full = mxq.quantize_nvfp4(x, mode="four_six")
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    _, _, os2, _ = oracle.quantize_nvfp4(bits(x), mode=1)
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), os2.view(np.uint32))
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), full["s2"].cpu().numpy().view(np.uint32))
    two = _run_s2(x, s2)
    assert torch.equal(two["codes"], full["codes"]) and torch.equal(two["scales"], full["scales"])
    # gate and up held apart: the larger of the halves' scales is the shared one
    sg, _ = mxq.global_scale_nvfp4(x[:, :R // 2].contiguous()) if R % 2 == 0 else (s2, None)
    su, _ = mxq.global_scale_nvfp4(x[:, R // 2:].contiguous()) if R % 2 == 0 else (s2, None)
    assert torch.equal(torch.maximum(sg, su), s2)


def test_global_scale_reports_nonfinite_input():
    x = (torch.randn((2, 16, 64)) * 0.1).to(torch.bfloat16)
    xb = bits(x).copy()
    xb[1, 2, 3] = 0x7FC0                                   # NaN
    _, st = mxq.global_scale_nvfp4(to_dev_bf16(xb))
    torch.cuda.synchronize()
    assert int(st.item()) & mxq.DEV_NONFINITE_INPUT
