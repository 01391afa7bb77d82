"""Guard bytes around every output of the entry points other than the
single-pass quantizer (whose canaries are in test_gpu_parity.py): the MX
quantizer, activation tiles (one cluster and one grid), the quantizer with
given scales (whole and partial M-bit words), the weighted search and the
verifier write exactly their outputs, which equal those of the allocating
wrappers (themselves checked against the oracle elsewhere), and not one byte
before or after."""
import pytest
import torch

from mxfp_block_scaled_b200 import mxq, workloads

pytestmark = pytest.mark.gpu

PAD = 256                                               # bytes on each side


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mxq.load()


def guarded(n, dtype, fill):
    p = PAD // torch.empty(0, dtype=dtype).element_size()
    full = torch.full((n + 2 * p,), fill, dtype=dtype, device="cuda")
    return full, full[p:p + n], p


def intact(full, p, n, fill):
    return bool(torch.all(full[:p] == fill)) and bool(torch.all(full[p + n:] == fill))


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


@pytest.mark.parametrize("fmt", ["mxfp8", "mxfp4"])
@pytest.mark.parametrize("layout", ["linear", "swizzled_128x4"])
def test_mx_outputs_stay_inside_their_buffers(fmt, layout):
    x = workloads.activation_tile(37, seed=3, device="cuda", hidden=96)
    R, C = x.shape
    ref = mxq.quantize_mx(x, fmt, layout=layout)
    nc = R * C if fmt == "mxfp8" else R * C // 2
    ns = mxq.scale_bytes(fmt, layout, 1, R, C)
    cf, cv, cp = guarded(nc, torch.uint8, 0xA5)
    sf, sv, sp = guarded(ns, torch.uint8, 0x5A)
    st = _status()
    mxq.mxq_quantize_mx(x, R, C, fmt, 32, layout, cv, sv, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert intact(cf, cp, nc, 0xA5) and intact(sf, sp, ns, 0x5A)
    assert torch.equal(cv, ref["codes"].reshape(-1)) and torch.equal(sv, ref["scales"].reshape(-1)[:ns])


@pytest.mark.parametrize("T", [37, 1000])               # one cluster; one grid
@pytest.mark.parametrize("mode", ["rtn", "four_six"])
def test_activation_outputs_stay_inside_their_buffers(T, mode):
    H = 2048
    a = workloads.activation_tile(T, seed=T, device="cuda")
    ref = mxq.quantize_act(a, "nvfp4", mode=mode)
    nc, ns = T * H // 2, T * H // 16
    cf, cv, cp = guarded(nc, torch.uint8, 0xA5)
    sf, sv, sp = guarded(ns, torch.uint8, 0x5A)
    xf, xv, xp = guarded(1, torch.float32, -7.0)
    st = _status()
    ws, _ = mxq._workspace("quantize_act", T, H, 0, "cuda")
    mxq.mxq_quantize_act(a, T, H, "nvfp4", mode, "linear", cv, sv, xv, st, ws)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert intact(cf, cp, nc, 0xA5) and intact(sf, sp, ns, 0x5A) and intact(xf, xp, 1, -7.0)
    assert torch.equal(cv, ref["codes"].reshape(-1)) and torch.equal(sv, ref["scales"].reshape(-1))
    assert torch.equal(xv, ref["input_scale"])


@pytest.mark.parametrize("hidden", [64, 48])            # 160 and 120 blocks per group
def test_given_scale_outputs_stay_inside_their_buffers(hidden):
    x, _ = workloads.tiny_moe_layer(seed=21, experts=3, hidden=hidden, inter=20)
    x = x.cuda()
    G, R, C = x.shape
    s2, _ = mxq.global_scale_nvfp4(x)
    ref = mxq.quantize_nvfp4_s2(x, s2)
    n = G * R * C
    nw = (n // 16 + 31) // 32
    cf, cv, cp = guarded(n // 2, torch.uint8, 0xA5)
    sf, sv, sp = guarded(n // 16, torch.uint8, 0x5A)
    mf, mv, mp = guarded(nw, torch.int32, -1)
    kf, kv, kp = guarded(G, torch.int32, -1)
    st = _status()
    mxq.mxq_quantize_nvfp4_s2(x, G, R, C, s2, "four_six", "linear", cv, sv, mv, kv, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert intact(cf, cp, n // 2, 0xA5) and intact(sf, sp, n // 16, 0x5A)
    assert intact(mf, mp, nw, -1) and intact(kf, kp, G, -1)
    assert torch.equal(cv, ref["codes"].reshape(-1)) and torch.equal(sv, ref["scales"].reshape(-1))
    assert torch.equal(mv, ref["mbits"][:nw]) and torch.equal(kv, ref["m4_count"][:G])


def test_weighted_outputs_stay_inside_their_buffers():
    x, _ = workloads.tiny_moe_layer(seed=22, experts=2, hidden=64, inter=16)
    x = x.cuda()
    G, R, C = x.shape
    h = torch.rand(C, generator=torch.Generator(device="cuda").manual_seed(5), device="cuda")
    ref = mxq.quantize_nvfp4_weighted(x, h)
    n = G * R * C
    cf, cv, cp = guarded(n // 2, torch.uint8, 0xA5)
    sf, sv, sp = guarded(n // 16, torch.uint8, 0x5A)
    qf, qv, qp = guarded(G, torch.float32, -7.0)
    st = _status()
    ws, _ = mxq._workspace("quantize_nvfp4", G, R, C, "cuda")
    mxq.mxq_quantize_nvfp4_weighted(x, G, R, C, h, 1, "linear", cv, sv, qv, st, ws)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert intact(cf, cp, n // 2, 0xA5) and intact(sf, sp, n // 16, 0x5A) and intact(qf, qp, G, -7.0)
    assert torch.equal(cv, ref["codes"].reshape(-1)) and torch.equal(sv, ref["scales"].reshape(-1))
    assert torch.equal(qv, ref["s2"][:G])


def test_verifier_outputs_stay_inside_their_buffers():
    x, _ = workloads.tiny_moe_layer(seed=23, experts=4, hidden=64, inter=16)
    x = x.cuda()
    G, R, C = x.shape
    q = mxq.quantize_nvfp4(x)
    nt = 2 * G
    ref = mxq.dequant_relerr(x, q["codes"], q["scales"], q["s2"], "nvfp4", nt, R // 2, C, 2)
    outs = [guarded(nt, torch.float64, -3.0) for _ in range(3)]
    ws, _ = mxq._workspace("dequant_relerr", nt, R // 2, C, "cuda")
    mxq.mxq_dequant_relerr(x, q["codes"], q["scales"], q["s2"], "nvfp4", "linear", nt, R // 2, C, 2,
                           outs[0][1], outs[1][1], outs[2][1], ws)
    torch.cuda.synchronize()
    for (full, view, p), r in zip(outs, ref):
        assert intact(full, p, nt, -3.0)
        assert torch.equal(view, r)
