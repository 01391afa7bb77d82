"""The 128 x 4 tiled scale layout written by the CUDA kernels, the verifier
reading it, and 4/6-optimal block scales for activation tiles, each against
the CPU oracle on the same seeded inputs (bit-exact on codes, scales, s2 and
M bits; verifier sums within 1e-6 relative).  One more check needs no
oracle: a block-scaled tensor-core GEMM (cuBLAS through torch._scaled_mm)
fed our codes and tiled scales must reproduce the product of the
dequantized matrices; a wrong tile layout scrambles the scales it applies."""
import numpy as np
import pytest
import torch

import oracle
from oracle import layout
from mxfp_block_scaled_b200 import mxq, workloads

pytestmark = pytest.mark.gpu

SWZ = "swizzled_128x4"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from mxfp_block_scaled_b200 import build
    build.build()
    mxq.load()
    oracle.build()


def _rand_bf16(shape, seed, std=0.05):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16).cuda()


def _tiled_groups(scales_linear, G, rows, cb):
    s = np.asarray(scales_linear, dtype=np.uint8).reshape(G, rows, cb)
    return np.concatenate([layout.to_tiled_128x4(s[g]) for g in range(G)])


# single pass (blocks per group a multiple of 32) and two-pass shapes, with
# and without row / column padding of the scale matrices
NVFP4_SHAPES = [(2, 130, 256), (2, 256, 80), (1, 256, 2048), (3, 130, 80), (1, 40, 48), (4, 5, 16)]


@pytest.mark.parametrize("shape", NVFP4_SHAPES)
@pytest.mark.parametrize("mode", ["four_six", "rtn"])
def test_nvfp4_tiled_scales_bit_exact(shape, mode):
    G, R, C = shape
    x = _rand_bf16(shape, seed=G * 7 + R + C)
    out = mxq.quantize_nvfp4(x, mode=mode, layout=SWZ)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    c, s, s2, m4 = oracle.quantize_nvfp4(workloads.bf16_bits(x).reshape(G, R, C),
                                         mode=1 if mode == "four_six" else 0)
    assert np.array_equal(out["codes"].cpu().numpy().reshape(-1), c.reshape(-1))
    assert np.array_equal(out["s2"].cpu().numpy().view(np.uint32), s2.view(np.uint32))
    got = out["scales"].cpu().numpy()
    want = _tiled_groups(s, G, R, C // 16)
    assert got.size == want.size == mxq.scale_bytes("nvfp4", SWZ, G, R, C)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, "tiled scales differ at bytes %s" % bad[:10]
    mb = np.unpackbits(out["mbits"].cpu().numpy().view(np.uint8), bitorder="little")[:G * R * C // 16]
    assert np.array_equal(mb, m4.reshape(-1))


@pytest.mark.parametrize("fmt", ["mxfp8", "mxfp4"])
@pytest.mark.parametrize("shape", [(130, 160), (256, 2048), (7, 32)])
def test_mx_tiled_scales_bit_exact(fmt, shape):
    R, C = shape
    x = _rand_bf16(shape, seed=R + C + (fmt == "mxfp4"))
    out = mxq.quantize_mx(x, fmt, layout=SWZ)
    torch.cuda.synchronize()
    c, s = oracle.quantize_mx(workloads.bf16_bits(x).reshape(R, C), fmt)
    assert np.array_equal(out["codes"].cpu().numpy().reshape(-1), c.reshape(-1))
    got = out["scales"].cpu().numpy()
    want = layout.to_tiled_128x4(s.reshape(R, C // 32))
    assert np.array_equal(got, want)


@pytest.mark.parametrize("inter", [128, 96])
def test_verifier_reads_tiled_scales(inter):
    """Fused gate_up [E, 2I, H] unstacked into 2E tensors of [I, H]: two
    consecutive tensors share one s2 and one tiled scale matrix (for I = 96
    the matrix boundary falls inside a row tile, so the tensor rows must be
    offset inside it)."""
    E, H = 3, 256
    gu = _rand_bf16((E, 2 * inter, H), seed=inter)
    lin = mxq.quantize_nvfp4(gu)
    swz = mxq.quantize_nvfp4(gu, layout=SWZ)
    a = mxq.dequant_relerr(gu, lin["codes"], lin["scales"], lin["s2"], "nvfp4", 2 * E, inter, H, 2)
    b = mxq.dequant_relerr(gu, swz["codes"], swz["scales"], swz["s2"], "nvfp4", 2 * E, inter, H, 2,
                           layout=SWZ)
    torch.cuda.synchronize()
    for u, v in zip(a, b):
        assert torch.equal(u, v)
    oe, orf = oracle.dequant_relerr(workloads.bf16_bits(gu), lin["codes"].cpu().numpy(),
                                    lin["scales"].cpu().numpy(), lin["s2"].cpu().numpy(), "nvfp4",
                                    2 * E, inter, H, 2)
    np.testing.assert_allclose(b[0].cpu().numpy(), oe, rtol=1e-6, atol=0)
    np.testing.assert_allclose(b[1].cpu().numpy(), orf, rtol=1e-6, atol=0)
    # MX: the stack quantized as one matrix is one scale matrix of n tensors
    x = _rand_bf16((4, 96, 64), seed=5)
    q = mxq.quantize_mx(x.view(4 * 96, 64), "mxfp8", layout=SWZ)
    ql = mxq.quantize_mx(x.view(4 * 96, 64), "mxfp8")
    e1 = mxq.dequant_relerr(x, ql["codes"], ql["scales"], None, "mxfp8", 4, 96, 64)
    e2 = mxq.dequant_relerr(x, q["codes"], q["scales"], None, "mxfp8", 4, 96, 64, 4, layout=SWZ)
    torch.cuda.synchronize()
    for u, v in zip(e1, e2):
        assert torch.equal(u, v)


@pytest.mark.parametrize("T", [1, 16, 256, 4096])
def test_activation_four_six_bit_exact(T):
    a = workloads.activation_tile(T, seed=T).cuda()
    o = mxq.quantize_act(a, "nvfp4", mode="four_six")
    torch.cuda.synchronize()
    assert int(o["status"].item()) == 0
    c, s, s2, m4 = oracle.quantize_nvfp4(workloads.bf16_bits(a).reshape(1, T, -1), mode=1)
    assert np.array_equal(o["codes"].cpu().numpy().reshape(-1), c.reshape(-1))
    assert np.array_equal(o["scales"].cpu().numpy().reshape(-1), s.reshape(-1))
    assert o["input_scale"].cpu().numpy().view(np.uint32)[0] == s2.view(np.uint32)[0]
    # blocks that kept M = 6 are byte-identical to plain amax/6 (RTN) mode
    r = mxq.quantize_act(a, "nvfp4")
    torch.cuda.synchronize()
    keep6 = m4.reshape(-1) == 0
    rc, oc = r["codes"].cpu().numpy().reshape(-1, 8), o["codes"].cpu().numpy().reshape(-1, 8)
    rs, os_ = r["scales"].cpu().numpy().reshape(-1), o["scales"].cpu().numpy().reshape(-1)
    assert np.array_equal(rc[keep6], oc[keep6]) and np.array_equal(rs[keep6], os_[keep6])
    if T >= 16:
        assert 0.1 < m4.mean() < 0.9


def test_activation_tiled_layout():
    T = 300
    a = workloads.activation_tile(T, seed=3).cuda()
    for fmt in ("nvfp4", "mxfp8"):
        lin = mxq.quantize_act(a, fmt)
        swz = mxq.quantize_act(a, fmt, layout=SWZ)
        torch.cuda.synchronize()
        assert torch.equal(lin["codes"], swz["codes"])
        blk = 16 if fmt == "nvfp4" else 32
        want = layout.to_tiled_128x4(lin["scales"].cpu().numpy().reshape(T, 2048 // blk))
        assert np.array_equal(swz["scales"].cpu().numpy(), want)


# -------------------------------------------- tiled scales in a real GEMM --
def _scaled_mm_or_skip(*args, **kw):
    try:
        return torch._scaled_mm(*args, **kw)
    except (RuntimeError, TypeError, NotImplementedError) as e:
        pytest.skip("torch._scaled_mm does not take this block-scaled form here: %s" % str(e)[:200])


def test_tiled_mxfp8_scales_drive_a_block_scaled_gemm():
    M, N, K = 256, 256, 512
    a = _rand_bf16((M, K), seed=11, std=1.0)
    b = _rand_bf16((N, K), seed=12, std=1.0)
    qa, qb = mxq.quantize_mx(a, "mxfp8", layout=SWZ), mxq.quantize_mx(b, "mxfp8", layout=SWZ)
    la, lb = mxq.quantize_mx(a, "mxfp8"), mxq.quantize_mx(b, "mxfp8")
    torch.cuda.synchronize()

    def deq(q):
        v = q["codes"].view(torch.float8_e4m3fn).float()
        e = q["scales"].float() - 127.0
        return v * torch.exp2(e).repeat_interleave(32, dim=1)

    ref = deq(la).double() @ deq(lb).double().t()
    out = _scaled_mm_or_skip(qa["codes"].view(torch.float8_e4m3fn), qb["codes"].view(torch.float8_e4m3fn).t(),
                             qa["scales"].view(torch.float8_e8m0fnu), qb["scales"].view(torch.float8_e8m0fnu),
                             out_dtype=torch.bfloat16)
    err = (out.double() - ref).abs().max().item()
    assert err <= 0.02 * ref.abs().max().item(), err
    # the same GEMM fed the linear (untiled) scales is visibly wrong
    bad = _scaled_mm_or_skip(qa["codes"].view(torch.float8_e4m3fn), qb["codes"].view(torch.float8_e4m3fn).t(),
                             la["scales"].reshape(-1).view(torch.float8_e8m0fnu),
                             lb["scales"].reshape(-1).view(torch.float8_e8m0fnu), out_dtype=torch.bfloat16)
    assert (bad.double() - ref).abs().max().item() > 10 * max(err, 1e-3)


def test_tiled_nvfp4_scales_drive_a_block_scaled_gemm():
    """NVFP4 operands (E2M1 pairs, E4M3 scale per 16 in the tiled layout) in a
    block-scaled FP4 GEMM; the global scales are applied outside it."""
    if not hasattr(torch, "float4_e2m1fn_x2"):
        pytest.skip("this torch has no packed FP4 dtype")
    M, N, K = 256, 256, 512
    a = _rand_bf16((1, M, K), seed=21, std=1.0)
    b = _rand_bf16((1, N, K), seed=22, std=1.0)
    qa, qb = mxq.quantize_nvfp4(a, layout=SWZ), mxq.quantize_nvfp4(b, layout=SWZ)
    la, lb = mxq.quantize_nvfp4(a), mxq.quantize_nvfp4(b)
    torch.cuda.synchronize()
    e2m1 = torch.tensor([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6],
                        dtype=torch.float64, device="cuda")

    def qd(q, rows):     # q * D (the global scale left out), [rows, K]
        c = q["codes"].reshape(rows, K // 2).long()
        v = torch.stack([e2m1[c & 15], e2m1[c >> 4]], dim=-1).reshape(rows, K)
        d = q["scales"].reshape(rows, K // 16).view(torch.float8_e4m3fn).double()
        return v * d.repeat_interleave(16, dim=1)

    ref = qd(la, M) @ qd(lb, N).t()
    fp4 = torch.float4_e2m1fn_x2
    out = _scaled_mm_or_skip(qa["codes"].reshape(M, K // 2).view(fp4), qb["codes"].reshape(N, K // 2).view(fp4).t(),
                             qa["scales"].view(torch.float8_e4m3fn), qb["scales"].view(torch.float8_e4m3fn),
                             out_dtype=torch.bfloat16)
    err = (out.double() - ref).abs().max().item()
    assert err <= 0.02 * ref.abs().max().item(), err
