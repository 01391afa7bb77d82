"""FP8 -> MX requantization on the GPU (mxq_requant_fp8_mx, through the C
ABI) against the CPU oracle on the same seeded block-FP8 sources:
bit-exact codes and scale bytes, linear and tiled scale layouts, source
blocks that do and do not align with the tensor edges."""
import numpy as np
import pytest
import torch

import oracle
from oracle import layout
from mxfp_block_scaled_b200 import mxq, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from mxfp_block_scaled_b200 import build
    build.build()
    mxq.load()
    oracle.build()


@pytest.mark.parametrize("fmt", ["mxfp8", "mxfp4"])
@pytest.mark.parametrize("rows,cols,brows,bcols", [(256, 512, 128, 128), (200, 384, 128, 128),
                                                   (96, 256, 32, 64), (1, 32, 128, 128),
                                                   (1536, 2048, 128, 128)])
@pytest.mark.parametrize("lay", ["linear", "swizzled_128x4"])
def test_requant_bit_exact(fmt, rows, cols, brows, bcols, lay):
    codes, scales = workloads.block_fp8_source(rows, cols, seed=rows + cols, brows=brows, bcols=bcols)
    out = mxq.requant_fp8_mx(codes.cuda(), scales.cuda(), brows, bcols, fmt, layout=lay)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    oc, os_ = oracle.requant_fp8_mx(codes.numpy(), scales.numpy(), brows, bcols, fmt)
    assert np.array_equal(out["codes"].cpu().numpy(), oc)
    got = out["scales"].cpu().numpy().reshape(-1)
    want = os_.reshape(-1) if lay == "linear" else layout.to_tiled_128x4(os_)
    assert np.array_equal(got, want)


def test_requant_nonfinite_source_sets_status():
    codes, scales = workloads.block_fp8_source(128, 256, seed=9)
    codes[5, 77] = 0x7F                       # the E4M3 NaN pattern
    out = mxq.requant_fp8_mx(codes.cuda(), scales.cuda(), 128, 128, "mxfp8")
    torch.cuda.synchronize()
    assert int(out["status"].item()) & mxq.DEV_NONFINITE_INPUT
    codes, scales = workloads.block_fp8_source(128, 256, seed=9)
    scales[0, 1] = float("inf")
    out = mxq.requant_fp8_mx(codes.cuda(), scales.cuda(), 128, 128, "mxfp4")
    torch.cuda.synchronize()
    assert int(out["status"].item()) & mxq.DEV_NONFINITE_INPUT


@pytest.mark.parametrize("fmt", ["mxfp8", "mxfp4"])
def test_requant_extreme_block_scales(fmt):
    """Block scales outside the range where one multiply by sc 2^-e replaces
    the two roundings (tiny scales whose products go subnormal, huge ones),
    the range edges, a zero scale (an all-zero block: e = -127) and a
    negative scale: still bit-exact with the oracle."""
    codes, scales = workloads.block_fp8_source(256, 512, seed=21)
    s = scales.clone()
    s[0, 0] = 2.0 ** -120
    s[0, 1] = 1e-38
    s[0, 2] = 2.0 ** 101
    s[0, 3] = 0.0
    s[1, 0] = -0.75
    s[1, 1] = 2.0 ** -117
    s[1, 2] = 2.0 ** 100
    s[1, 3] = 2.0 ** -126
    out = mxq.requant_fp8_mx(codes.cuda(), s.cuda(), 128, 128, fmt)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    oc, os_ = oracle.requant_fp8_mx(codes.numpy(), s.numpy(), 128, 128, fmt)
    assert np.array_equal(out["codes"].cpu().numpy(), oc)
    assert np.array_equal(out["scales"].cpu().numpy(), os_)


def check_requant_sampled_rows(codes, bs, out, fmt, seed=8, n_rows=40):
    """Sampled output rows against the oracle.  A row's MX codes depend only
    on its source row and that row's block scales, so the sampled source
    rows form one small source whose every row is its own block row
    (brows = 1, the original 128-column blocks)."""
    rows = codes.shape[0]
    rng = np.random.default_rng(seed)
    sample = sorted(set(rng.integers(0, rows, n_rows).tolist()) | {0, rows - 1})
    src = codes[sample].cpu().numpy()
    sc = bs[[r // 128 for r in sample]].cpu().numpy()
    oc, os_ = oracle.requant_fp8_mx(src, sc, 1, 128, fmt)
    assert np.array_equal(out["codes"][sample].cpu().numpy(), oc)
    assert np.array_equal(out["scales"][sample].cpu().numpy(), os_)


def test_full_size_requant_sampled_rows():
    """The benchmark's launches at full size: the gate_up [512 * 1536, 2048]
    and down [512 * 2048, 768] stacks of a routed layer held as block FP8
    (128 x 128 source blocks), requantized to MXFP4 with linear scales."""
    for rows, cols in ((512 * 1536, 2048), (512 * 2048, 768)):
        codes, bs = workloads.block_fp8_stack(rows, cols, device="cuda")
        out = mxq.requant_fp8_mx(codes, bs, 128, 128, "mxfp4")
        torch.cuda.synchronize()
        assert int(out["status"].item()) == 0
        check_requant_sampled_rows(codes, bs, out, "mxfp4")
        del codes, bs, out


def test_dequantized_values_on_e2m1_ties():
    """Source values whose fp32 dequantization lands exactly on an E2M1 tie
    (1.125 * RN32(1.25 / 1.125) = 1.25 + 2^-24, rounded once to 1.25): at
    block exponent 0 (with a 4.0 in the block) and at exponent -2 (alone),
    each tie keeps its even code, bit-exact with the oracle."""
    sc = np.float32(np.float32(1.25) / np.float32(1.125))
    q = np.zeros((128, 64), np.uint8)
    q[:, 0] = 0x48                                       # 4.0
    q[:, 1] = 0x39                                       # 1.125
    q[:, 33] = 0x39
    bs = np.full((1, 1), sc, np.float32)
    out = mxq.requant_fp8_mx(torch.from_numpy(q).cuda(), torch.from_numpy(bs).cuda(), 128, 128, "mxfp4")
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    oc, os_ = oracle.requant_fp8_mx(q, bs, 128, 128, "mxfp4")
    assert np.array_equal(out["codes"].cpu().numpy(), oc)
    assert np.array_equal(out["scales"].cpu().numpy(), os_)
    assert oc[0, 0] == 0x26 and os_[0, 0] == 127         # 4.44 -> 4, 1.25 -> 1.0
    assert oc[0, 16] == 0x60 and os_[0, 1] == 125        # 1.25 * 4 = 5 -> 4 (code 6)
