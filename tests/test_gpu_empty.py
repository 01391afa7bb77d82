"""Inputs without elements on every entry point: the calls succeed, write
what the definition gives for them (a group without elements has amax 0,
so s2 = 0 and an M=4 count of 0; an empty activation tile has
input_scale 0; an empty tensor has error and reference sums 0 and a
relative error of 0, as in the oracle) and touch nothing else."""
import numpy as np
import pytest
import torch

import oracle
from mxfp_block_scaled_b200 import mxq

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    mxq.load()
    oracle.build()


def _x(shape):
    return torch.zeros(shape, dtype=torch.bfloat16, device="cuda")


@pytest.mark.parametrize("shape", [(0, 16, 32), (3, 0, 32), (1, 0, 16), (2, 8, 0)])
@pytest.mark.parametrize("mode", ["rtn", "four_six"])
@pytest.mark.parametrize("layout", ["linear", "swizzled_128x4"])
def test_nvfp4_groups_without_elements(shape, mode, layout):
    G = shape[0]
    out = mxq.quantize_nvfp4(_x(shape), mode=mode, layout=layout)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    _, _, s2, _ = oracle.quantize_nvfp4(np.zeros(shape, np.uint16), mode=1 if mode == "four_six" else 0)
    assert np.array_equal(out["s2"].cpu().numpy().view(np.uint32), np.asarray(s2).view(np.uint32))
    if G:
        assert np.all(out["m4_count"].cpu().numpy()[:G] == 0)
    gs2, st = mxq.global_scale_nvfp4(_x(shape))
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and np.all(gs2.cpu().numpy().view(np.uint32) == 0)


def test_nvfp4_given_scales_without_elements():
    ok = mxq.quantize_nvfp4_s2(_x((2, 0, 32)), torch.tensor([0.5, 1.0], device="cuda"))
    bad = mxq.quantize_nvfp4_s2(_x((2, 0, 32)), torch.tensor([-1.0, float("nan")], device="cuda"))
    torch.cuda.synchronize()
    assert int(ok["status"].item()) == 0 and np.all(ok["m4_count"].cpu().numpy()[:2] == 0)
    assert int(bad["status"].item()) == mxq.DEV_INVALID_SCALE     # the given scales are still checked


def test_weighted_search_without_elements():
    out = mxq.quantize_nvfp4_weighted(_x((3, 0, 32)), torch.ones(32, device="cuda"))
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0 and np.all(out["s2"].cpu().numpy()[:3] == 0)


@pytest.mark.parametrize("fmt", ["mxfp8", "mxfp4"])
def test_mx_and_activations_without_elements(fmt):
    out = mxq.quantize_mx(_x((0, 64)), fmt)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    for f in (fmt, "nvfp4"):
        a = mxq.quantize_act(_x((0, 2048)), f)
        torch.cuda.synchronize()
        assert int(a["status"].item()) == 0
        if f == "nvfp4":
            assert float(a["input_scale"].item()) == 0.0


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp8"])
def test_verifier_on_empty_tensors(fmt):
    x = _x((3, 0, 32))
    codes = torch.zeros(1, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(1, dtype=torch.uint8, device="cuda")
    s2 = torch.ones(3, dtype=torch.float32, device="cuda")
    err, ref, rel = mxq.dequant_relerr(x, codes, scales, s2, fmt, 3, 0, 32)
    torch.cuda.synchronize()
    assert torch.all(err == 0) and torch.all(ref == 0) and torch.all(rel == 0)
    e0, r0, l0 = mxq.dequant_relerr(x, codes, scales, s2, fmt, 0, 16, 32)
    assert e0.numel() == 0 and r0.numel() == 0 and l0.numel() == 0
    oe, orf = oracle.dequant_relerr(np.zeros((3, 0, 32), np.uint16), np.zeros(1, np.uint8),
                                    np.zeros(1, np.uint8), np.ones(3, np.float32), fmt, 3, 0, 32)
    assert np.all(np.asarray(oe) == 0) and np.all(np.asarray(orf) == 0)
    assert np.all(np.asarray(oracle.relerr_from_sums(oe, orf)) == 0)
