"""The allocation-free verifier entry point (mxq_dequant_relerr_noalloc).

It serves callers that cannot allocate device memory (engines that reserve
their whole memory budget up front, code that must not risk the
synchronisation of a cudaMalloc): its partial sums live in a fixed array in
the library instead of a caller workspace.  Checked here through the C ABI
against the workspace-taking verifier on the same inputs, bit for bit, on
calls in a row (each reuses the array the one before left behind, filled
from another input in between).  This file sorts last so that a run
stopping at the first failure has run every other test first."""
import ctypes

import pytest
import torch

from mxfp_block_scaled_b200 import mxq, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from mxfp_block_scaled_b200 import build
    build.build()
    return mxq.load()


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _case(fmt, x, tps):
    """Quantize x ([G, R, C] bf16 on the device) and return the verifier's
    arguments for it plus the workspace verifier's results."""
    G, R, C = x.shape
    nt, rows = G * tps, R // tps
    if fmt == "nvfp4":
        q = mxq.quantize_nvfp4(x, mode="four_six")
        s2 = q["s2"]
    else:
        q = mxq.quantize_mx(x.view(G * R, C), "mxfp8")
        s2, tps = None, 1
    want = mxq.dequant_relerr(x, q["codes"], q["scales"], s2, fmt, nt, rows, C, tps)
    return (x, q["codes"], q["scales"], s2, nt, rows, C, tps), want


def _noalloc(lib, fmt, args):
    x, codes, scales, s2, nt, rows, C, tps = args
    err = torch.full((nt,), -1.0, dtype=torch.float64, device="cuda")
    sq = torch.full_like(err, -1.0)
    rel = torch.full_like(err, -1.0)
    rc = lib.mxq_dequant_relerr_noalloc(
        _ptr(x), _ptr(codes), _ptr(scales), _ptr(s2), mxq.FMT[fmt], nt, rows, C, tps,
        _ptr(err), _ptr(sq), _ptr(rel), _stream())
    assert rc == 0, rc
    torch.cuda.synchronize()
    return err, sq, rel


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp8"])
def test_noalloc_verifier_matches_workspace_verifier_twice(lib, fmt):
    """Same kernels, same fixed summation order as the workspace verifier, so
    the results must be bit-identical, on two calls in a row; between them a
    call on another input and shape fills the shared array with other
    partials, and none of them may leak into the next call."""
    gu, dn = workloads.tiny_moe_layer(seed=5)
    a_args, a_want = _case(fmt, gu.cuda(), 2)
    b_args, b_want = _case(fmt, (dn.cuda() * 3).contiguous(), 1)
    for args, want in ((a_args, a_want), (b_args, b_want), (a_args, a_want)):
        got = _noalloc(lib, fmt, args)
        for g, w in zip(got, want):
            assert torch.equal(g, w), (g - w).abs().max().item()


def test_noalloc_rejects_requests_beyond_its_array(lib):
    # 131073 chunks of 16384 elements is one chunk more than the array holds;
    # the size check answers before any pointer is touched or work enqueued.
    fake = ctypes.c_void_p(0x100000)
    rc = lib.mxq_dequant_relerr_noalloc(fake, fake, fake, None, mxq.FMT["mxfp8"], 131073, 1,
                                        16384, 1, fake, fake, None, _stream())
    assert rc == 4   # MXQ_ERR_WORKSPACE
