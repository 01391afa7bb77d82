"""Failure paths on the GPU without faulting or hanging it.  A single-pass
launch told to stall (include/mxq_test.h: its publisher releases no group,
so every inter-CTA wait runs into its iteration limit) must end on its own
with MXQ_DEV_WAIT_TIMEOUT, well under a second, and the device must then
quantize the same input bit-exactly.  The failure is made by the host-side
request; no trap, assert or bad address is involved."""
import time

import numpy as np
import pytest
import torch

import oracle
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


def _expect_exact(x_cpu, out):
    G, R, C = x_cpu.shape
    c, s, s2, _ = oracle.quantize_nvfp4(workloads.bf16_bits(x_cpu).reshape(G, R, C), mode=1)
    assert np.array_equal(out["codes"].cpu().numpy().reshape(-1), c.reshape(-1))
    assert np.array_equal(out["scales"].cpu().numpy().reshape(-1), s.reshape(-1))
    assert np.array_equal(out["s2"].cpu().numpy()[:G].view(np.uint32), s2.view(np.uint32))


def test_stalled_single_pass_reports_wait_timeout_and_the_device_recovers():
    gu, _ = workloads.tiny_moe_layer(seed=3)      # 8 groups of 4096 blocks: the single pass
    x = gu.cuda()
    lib = mxq.load()
    torch.cuda.synchronize()
    lib.mxq_test_stall_next_single_pass(1)
    t0 = time.perf_counter()
    out = mxq.quantize_nvfp4(x)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(out["status"].item()) & mxq.DEV_WAIT_TIMEOUT
    assert elapsed < 5.0, elapsed
    # the request was taken by that launch: the next call is normal and exact
    out = mxq.quantize_nvfp4(x)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    _expect_exact(gu, out)


def test_stalled_one_grid_group_reports_wait_timeout_and_the_device_recovers():
    """The lone-group grid (an activation tile of 4096 tokens): its first CTA
    never reports its amax, every other CTA's bounded wait runs out."""
    a = workloads.activation_tile(4096, seed=5)
    x = a.cuda().reshape(1, 4096, -1)
    lib = mxq.load()
    torch.cuda.synchronize()
    lib.mxq_test_stall_next_single_pass(1)
    t0 = time.perf_counter()
    out = mxq.quantize_nvfp4(x)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(out["status"].item()) & mxq.DEV_WAIT_TIMEOUT
    assert elapsed < 5.0, elapsed
    out = mxq.quantize_nvfp4(x)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    _expect_exact(a.reshape(1, 4096, -1), out)


def test_withdrawn_stall_request_changes_nothing():
    gu, _ = workloads.tiny_moe_layer(seed=4)
    lib = mxq.load()
    lib.mxq_test_stall_next_single_pass(1)
    lib.mxq_test_stall_next_single_pass(0)
    out = mxq.quantize_nvfp4(gu.cuda())
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    _expect_exact(gu, out)
