"""Host-resident layers converted in overlapped chunks (HostLayerConverter)
give exactly the results of one call per stack on the device: codes, scale
bytes, global scales and per-tensor relative errors are bit-identical."""
import pytest
import torch

from mxfp_block_scaled_b200 import layers, mxq, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from mxfp_block_scaled_b200 import build
    build.build()
    mxq.load()


@pytest.mark.parametrize("chunk", [3, 8, 64])
def test_streamed_conversion_equals_whole_stack_calls(chunk):
    gu, dn = workloads.tiny_moe_layer(seed=11)
    h_gu, h_dn = gu.pin_memory(), dn.pin_memory()
    conv = layers.HostLayerConverter(gu.shape, dn.shape, chunk=chunk)
    out = layers.host_outputs(h_gu, h_dn)
    for _ in range(2):                                   # slots are reused across calls too
        conv.run(h_gu, h_dn, out)
        torch.cuda.synchronize()
    assert conv.status() == 0
    for name, x, tps in (("gate_up", gu.cuda(), 2), ("down", dn.cuda(), 1)):
        E, R, C = x.shape
        q = mxq.quantize_nvfp4(x)
        _, _, rel = mxq.dequant_relerr(x, q["codes"], q["scales"], q["s2"], "nvfp4", E * tps, R // tps,
                                       C, tps)
        torch.cuda.synchronize()
        o = out[name]
        assert torch.equal(o["codes"], q["codes"].cpu())
        assert torch.equal(o["scales"], q["scales"].cpu())
        assert torch.equal(o["s2"], q["s2"].cpu())
        assert torch.equal(o["relerr"], rel.cpu())
