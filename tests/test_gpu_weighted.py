"""Weighted-SSE block-scale search on the GPU (mxq_quantize_nvfp4_weighted,
through the C ABI) against the CPU oracle on the same seeded inputs:
bit-exact codes, scale bytes and s2, with shared and per-expert weights,
linear and tiled scales.  The weights stand in for a diagonal Hessian: the
mean squared activation of each input channel over a synthetic token tile
(the real calibration corpora are not available)."""
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


def _channel_weights(hidden, seed):
    a = workloads.activation_tile(64, seed=seed, hidden=hidden).float()
    return (a * a).mean(0).contiguous()


def _check(x, h, lay="linear"):
    G, R, C = x.shape
    out = mxq.quantize_nvfp4_weighted(x, h.cuda(), layout=lay)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    c, s, s2 = oracle.quantize_nvfp4_weighted(workloads.bf16_bits(x).reshape(G, R, C), h.numpy())
    assert np.array_equal(out["codes"].cpu().numpy(), c)
    assert np.array_equal(out["s2"].cpu().numpy()[:G].view(np.uint32), s2.view(np.uint32))
    got = out["scales"].cpu().numpy().reshape(-1)
    want = s.reshape(-1) if lay == "linear" else np.concatenate(
        [layout.to_tiled_128x4(s[g]) for g in range(G)])
    assert np.array_equal(got, want)
    return s


def test_tiny_layer_shared_weights():
    gu, _ = workloads.tiny_moe_layer(seed=4)
    s = _check(gu.cuda(), _channel_weights(gu.shape[2], seed=4))
    # the search leaves the 4/6 plans' codes in place on most blocks but not all
    c46, s46, _, _ = oracle.quantize_nvfp4(workloads.bf16_bits(gu).reshape(gu.shape), mode=1)
    frac = (s != s46).mean()
    assert 0.0 < frac < 0.9


def test_per_expert_weights_and_tiled_scales():
    gu, dn = workloads.tiny_moe_layer(seed=5)
    g = torch.Generator().manual_seed(5)
    h = torch.distributions.Gamma(torch.tensor(0.7), torch.tensor(1.0)).sample((dn.shape[0], dn.shape[2]))
    _check(dn.cuda(), h.float().contiguous())
    _check(gu.cuda(), _channel_weights(gu.shape[2], seed=6), lay="swizzled_128x4")


@pytest.mark.parametrize("shape", [(3, 5, 48), (1, 1, 16), (2, 130, 80)])
def test_ragged_shapes(shape):
    g = torch.Generator().manual_seed(sum(shape))
    x = (torch.randn(shape, generator=g) * 0.05).to(torch.bfloat16).cuda()
    h = torch.rand(shape[2], generator=g) * 3.0
    _check(x, h.contiguous())


def test_bad_weight_sets_status():
    x = (torch.randn((2, 4, 32)) * 0.05).to(torch.bfloat16).cuda()
    h = torch.ones(32)
    h[7] = -1.0
    out = mxq.quantize_nvfp4_weighted(x, h.cuda())
    torch.cuda.synchronize()
    assert int(out["status"].item()) & mxq.DEV_NONFINITE_INPUT


def _grid_blocks(seed, nblocks):
    """Blocks on grids several candidate scales represent exactly (ties of
    the weighted error), mixed with random blocks; group amax 2.625 makes
    s2 = 2^-10 exactly."""
    rng = np.random.default_rng(seed)
    x = np.zeros((nblocks, 16), np.float32)
    for b in range(nblocks):
        base = np.float32(2.0 ** -10 * rng.choice([2.0, 4.0, 8.0, 16.0]))
        if b % 3 == 2:
            x[b] = rng.standard_normal(16) * 0.2
        else:
            x[b] = rng.choice([0.0, 1.0, 2.0, 3.0, -1.0, -2.0, -4.0], 16) * base
            x[b, 0] = 4.0 * base
    x[0] = 0.0
    x[0, 0] = 2.625
    return torch.from_numpy(x.reshape(1, nblocks, 16)).to(torch.bfloat16)


@pytest.mark.parametrize("kind", ["zero", "one_hot", "huge", "gamma"])
def test_ties_and_unfiltered_weights_take_the_binary64_search(kind):
    """Exact ties (all-zero weights: every candidate scores 0; one-hot
    weights on grid blocks), weights beyond the fp32 filter's range and plain
    weights on tie-rich blocks must all give the binary64 choice (ties to
    the smaller code), bit-exact with the oracle."""
    x = _grid_blocks(7, 96)
    h = {"zero": torch.zeros(16),
         "one_hot": torch.nn.functional.one_hot(torch.tensor(3), 16).float(),
         "huge": torch.full((16,), 2.0 ** 60),
         "gamma": torch.distributions.Gamma(torch.tensor(0.5), torch.tensor(1.0)).sample((16,))}[kind]
    _check(x.cuda(), h.float().contiguous())


def test_full_size_layer_sampled_experts():
    """The benchmark's launch at full size: gate_up [512, 1536, 2048] and
    down [512, 2048, 768], each stack with one row of per-channel weights
    (the mean squared activation over a 4096-token tile).  Groups are
    experts, so an expert's slab quantizes alone exactly as inside its
    stack: sampled experts are checked against the oracle."""
    gu, dn, _ = workloads.full_moe_layer(seed=0, device="cuda")
    for x in (gu, dn):
        G, R, C = x.shape
        a = workloads.activation_tile(4096, seed=7, hidden=C).float()
        h = (a * a).mean(0).contiguous()
        out = mxq.quantize_nvfp4_weighted(x, h.cuda())
        torch.cuda.synchronize()
        assert int(out["status"].item()) == 0
        for e in (0, 300, G - 1):
            c, s, s2 = oracle.quantize_nvfp4_weighted(workloads.bf16_bits(x[e:e + 1]), h.numpy())
            assert np.array_equal(out["codes"][e].cpu().numpy(), c[0]), e
            assert np.array_equal(out["scales"][e].cpu().numpy(), s[0]), e
            assert out["s2"][e].cpu().numpy().view(np.uint32) == s2.view(np.uint32)[0], e
