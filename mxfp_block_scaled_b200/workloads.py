"""Seeded synthetic inputs shaped like the MoE checkpoints the quantizer
converts.  Random numbers only: nothing here quantizes, scales or rounds
beyond the single cast of each drawn value to bf16.

The real checkpoints (Qwen3.8-Flash-Next bf16 experts) are not available,
so these stand in for them, with the shapes the model cards give:

* routed experts stored stacked, fused gate_up ``[E, 2I, H]`` and down
  ``[E, H, I]`` (dabsLabs/Qwen3.8-Flash-Next-NVFP4, "What makes this build
  different": ``[512, out, in]``, fused gate_up; the census there is 48
  layers x 512 experts x 3 projections);
* the shared expert, gate/up ``[2560, 2048]`` and down ``[2048, 1280]``,
  with an MTP-style copy whose widening 640 -> 1280 is zero rows in gate
  and up and zero columns in down (azampatti/Qwen3.8-Flash-Next-FP4-Local-AZ,
  "The shared expert");
* activation token tiles ``[T, 2048]`` (MJPansa/Qwen3.8-Flash-Next-MXFP4-FP8-R12,
  "Quantization format": activations dynamically quantized at run time).

Every generator takes a seed and a torch device and returns bf16 tensors.
A given (seed, device type) always yields the same bits.
"""
import math

import torch

# Four fixed outlier channels of the activation tiles (a fixed reading:
# the workload asks for "4 fixed outlier channels" without naming them).
ACT_OUTLIER_CHANNELS = (101, 717, 1333, 1949)


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal_bf16(shape, std, gen, device):
    return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std)


def tiny_moe_layer(seed=0, device="cpu", experts=8, hidden=256, inter=128):
    """Tiny routed-expert layer: gate_up [E, 2I, H], down [E, H, I] with
    2I = hidden here (8 x 256 x 256 and 8 x 256 x 128 by default).
    Values N(0, 0.02); 0.1 % of entries (Bernoulli per element) x 10."""
    g = _gen(seed, device)
    out = []
    for shape in ((experts, 2 * inter, hidden), (experts, hidden, inter)):
        w = _normal_bf16(shape, 0.02, g, device)
        mask = torch.rand(shape, generator=g, device=device) < 0.001
        w = torch.where(mask, w * 10.0, w)
        out.append(w.to(torch.bfloat16))
    return out[0], out[1]


def full_moe_layer(seed=0, device="cuda", experts=512, hidden=2048, inter=768,
                   chunk=64):
    """Full-size routed-expert layer: gate_up [E, 2I, H], down [E, H, I]
    (512 x 1536 x 2048 and 512 x 2048 x 768 by default, 2,415,919,104
    values).  Per expert sigma_e = exp(U(ln 0.005, ln 0.05)), shared by
    that expert's gate_up and down; values N(0, sigma_e); 0.05 % of entries
    replaced by sign(x) * 8 sigma_e."""
    g = _gen(seed, device)
    sig = torch.exp(torch.empty(experts, device=device).uniform_(
        math.log(0.005), math.log(0.05), generator=g))
    gate_up = torch.empty((experts, 2 * inter, hidden), dtype=torch.bfloat16, device=device)
    down = torch.empty((experts, hidden, inter), dtype=torch.bfloat16, device=device)
    for t in (gate_up, down):
        for e0 in range(0, experts, chunk):
            e1 = min(experts, e0 + chunk)
            s = sig[e0:e1].view(-1, 1, 1)
            w = torch.randn((e1 - e0,) + tuple(t.shape[1:]), generator=g, device=device) * s
            mask = torch.rand(w.shape, generator=g, device=device) < 0.0005
            w = torch.where(mask, torch.sign(w) * 8.0 * s, w)
            t[e0:e1] = w.to(torch.bfloat16)
            del w, mask
    return gate_up, down, sig


def shared_expert_layer(seed=0, device="cpu", inter=1280, hidden=2048,
                        pad_from=640, padded=False, pad_up=True):
    """One layer's shared expert: fused gate/up [2*inter, hidden] (gate rows
    first) and down [hidden, inter], values N(0, 0.02).  ``padded`` gives the
    MTP-style copy: gate rows [pad_from, inter) zero, up rows likewise when
    ``pad_up`` (fused rows [inter + pad_from, 2*inter)), and down columns
    [pad_from, inter) zero."""
    g = _gen(seed, device)
    gu = _normal_bf16((2 * inter, hidden), 0.02, g, device)
    dn = _normal_bf16((hidden, inter), 0.02, g, device)
    if padded:
        gu[pad_from:inter] = 0
        if pad_up:
            gu[inter + pad_from:] = 0
        dn[:, pad_from:] = 0
    return gu.to(torch.bfloat16), dn.to(torch.bfloat16)


def student_t_mix_layer(seed=0, device="cuda", experts=512, hidden=2048, inter=768,
                        p_tail=0.01, chunk=64):
    """Mixed-format layer input: gate_up [E, 2I, H], down [E, H, I]; values
    N(0, 0.02), except a fraction ``p_tail`` (a reading: the workload names a
    Student-t(4) tail mix without its weight) drawn from 0.02 * t_4 with
    t_4 = N / sqrt(chi2_4 / 4)."""
    g = _gen(seed, device)
    out = []
    for shape in ((experts, 2 * inter, hidden), (experts, hidden, inter)):
        t = torch.empty(shape, dtype=torch.bfloat16, device=device)
        for e0 in range(0, experts, chunk):
            e1 = min(experts, e0 + chunk)
            sub = (e1 - e0,) + shape[1:]
            w = torch.randn(sub, generator=g, device=device) * 0.02
            z = torch.randn(sub, generator=g, device=device)
            chi2 = torch.randn(sub + (4,), generator=g, device=device).square().sum(-1)
            tail = 0.02 * z / torch.sqrt(chi2 / 4.0)
            mask = torch.rand(sub, generator=g, device=device) < p_tail
            t[e0:e1] = torch.where(mask, tail, w).to(torch.bfloat16)
            del w, z, chi2, tail, mask
        out.append(t)
    return out[0], out[1]


def activation_tile(T, seed=0, device="cpu", hidden=2048):
    """Token tile [T, hidden], values N(0, 1) with the four fixed outlier
    channels scaled x 30."""
    g = _gen(seed, device)
    a = torch.randn((T, hidden), generator=g, device=device)
    for c in ACT_OUTLIER_CHANNELS:
        if c < hidden:
            a[:, c] *= 30.0
    return a.to(torch.bfloat16)


def block_fp8_source(rows, cols, seed=0, device="cpu", brows=128, bcols=128):
    """A block-FP8 source tensor as stored by FP8 checkpoints: E4M3 codes
    [rows, cols] (uint8) and one fp32 scale per brows x bcols block
    (MJPansa/Qwen3.8-Flash-Next-MXFP4-FP8-R12, "Quantization format": the
    retained layers keep the source block-FP8 format; the block shape is a
    reading, 128 x 128).  Codes are drawn directly, not encoded from values:
    random sign, exponent field 1..15 drawn with weight 2^field (large
    magnitudes most frequent, as in a tensor scaled to use the FP8 range),
    uniform mantissa, the NaN pattern S.1111.111 replaced by S.1111.110, and
    1 % of codes zero.  Scales are log-uniform in [2^-16, 2^-6]."""
    g = _gen(seed, device)
    w = torch.pow(2.0, torch.arange(1, 16, dtype=torch.float32, device=device))
    expo = torch.multinomial(w / w.sum(), rows * cols, replacement=True, generator=g) + 1
    mant = torch.randint(0, 8, (rows * cols,), generator=g, device=device)
    sign = torch.randint(0, 2, (rows * cols,), generator=g, device=device)
    mag = expo * 8 + mant
    mag = torch.where(mag == 0x7F, torch.full_like(mag, 0x7E), mag)
    zero = torch.rand(rows * cols, generator=g, device=device) < 0.01
    mag = torch.where(zero, torch.zeros_like(mag), mag)
    codes = (sign * 128 + mag).to(torch.uint8).reshape(rows, cols)
    nbr, nbc = -(-rows // brows), -(-cols // bcols)
    scales = torch.pow(2.0, torch.empty((nbr, nbc), device=device).uniform_(-16.0, -6.0, generator=g))
    return codes, scales.to(torch.float32)


def block_fp8_stack(rows, cols, device="cpu", seed0=1000, chunk_rows=128 * 256):
    """A full-size block-FP8 stack (128 x 128 source blocks) built from
    block_fp8_source in runs of chunk_rows rows (a multiple of 128), seeds
    seed0, seed0 + 1, ... per run, so the generator's temporaries stay small.
    Returns codes [rows, cols] uint8 and scales [ceil(rows/128),
    ceil(cols/128)] fp32."""
    assert chunk_rows % 128 == 0
    codes = torch.empty((rows, cols), dtype=torch.uint8, device=device)
    scales = torch.empty((-(-rows // 128), -(-cols // 128)), dtype=torch.float32, device=device)
    for i, r0 in enumerate(range(0, rows, chunk_rows)):
        c, b = block_fp8_source(min(chunk_rows, rows - r0), cols, seed=seed0 + i, device=device)
        codes[r0:r0 + c.shape[0]] = c
        scales[r0 // 128:r0 // 128 + b.shape[0]] = b
    return codes, scales


def bf16_bits(t):
    """bf16 tensor -> numpy uint16 array of its bit patterns (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view("uint16")
