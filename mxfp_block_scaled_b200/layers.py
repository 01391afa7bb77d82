"""Layer-level conversion: loops over the C-ABI calls for whole MoE layers.

Argument marshalling only; every step runs in libmxq.so.

* A routed-expert layer is stored stacked: fused gate_up [E, 2I, H] and down
  [E, H, I] (dabsLabs/Qwen3.8-Flash-Next-NVFP4, "What makes this build
  different": [512, out, in], fused gate_up).  NVFP4 groups are the
  per-expert slabs, so gate and up share one weight_scale_2
  (josch15366/Qwen3.8-Flash-Next-NVFP4-LocalHessian-Experts, introduction).
* Unstacking into per-expert gate / up / down tensors is a zero-copy view of
  row ranges of the codes and scales: gate_e = rows [0, I) of slab e,
  up_e = rows [I, 2I) (the split convention; the codes do not depend on it
  because the slab shares one s2 and blocks are row-local).
* A mixed-format model keeps a per-layer format list
  (MJPansa/Qwen3.8-Flash-Next-MXFP4-FP8-R12, "Quantization format" and
  "Retained layers": some routed-expert layers MXFP4, the others in another
  format).
"""
import torch

from . import mxq


def quantize_routed_layer(gate_up, down, fmt="nvfp4", mode="four_six", stream=None):
    """Quantize one stacked routed-expert layer and verify it.

    fmt: "nvfp4" (4/6-optimal or RTN block scales, per-expert weight_scale_2)
    or "mxfp4" / "mxfp8".  Returns {"gate_up": q, "down": q} where q holds the
    codes, scales (and s2 for NVFP4) and the per-tensor relative errors of the
    unstacked tensors (gate_0, up_0, gate_1, ... for gate_up)."""
    out = {}
    for name, x in (("gate_up", gate_up), ("down", down)):
        E, R, C = x.shape
        tps = 2 if name == "gate_up" else 1
        if fmt == "nvfp4":
            q = mxq.quantize_nvfp4(x, mode=mode, stream=stream)
            s2 = q["s2"]
        else:
            q = mxq.quantize_mx(x, fmt, stream=stream)
            s2 = None
        err, ref, rel = mxq.dequant_relerr(x, q["codes"], q["scales"], s2, fmt, E * tps, R // tps,
                                           C, tps if fmt == "nvfp4" else 1, stream=stream)
        q.update(fmt=fmt, sum_sq_err=err, sum_sq_ref=ref, relerr=rel)
        out[name] = q
    return out


def unstack_expert(layer_q, e):
    """Per-expert tensors of a quantized layer as zero-copy views:
    {"gate": (codes, scales), "up": ..., "down": ..., "weight_scale_2_gate_up",
    "weight_scale_2_down"} (the last two for NVFP4 only; gate and up share
    the first)."""
    gu, dn = layer_q["gate_up"], layer_q["down"]
    I = gu["codes"].shape[1] // 2
    res = {
        "gate": (gu["codes"][e, :I], gu["scales"][e, :I]),
        "up": (gu["codes"][e, I:], gu["scales"][e, I:]),
        "down": (dn["codes"][e], dn["scales"][e]),
    }
    if "s2" in gu:
        res["weight_scale_2_gate_up"] = gu["s2"][e]
        res["weight_scale_2_down"] = dn["s2"][e]
    return res


def quantize_mixed(layers, formats, stream=None):
    """Convert a list of (gate_up, down) layers with one format per layer
    ("nvfp4" = NVFP4 4/6-optimal, "mxfp4", "mxfp8").  Returns the list of
    per-layer results of quantize_routed_layer."""
    if len(layers) != len(formats):
        raise ValueError("one format per layer")
    return [quantize_routed_layer(gu, dn, fmt=f, stream=stream) for (gu, dn), f in zip(layers, formats)]


def relerr_census(results):
    """Mean and max relative error over every unstacked tensor of the given
    layer results (the metric-table figures: mean / max rel-err over the
    expert census)."""
    rel = torch.cat([q[k]["relerr"] for q in results for k in ("gate_up", "down")])
    return float(rel.mean()), float(rel.max()), int(rel.numel())
