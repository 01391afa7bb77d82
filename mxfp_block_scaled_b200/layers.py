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


def census(results, results_rtn=None, stream=None):
    """The census of the given layer results, formed on the device by
    mxq_census_add (dabsLabs/Qwen3.8-Flash-Next-NVFP4, metric table: mean
    and max relative error over the unstacked tensors; "What makes this
    build different": SSE(chosen) / SSE(RTN) - 1 and the share of 16-blocks
    that chose M=4).  `results` are quantize_routed_layer results; with
    `results_rtn` (the same layers quantized in "rtn" mode) each tensor is
    added with its RTN error sum, which gives sse_vs_rtn.  Returns the
    struct's fields as a dict (mxq.CENSUS_FIELDS)."""
    dev = results[0]["gate_up"]["codes"].device if results else "cuda"
    c = mxq.Census(device=dev, stream=stream)
    for i, q in enumerate(results):
        for k in ("gate_up", "down"):
            s = q[k]
            rtn = results_rtn[i][k]["sum_sq_err"] if results_rtn is not None else None
            nvfp4 = s["fmt"] == "nvfp4"
            E, R, C2 = s["codes"].shape
            C = C2 * 2 if s["fmt"] != "mxfp8" else C2
            c.add(n_tensors=s["relerr"].numel(), sum_sq_err=s["sum_sq_err"], sum_sq_ref=s["sum_sq_ref"],
                  relerr=s["relerr"], sum_sq_err_rtn=rtn, n_groups=E if nvfp4 else 0,
                  m4_count=s["m4_count"] if nvfp4 else None, blocks_per_group=R * C // 16 if nvfp4 else 0,
                  stream=stream)
    return c.result()


def relerr_census(results):
    """Mean and max relative error over every unstacked tensor of the given
    layer results, and the tensor count (the metric-table figures)."""
    r = census(results)
    return r["mean_relerr"], r["max_relerr"], r["n_tensors"]


def sse_vs_rtn(results, results_rtn):
    """SSE(chosen) / SSE(RTN) - 1 over every unstacked tensor of the given
    layer results ("four_six" and "rtn" quantize_routed_layer results of the
    same layers).  The 4/6 rule is never worse than RTN per block on the exact
    error, so the exact figure is never above 0; from the verifier's sums,
    each within 11 * 2^-24 relative of its exact value, it can come out above
    0 by at most about 1.4e-6 (a layer whose blocks nearly all tie)."""
    return census(results, results_rtn)["sse_vs_rtn"]


def m4_fraction(results):
    """Fraction of NVFP4 blocks that took the M=4 plan (from the per-group
    M=4 counts of the quantizer)."""
    return census(results)["m4_fraction"]


# ------------------------------------------------ host-resident layers --
def host_outputs(h_gate_up, h_down):
    """Pinned host buffers for convert_layer_from_host: per stack the codes,
    scales, s2 and per-tensor relative errors (gate_up unstacked into 2E
    tensors, down into E)."""
    out = {}
    for name, h in (("gate_up", h_gate_up), ("down", h_down)):
        E, R, C = h.shape
        nt = 2 * E if name == "gate_up" else E
        out[name] = {
            "codes": torch.empty((E, R, C // 2), dtype=torch.uint8, pin_memory=True),
            "scales": torch.empty((E, R, C // 16), dtype=torch.uint8, pin_memory=True),
            "s2": torch.empty(E, dtype=torch.float32, pin_memory=True),
            "relerr": torch.empty(nt, dtype=torch.float64, pin_memory=True),
        }
    return out


class _Slot:
    """Device buffers of one chunk of `chunk` experts of one stack."""

    def __init__(self, chunk, R, C, tps, device):
        self.x = torch.empty((chunk, R, C), dtype=torch.bfloat16, device=device)
        self.codes = torch.empty((chunk, R, C // 2), dtype=torch.uint8, device=device)
        self.scales = torch.empty((chunk, R, C // 16), dtype=torch.uint8, device=device)
        self.s2 = torch.empty(chunk, dtype=torch.float32, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        nt = chunk * tps
        self.err = torch.empty(nt, dtype=torch.float64, device=device)
        self.ref = torch.empty(nt, dtype=torch.float64, device=device)
        self.rel = torch.empty(nt, dtype=torch.float64, device=device)
        self.wsq, _ = mxq._workspace("quantize_nvfp4", chunk, R, C, device)
        self.wsv, _ = mxq._workspace("dequant_relerr", nt, R // tps, C, device)
        self.ev_in = torch.cuda.Event()      # input copied in
        self.ev_done = torch.cuda.Event()    # outputs written
        self.ev_out = torch.cuda.Event()     # outputs copied out (slot free again)
        self.used = False


class HostLayerConverter:
    """NVFP4 4/6 quantize + verify of routed-expert layers that live in pinned
    host memory, in chunks of `chunk` experts.  Host -> device copies, the
    kernels and device -> host copies of neighbouring chunks are queued on
    three streams (event-ordered, `nbuf` device buffers per stack), so both
    PCIe directions and the GPU work at the same time.  The results equal one
    call per stack over the whole layer: every expert is its own NVFP4 group
    (gate and up of an expert still share one weight_scale_2) and every
    unstacked tensor is verified on its own.

        conv = HostLayerConverter(h_gate_up.shape, h_down.shape)
        out = host_outputs(h_gate_up, h_down)
        conv.run(h_gate_up, h_down, out)    # enqueues; the current stream waits for it
        torch.cuda.current_stream().synchronize()
    """

    def __init__(self, gate_up_shape, down_shape, chunk=64, mode="four_six", device="cuda", nbuf=2):
        self.chunk, self.mode, self.device = int(chunk), mode, torch.device(device)
        self.stacks = []
        for name, shape, tps in (("gate_up", tuple(gate_up_shape), 2), ("down", tuple(down_shape), 1)):
            E, R, C = shape
            c = min(self.chunk, E)
            self.stacks.append((name, shape, tps, [_Slot(c, R, C, tps, self.device) for _ in range(nbuf)]))
        self.s_h2d = torch.cuda.Stream(device=self.device)
        self.s_comp = torch.cuda.Stream(device=self.device)
        self.s_d2h = torch.cuda.Stream(device=self.device)

    def run(self, h_gate_up, h_down, out):
        cur = torch.cuda.current_stream(self.device)
        for s in (self.s_h2d, self.s_comp, self.s_d2h):
            s.wait_stream(cur)
        for (name, shape, tps, slots), h in zip(self.stacks, (h_gate_up, h_down)):
            E, R, C = shape
            o = out[name]
            for k, e0 in enumerate(range(0, E, self.chunk)):
                n = min(self.chunk, E - e0)
                sl = slots[k % len(slots)]
                with torch.cuda.stream(self.s_h2d):
                    if sl.used:
                        self.s_h2d.wait_event(sl.ev_done)       # the previous chunk has read x
                    sl.x[:n].copy_(h[e0:e0 + n], non_blocking=True)
                    sl.ev_in.record(self.s_h2d)
                with torch.cuda.stream(self.s_comp):
                    self.s_comp.wait_event(sl.ev_in)
                    if sl.used:
                        self.s_comp.wait_event(sl.ev_out)       # its outputs have been copied out
                    mxq.mxq_quantize_nvfp4(sl.x[:n], n, R, C, self.mode, "linear", sl.codes[:n],
                                           sl.scales[:n], sl.s2[:n], None, None, sl.status, sl.wsq,
                                           stream=self.s_comp)
                    mxq.mxq_dequant_relerr(sl.x[:n], sl.codes[:n], sl.scales[:n], sl.s2[:n], "nvfp4",
                                           "linear", n * tps, R // tps, C, tps, sl.err[:n * tps],
                                           sl.ref[:n * tps], sl.rel[:n * tps], sl.wsv,
                                           stream=self.s_comp)
                    sl.ev_done.record(self.s_comp)
                with torch.cuda.stream(self.s_d2h):
                    self.s_d2h.wait_event(sl.ev_done)
                    o["codes"][e0:e0 + n].copy_(sl.codes[:n], non_blocking=True)
                    o["scales"][e0:e0 + n].copy_(sl.scales[:n], non_blocking=True)
                    o["s2"][e0:e0 + n].copy_(sl.s2[:n], non_blocking=True)
                    o["relerr"][e0 * tps:(e0 + n) * tps].copy_(sl.rel[:n * tps], non_blocking=True)
                    sl.ev_out.record(self.s_d2h)
                sl.used = True
        cur.wait_stream(self.s_d2h)

    def status(self):
        """OR of the device status words of every chunk (after a sync)."""
        v = 0
        for _, _, _, slots in self.stacks:
            for sl in slots:
                v |= int(sl.status.item())
        return v
