"""Benchmark: NVFP4 4/6-optimal quantize + verify of one full-size
routed-expert layer on B200, reported as algorithmic HBM GB/s.

A step is one pass of the whole hot path over the layer: NVFP4 4/6
quantization of the fused gate_up stack [512, 1536, 2048] (one
weight_scale_2 per expert, shared by gate and up) and of the down stack
[512, 2048, 768], then the dequantize + relative-error verifier over every
unstacked tensor (1024 gate/up tensors [768, 2048] and 512 down tensors
[2048, 768]).  Inputs are synthetic (seeded), resident in HBM, 4.8 GB, far
larger than L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mine|reference]
    python bench.py --workload fp8_requant     # FP8 -> MXFP4 requantization of the same layer
    python bench.py --workload nvfp4_weighted  # weighted-SSE scale search on the same layer

Prints one JSON line on rank 0.  Under torchrun every rank converts its own
layer (independent units, no data-path collective: weak scaling); the step
time is the max over ranks.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

EXPERTS, HIDDEN, INTER = 512, 2048, 768
# Algorithmic bytes per element (unique traffic the method needs):
# quantize reads 2 B and writes 0.5 B of codes + 1/16 B of scales;
# the verifier reads the same 2.5625 B again.
Q_BYTES = 2.0 + 0.5 + 1.0 / 16
V_BYTES = 2.0 + 0.5 + 1.0 / 16
STEP_BYTES_PER_ELEM = Q_BYTES + V_BYTES
# Kernels of this library launched per call (cudaMemsetAsync not counted).
KERNELS_PER_QUANTIZE_NVFP4 = 1   # the single-pass kernel (full-size stacks)
KERNELS_PER_VERIFY = 2           # chunk reduction, per-tensor finalize
METRIC = "NVFP4 4/6-optimal quantize+verify HBM GB/s and % of B200 peak (1 GPU)"
WORKLOAD = ("one full-size routed-expert layer, NVFP4 4/6-optimal quantize + verify: "
            "gate_up bf16 [512,1536,2048] + down [512,2048,768]")
FALLBACK_HBM_GBS = 6650.0


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_sha():
    h = hashlib.sha256()
    for f in ("nvfp4.cu", "mxq_device.cuh"):
        with open(os.path.join(ROOT, "mxfp_block_scaled_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic_per_launch():
    """DRAM bytes per quantize launch from the committed ncu summary, or None
    when the kernel source changed since it was captured."""
    p = os.path.join(ROOT, "profiles", "nvfp4_quant_gate_up_fullsize_traffic.txt")
    try:
        kv = {}
        with open(p) as f:
            for line in f:
                line = line.strip()
                if line and not line.startswith("#") and " " in line:
                    k, v = line.split(None, 1)
                    kv[k] = v
        if kv.get("source_sha") != kernel_source_sha():
            return None
        return float(kv["dram_bytes_per_call"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "200", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                if self.uuid and parts[1] != self.uuid:
                    continue
                try:
                    sm.append(float(parts[2]))
                    mx = float(parts[3])
                except ValueError:
                    continue
                for n, v in zip(names, parts[6:10]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        loaded = [s for s in sm if mx is None or s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def device_uuid():
    try:
        u = torch.cuda.get_device_properties(torch.cuda.current_device()).uuid
        return "GPU-" + str(u)
    except Exception:
        return None


# --------------------------------------------------------------- layer I/O --
class Layer:
    """Device-resident layer and preallocated outputs."""

    def __init__(self, seed, device, experts=EXPERTS):
        from mxfp_block_scaled_b200 import mxq, workloads
        self.mxq = mxq
        self.gu, self.dn, _ = workloads.full_moe_layer(seed=seed, device=device, experts=experts,
                                                        hidden=HIDDEN, inter=INTER)
        self.n_elems = self.gu.numel() + self.dn.numel()
        self.out = {}
        for name, x in (("gu", self.gu), ("dn", self.dn)):
            G, R, C = x.shape
            ws_q = mxq.workspace_bytes("quantize_nvfp4", G, R, C)
            if name == "gu":
                nt, rows, cols, tps = 2 * G, R // 2, C, 2
            else:
                nt, rows, cols, tps = G, R, C, 1
            ws_v = mxq.workspace_bytes("dequant_relerr", nt, rows, cols)
            self.out[name] = dict(
                x=x, G=G, R=R, C=C, nt=nt, rows=rows, cols=cols, tps=tps,
                codes=torch.empty((G, R, C // 2), dtype=torch.uint8, device=device),
                scales=torch.empty((G, R, C // 16), dtype=torch.uint8, device=device),
                s2=torch.empty(G, dtype=torch.float32, device=device),
                mbits=torch.empty((G * R * C // 16 + 31) // 32, dtype=torch.int32, device=device),
                m4=torch.empty(G, dtype=torch.int32, device=device),
                status=torch.zeros(1, dtype=torch.int32, device=device),
                wsq=torch.empty(max(ws_q, 256), dtype=torch.uint8, device=device),
                wsv=torch.empty(max(ws_v, 256), dtype=torch.uint8, device=device),
                err=torch.empty(nt, dtype=torch.float64, device=device),
                ref=torch.empty(nt, dtype=torch.float64, device=device),
                rel=torch.empty(nt, dtype=torch.float64, device=device),
            )

    def quantize(self, name):
        o = self.out[name]
        self.mxq.mxq_quantize_nvfp4(o["x"], o["G"], o["R"], o["C"], "four_six", "linear", o["codes"],
                                    o["scales"], o["s2"], o["mbits"], o["m4"], o["status"], o["wsq"])

    def verify(self, name):
        o = self.out[name]
        self.mxq.mxq_dequant_relerr(o["x"], o["codes"], o["scales"], o["s2"], "nvfp4", "linear", o["nt"],
                                    o["rows"], o["cols"], o["tps"], o["err"], o["ref"], o["rel"],
                                    o["wsv"])

    CALLS = (("quantize", "gu"), ("quantize", "dn"), ("verify", "gu"), ("verify", "dn"))

    def step(self, events=None):
        for i, (kind, name) in enumerate(self.CALLS):
            if events is not None:
                events[i][0].record()
            getattr(self, kind)(name)
            if events is not None:
                events[i][1].record()


def run_cpu_baseline(layer, budget_s=20.0):
    """The oracle as it stands, single-threaded on the host, on whole
    experts of the same layer until about budget_s of CPU work."""
    import oracle
    from mxfp_block_scaled_b200 import workloads
    oracle.build()
    n_el, t_total, experts = 0, 0.0, 0
    while t_total < budget_s and experts < EXPERTS:
        e = experts
        gu = workloads.bf16_bits(layer.gu[e:e + 1])
        dn = workloads.bf16_bits(layer.dn[e:e + 1])
        t0 = time.perf_counter()
        c, s, s2, _ = oracle.quantize_nvfp4(gu, mode=1)
        oracle.dequant_relerr(gu, c, s, s2, "nvfp4", 2, INTER, HIDDEN, 2)
        c, s, s2, _ = oracle.quantize_nvfp4(dn, mode=1)
        oracle.dequant_relerr(dn, c, s, s2, "nvfp4", 1, HIDDEN, INTER, 1)
        t_total += time.perf_counter() - t0
        n_el += gu.size + dn.size
        experts += 1
    gbs = n_el * STEP_BYTES_PER_ELEM / t_total / 1e9
    return {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": "%d of %d experts (gate_up + down, %.1fM elements), quantize + verify, "
                      "%.1f s single-threaded C" % (experts, EXPERTS, n_el / 1e6, t_total),
            "elements_per_s": n_el / t_total}


def run_e2e(layer, steps, device, chunk=64):
    """Same metric through the public Python API with host buffers: every step
    copies the layer from pinned host memory, quantizes and verifies it, and
    copies codes, scales, global scales and per-tensor errors back
    (layers.HostLayerConverter: chunks of `chunk` experts, with the copies in
    both directions overlapping the kernels of neighbouring chunks)."""
    from mxfp_block_scaled_b200 import layers
    h_gu = torch.empty(layer.gu.shape, dtype=torch.bfloat16, pin_memory=True)
    h_dn = torch.empty(layer.dn.shape, dtype=torch.bfloat16, pin_memory=True)
    h_gu.copy_(layer.gu)
    h_dn.copy_(layer.dn)
    out = layers.host_outputs(h_gu, h_dn)
    h2d = h_gu.numel() * 2 + h_dn.numel() * 2
    d2h = sum(t.numel() * t.element_size() for o in out.values() for t in o.values())
    conv = layers.HostLayerConverter(layer.gu.shape, layer.dn.shape, chunk=chunk, device=device)
    conv.run(h_gu, h_dn, out)
    torch.cuda.synchronize()
    if conv.status() != 0:
        raise RuntimeError("device status %#x in the e2e leg" % conv.status())
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        conv.run(h_gu, h_dn, out)
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    return {"value": layer.n_elems * STEP_BYTES_PER_ELEM / (ms * 1e-3) / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "pipeline": "chunks of %d experts, H2D / kernels / D2H on three streams" % chunk}


# ------------------------------------------------------------- reference --
def max_over_ranks(x, world, device):
    """The largest per-rank value over all ranks (the step time of a weak-
    scaling run is the slowest rank's).  One all-reduce of one number: the
    data path itself exchanges nothing between ranks."""
    if world <= 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_reference(args, rank, world):
    """The oracle (CPU) as the reference arm: each step converts one expert
    (gate_up + down) of the same layer shape, quantize + verify."""
    if rank != 0:
        return 0
    import oracle
    from mxfp_block_scaled_b200 import workloads
    oracle.build()
    gu, dn, _ = workloads.full_moe_layer(seed=0, device="cpu", experts=1, hidden=HIDDEN,
                                         inter=INTER)
    xg, xd = workloads.bf16_bits(gu), workloads.bf16_bits(dn)

    def step():
        c, s, s2, _ = oracle.quantize_nvfp4(xg, mode=1)
        oracle.dequant_relerr(xg, c, s, s2, "nvfp4", 2, INTER, HIDDEN, 2)
        c, s, s2, _ = oracle.quantize_nvfp4(xd, mode=1)
        oracle.dequant_relerr(xd, c, s, s2, "nvfp4", 1, HIDDEN, INTER, 1)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    n = xg.size + xd.size
    v = n * STEP_BYTES_PER_ELEM / dt / 1e9
    line = {"metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD, "sample": "one expert per step (gate_up [1,1536,2048] + "
                                                      "down [1,2048,768])"},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": "one expert per step, %d steps" % args.steps},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ main --
REQ_BYTES = 1.0 + 0.5 + 1.0 / 32    # read E4M3, write E2M1 codes + UE8M0 scales (block scales ~0)


def run_requant(args, device):
    """FP8 -> MXFP4 requantization of one full-size routed-expert layer held
    as block-FP8 (E4M3 codes + one fp32 scale per 128 x 128 block):
    gate_up [512 * 1536, 2048] and down [512 * 2048, 768]."""
    from mxfp_block_scaled_b200 import mxq, workloads
    E = args.experts
    srcs = []
    for name, rows, cols in (("gate_up", E * 2 * INTER, HIDDEN), ("down", E * HIDDEN, INTER)):
        codes = torch.empty((rows, cols), dtype=torch.uint8, device=device)
        bs = torch.empty((rows // 128, -(-cols // 128)), dtype=torch.float32, device=device)
        step = 128 * 256
        for i, r0 in enumerate(range(0, rows, step)):
            c, b = workloads.block_fp8_source(min(step, rows - r0), cols, seed=1000 + i, device=device)
            codes[r0:r0 + c.shape[0]] = c
            bs[r0 // 128:r0 // 128 + b.shape[0]] = b
        out = {"codes": torch.empty((rows, cols // 2), dtype=torch.uint8, device=device),
               "scales": torch.empty((rows, cols // 32), dtype=torch.uint8, device=device),
               "status": torch.zeros(1, dtype=torch.int32, device=device)}
        srcs.append((name, rows, cols, codes, bs, out))
    torch.cuda.synchronize()

    def step(ev=None):
        for i, (name, rows, cols, codes, bs, out) in enumerate(srcs):
            if ev is not None:
                ev[i][0].record()
            mxq.mxq_requant_fp8_mx(codes, bs, rows, cols, 128, 128, "mxfp4", "linear", out["codes"],
                                   out["scales"], out["status"])
            if ev is not None:
                ev[i][1].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for s_ in srcs:
        if int(s_[5]["status"].item()) != 0:
            raise RuntimeError("device status on " + s_[0])
    events = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
               for _ in srcs] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device_uuid()) as clk:
        torch.cuda.synchronize()
        t0.record()
        for k in range(args.steps):
            step(events[k])
        t1.record()
        torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / args.steps
    call_ms = [statistics.mean(events[k][i][0].elapsed_time(events[k][i][1]) for k in range(args.steps))
               for i in range(len(srcs))]
    n = sum(r * c for _, r, c, _, _, _ in srcs)
    peak, peak_kind = measured_peak()
    value = n * REQ_BYTES / (ms * 1e-3) / 1e9
    gu_n = srcs[0][1] * srcs[0][2]
    achieved = gu_n * REQ_BYTES / (call_ms[0] * 1e-3) / 1e9
    return {
        "metric": "FP8 -> MXFP4 requantization HBM GB/s (1 GPU)", "value": value, "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": "one full-size routed-expert layer as block FP8 (E4M3 + fp32 scale per "
                               "128x128) -> MXFP4: gate_up [512*1536, 2048] + down [512*2048, 768]",
                   "elements_per_gpu": n, "algorithmic_bytes_per_element": REQ_BYTES,
                   "l2": "inputs 2.4 GB, larger than L2; no flush",
                   "call_ms": dict(zip(["requant_gate_up", "requant_down"], call_ms))},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": None,
                     "kernel": "requant_fp8_mx_kernel<MXFP4> (gate_up)", "peak_kind": peak_kind},
        "gpu_launches": args.steps * len(srcs),
        "clocks": clk.summary(),
    }


def run_weighted(args, device):
    """NVFP4 with the weighted-SSE scale search over one full-size layer:
    gate_up [512, 1536, 2048] and down [512, 2048, 768], each with one shared
    row of per-input-channel weights (the mean squared activation of a
    synthetic 4096-token tile)."""
    from mxfp_block_scaled_b200 import mxq, workloads
    layer = Layer(seed=0, device=device, experts=args.experts)
    calls = []
    for name, x in (("gate_up", layer.gu), ("down", layer.dn)):
        G, R, C = x.shape
        a = workloads.activation_tile(4096, seed=7, device=device, hidden=C).float()
        h = (a * a).mean(0).contiguous()
        ws, _ = mxq._workspace("quantize_nvfp4", G, R, C, device)
        out = {"codes": torch.empty((G, R, C // 2), dtype=torch.uint8, device=device),
               "scales": torch.empty((G, R, C // 16), dtype=torch.uint8, device=device),
               "s2": torch.empty(G, dtype=torch.float32, device=device),
               "status": torch.zeros(1, dtype=torch.int32, device=device)}
        calls.append((name, x, h, ws, out))
    torch.cuda.synchronize()

    def step(ev=None):
        for i, (name, x, h, ws, out) in enumerate(calls):
            G, R, C = x.shape
            if ev is not None:
                ev[i][0].record()
            mxq.mxq_quantize_nvfp4_weighted(x, G, R, C, h, 1, "linear", out["codes"], out["scales"],
                                            out["s2"], out["status"], ws)
            if ev is not None:
                ev[i][1].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for c in calls:
        if int(c[4]["status"].item()) != 0:
            raise RuntimeError("device status on " + c[0])
    events = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
               for _ in calls] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device_uuid()) as clk:
        torch.cuda.synchronize()
        t0.record()
        for k in range(args.steps):
            step(events[k])
        t1.record()
        torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / args.steps
    call_ms = [statistics.mean(events[k][i][0].elapsed_time(events[k][i][1]) for k in range(args.steps))
               for i in range(len(calls))]
    n = layer.n_elems
    peak, peak_kind = measured_peak()
    gu_n = layer.gu.numel()
    achieved = gu_n * Q_BYTES / (call_ms[0] * 1e-3) / 1e9
    return {
        "metric": "NVFP4 weighted-SSE scale search, quantize HBM GB/s (1 GPU)",
        "value": n * Q_BYTES / (ms * 1e-3) / 1e9, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "one full-size routed-expert layer, NVFP4 with the weighted-SSE scale "
                               "search: gate_up bf16 [512,1536,2048] + down [512,2048,768]",
                   "elements_per_gpu": n, "algorithmic_bytes_per_element": Q_BYTES,
                   "passes": "two (group amax, then the search): W is read twice",
                   "call_ms": dict(zip(["gate_up", "down"], call_ms))},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": None,
                     "kernel": "nvfp4_weighted_kernel (gate_up; limited by its binary64 "
                               "arithmetic, not by HBM)", "peak_kind": peak_kind},
        "gpu_launches": args.steps * len(calls) * 2,
        "clocks": clk.summary(),
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="mine", choices=["mine", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the e2e and CPU-baseline legs (profiling runs)")
    ap.add_argument("--workload", default="nvfp4_layer",
                    choices=["nvfp4_layer", "fp8_requant", "nvfp4_weighted"],
                    help="nvfp4_layer: the headline quantize + verify step; fp8_requant: block-FP8 "
                         "-> MXFP4 requantization of the same layer")
    ap.add_argument("--experts", type=int, default=EXPERTS,
                    help="experts in the layer; fewer than 512 only for small profiling captures")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if args.impl == "mine" else args.warmup

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import datetime
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    device = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(device)

    from mxfp_block_scaled_b200 import build, mxq
    build.build()
    mxq.load()
    if args.workload == "fp8_requant":
        if world > 1:
            raise SystemExit("--workload fp8_requant runs on one GPU")
        print(json.dumps(run_requant(args, device)), flush=True)
        return 0
    if args.workload == "nvfp4_weighted":
        if world > 1:
            raise SystemExit("--workload nvfp4_weighted runs on one GPU")
        print(json.dumps(run_weighted(args, device)), flush=True)
        return 0

    layer = Layer(seed=rank, device=device, experts=args.experts)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        layer.step()
    barrier()
    for name in ("gu", "dn"):
        st = int(layer.out[name]["status"].item())
        if st != 0:
            raise RuntimeError("device status %#x on %s" % (st, name))

    events = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
               for _ in Layer.CALLS] for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(device_uuid()) as clk:
        barrier()
        start.record()
        for k in range(args.steps):
            layer.step(events[k])
        end.record()
        barrier()
    ms = max_over_ranks(start.elapsed_time(end) / args.steps, world, device)
    call_ms = [statistics.mean(events[k][i][0].elapsed_time(events[k][i][1]) for k in range(args.steps))
               for i in range(len(Layer.CALLS))]
    total_elems = layer.n_elems * world
    value = total_elems * STEP_BYTES_PER_ELEM / (ms * 1e-3) / 1e9
    peak, peak_kind = measured_peak()

    # dominant call: quantize of the gate_up stack
    gu_elems = layer.gu.numel()
    q_ms = call_ms[0]
    achieved = gu_elems * Q_BYTES / (q_ms * 1e-3) / 1e9
    traffic = ncu_traffic_per_launch()
    quality = {}
    for name in ("gu", "dn"):
        o = layer.out[name]
        rel = o["rel"].cpu().numpy()
        quality[name] = {"relerr_mean": float(rel.mean()), "relerr_max": float(rel.max()),
                         "m4_fraction": float(o["m4"].sum().item()) / (o["G"] * o["R"] * o["C"] / 16)}

    result = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD if args.experts == EXPERTS else
                   "PROFILING CASE, %d experts (not the headline workload)" % args.experts,
                   "experts": args.experts, "hidden": HIDDEN, "inter": INTER,
                   "elements_per_gpu": layer.n_elems, "algorithmic_bytes_per_element": STEP_BYTES_PER_ELEM,
                   "l2": "inputs 4.8 GB per GPU, larger than L2; no flush",
                   "fraction_of_peak": value / peak, "peak_gbs": peak, "peak_kind": peak_kind,
                   "fraction_of_8tbs_nominal": value / 8000.0,
                   "call_ms": dict(zip(["quantize_gate_up", "quantize_down", "verify_gate_up",
                                        "verify_down"], call_ms)),
                   "quality": quality},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "nvfp4_fused_kernel (mxq_quantize_nvfp4 on the gate_up stack)",
                     "algorithmic_bytes_per_launch": gu_elems * Q_BYTES,
                     "peak_kind": peak_kind},
        "gpu_launches": args.steps * 2 * (KERNELS_PER_QUANTIZE_NVFP4 + KERNELS_PER_VERIFY),
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_extras:
        result["e2e"] = run_e2e(layer, args.e2e_steps, device)
        result["cpu_baseline"] = run_cpu_baseline(layer, args.cpu_budget)
    elif rank == 0:
        result["e2e"] = None
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
