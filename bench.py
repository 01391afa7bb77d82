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
    python bench.py --workload mxfp8_shared    # MXFP8 rewrite of 48 shared experts (dense + padded)
    python bench.py --workload mxfp4_layer     # MXFP4 quantize + verify of a full-size layer
    python bench.py --workload act_sweep       # activation tiles [T, 2048], NVFP4 and MXFP8
    python bench.py --workload mixed8          # 8 layers: NVFP4 4/6 (even) and MXFP4 (odd)
    --layout swizzled_128x4   block scales in the 128x4 tiled layout (layer and MX workloads)
    --act-mode four_six       4/6-optimal NVFP4 block scales in act_sweep

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
    """Hash of the single-pass quantizer's source: its part of nvfp4.cu (from
    the argument struct to its launch function) and the headers it uses, so
    that edits to the other kernels of that file leave the record valid."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mxfp_block_scaled_b200", "csrc")
    with open(os.path.join(csrc, "nvfp4.cu"), "rb") as fh:
        src = fh.read()
    h.update(src[src.index(b"struct FusedArgs {"):src.index(b"cudaError_t launch_nvfp4_quant(")])
    for f in ("nvfp4_block.cuh", "mxq_device.cuh", "mxq_internal.h"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _traffic_record():
    """Fields of the committed ncu traffic summary, or None when the kernel
    source changed since it was captured."""
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
        return kv
    except Exception:
        return None


def ncu_traffic_per_launch():
    """DRAM bytes (read + write) per quantize launch from the committed ncu
    summary, or None when the kernel source changed since it was captured."""
    kv = _traffic_record()
    try:
        return float(kv["dram_bytes_per_call"]) if kv else None
    except (KeyError, ValueError):
        return None


def ncu_traffic_split():
    """{"traffic_read": R, "traffic_write": W, "ncu_dram_gbs": G} per quantize
    launch from the same summary (empty when unavailable); G is the captured
    launch's DRAM bytes over its ncu duration (cold, serialised)."""
    kv = _traffic_record()
    try:
        out = {"traffic_read": float(kv["dram_read_per_call"]),
               "traffic_write": float(kv["dram_write_per_call"])} if kv else {}
        if kv and "ncu_capture_ns" in kv:
            out["ncu_dram_gbs"] = float(kv["ncu_capture_dram_bytes"]) / float(kv["ncu_capture_ns"])
        return out
    except (KeyError, ValueError, ZeroDivisionError):
        return {}


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

    def __init__(self, seed, device, experts=EXPERTS, tensors=None, layout="linear"):
        from mxfp_block_scaled_b200 import mxq, workloads
        self.mxq = mxq
        self.layout = layout
        if tensors is None:
            self.gu, self.dn, _ = workloads.full_moe_layer(seed=seed, device=device, experts=experts,
                                                            hidden=HIDDEN, inter=INTER)
        else:
            self.gu, self.dn = tensors
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
                scales=torch.empty(mxq.scale_bytes("nvfp4", layout, G, R, C), dtype=torch.uint8,
                                   device=device),
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

    def quantize(self, name, mode="four_six"):
        o = self.out[name]
        self.mxq.mxq_quantize_nvfp4(o["x"], o["G"], o["R"], o["C"], mode, self.layout, o["codes"],
                                    o["scales"], o["s2"], o["mbits"], o["m4"], o["status"], o["wsq"])

    def verify(self, name):
        o = self.out[name]
        self.mxq.mxq_dequant_relerr(o["x"], o["codes"], o["scales"], o["s2"], "nvfp4", self.layout, o["nt"],
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


def nvfp4_census(lays, with_rtn=True):
    """The census of Layer objects whose buffers hold their 4/6 results,
    formed on the device (mxq_census_add): mean / max relative error over the
    unstacked tensors and the M=4 fraction; with_rtn also SSE(chosen) /
    SSE(RTN) - 1, for which the stacks are quantized again with plain amax/6
    block scales and verified into the same buffers (so call it after
    everything that reads the 4/6 outputs).  A quality figure only: a
    failure is reported, not raised."""
    from mxfp_block_scaled_b200 import mxq
    try:
        saved = [{t: (lay.out[t]["err"].clone(), lay.out[t]["rel"].clone(), lay.out[t]["m4"].clone())
                  for t in ("gu", "dn")} for lay in lays]
        rtn = None
        if with_rtn:
            try:
                for lay in lays:
                    for t in ("gu", "dn"):
                        lay.quantize(t, mode="rtn")
                        lay.verify(t)
                torch.cuda.synchronize()
                rtn = True
            except Exception as e:
                rtn = {"unavailable": str(e)[:200]}
        c = mxq.Census(device=lays[0].gu.device)
        for lay, sv in zip(lays, saved):
            for t in ("gu", "dn"):
                o = lay.out[t]
                err, rel, m4 = sv[t]
                c.add(n_tensors=o["nt"], sum_sq_err=err, sum_sq_ref=o["ref"], relerr=rel,
                      sum_sq_err_rtn=o["err"] if rtn is True else None, n_groups=o["G"], m4_count=m4,
                      blocks_per_group=o["R"] * o["C"] // 16)
        r = c.result()
        out = {k: r[k] for k in ("mean_relerr", "max_relerr", "n_tensors", "m4_fraction")}
        if with_rtn:
            out["sse_vs_rtn"] = r["sse_vs_rtn"] if rtn is True else rtn
        return out
    except Exception as e:
        return {"unavailable": str(e)[:200]}


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


def run_cpu_parallel(layer, per_thread=3):
    """The same oracle on every host core: one thread per core (the C calls
    release the interpreter lock), each converting whole experts of the
    layer (quantize + verify), `per_thread` experts per thread, at most 512."""
    import concurrent.futures as cf
    import oracle
    from mxfp_block_scaled_b200 import workloads
    oracle.build()
    oracle.lib()                                        # load once, before the threads start
    n = min(os.cpu_count() or 1, 128)
    experts = min(EXPERTS, n * per_thread)
    work = [(workloads.bf16_bits(layer.gu[e:e + 1]), workloads.bf16_bits(layer.dn[e:e + 1]))
            for e in range(experts)]

    def one(item):
        gu, dn = item
        c, s, s2, _ = oracle.quantize_nvfp4(gu, mode=1)
        oracle.dequant_relerr(gu, c, s, s2, "nvfp4", 2, INTER, HIDDEN, 2)
        c, s, s2, _ = oracle.quantize_nvfp4(dn, mode=1)
        oracle.dequant_relerr(dn, c, s, s2, "nvfp4", 1, HIDDEN, INTER, 1)
        return gu.size + dn.size

    with cf.ThreadPoolExecutor(max_workers=n) as ex:
        t0 = time.perf_counter()
        n_el = sum(ex.map(one, work))
        t = time.perf_counter() - t0
    return {"value": n_el * STEP_BYTES_PER_ELEM / t / 1e9, "unit": "GB/s", "cores": n, "kind": "oracle",
            "sample": "%d of %d experts (gate_up + down, %.1fM elements), quantize + verify, %.1f s "
                      "on %d threads" % (experts, EXPERTS, n_el / 1e6, t, n),
            "elements_per_s": n_el / t}


def run_e2e(layer, steps, device, chunk=64, world=1):
    """Same metric through the public Python API with host buffers: every step
    copies the layer from pinned host memory, quantizes and verifies it, and
    copies codes, scales, global scales and per-tensor errors back
    (layers.HostLayerConverter: chunks of `chunk` experts, with the copies in
    both directions overlapping the kernels of neighbouring chunks).  Under
    torchrun every rank converts its own layer; the step time is the max
    over ranks and the value counts every rank's elements.  A rank that
    cannot set the leg up (e.g. pinned host memory refused) still takes part
    in the barrier and the reduction, and the leg reports itself unavailable."""
    from mxfp_block_scaled_b200 import layers
    failed, h2d, d2h = None, 0, 0
    try:
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
            failed = "device status %#x" % conv.status()
    except (RuntimeError, MemoryError) as e:
        failed = str(e).splitlines()[0][:200] if str(e) else type(e).__name__
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    ms = float("inf")
    if failed is None:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(steps):
            conv.run(h_gu, h_dn, out)
        t1.record()
        torch.cuda.synchronize()
        ms = t0.elapsed_time(t1) / steps
    ms = max_over_ranks(ms, world, device)
    if ms == float("inf"):
        return {"unavailable": "e2e leg could not run on every rank: %s" % (failed or "another rank failed")}
    return {"value": layer.n_elems * world * STEP_BYTES_PER_ELEM / (ms * 1e-3) / 1e9, "unit": "GB/s",
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
    """The oracle (CPU) as the reference arm: each step converts one expert's
    down slab [2048, 768] of the same layer (a whole NVFP4 group, the same
    per-element work as gate_up), quantize + verify, so that the default
    200 steps end in about two minutes."""
    if rank != 0:
        return 0
    import oracle
    from mxfp_block_scaled_b200 import workloads
    oracle.build()
    _, dn, _ = workloads.full_moe_layer(seed=0, device="cpu", experts=1, hidden=HIDDEN,
                                         inter=INTER)
    xd = workloads.bf16_bits(dn)

    def step():
        c, s, s2, _ = oracle.quantize_nvfp4(xd, mode=1)
        oracle.dequant_relerr(xd, c, s, s2, "nvfp4", 1, HIDDEN, INTER, 1)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    n = xd.size
    v = n * STEP_BYTES_PER_ELEM / dt / 1e9
    line = {"metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD, "sample": "one expert's down slab per step ([1,2048,768], "
                                                      "quantize + verify)"},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": "one expert's down slab per step, %d steps" % args.steps},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------- other workloads --
REQ_BYTES = 1.0 + 0.5 + 1.0 / 32    # read E4M3, write E2M1 codes + UE8M0 scales (block scales ~0)


def run_requant(args, device):
    """FP8 -> MXFP4 requantization of one full-size routed-expert layer held
    as block-FP8 (E4M3 codes + one fp32 scale per 128 x 128 block):
    gate_up [512 * 1536, 2048] and down [512 * 2048, 768]."""
    from mxfp_block_scaled_b200 import mxq, workloads
    E = args.experts
    srcs = []
    for name, rows, cols in (("gate_up", E * 2 * INTER, HIDDEN), ("down", E * HIDDEN, INTER)):
        codes, bs = workloads.block_fp8_stack(rows, cols, device=device)
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
        "config": {"workload": ("one full-size routed-expert layer as block FP8 (E4M3 + fp32 scale per "
                                "128x128) -> MXFP4: gate_up [512*1536, 2048] + down [512*2048, 768]")
                   if args.experts == EXPERTS else
                   "PROFILING CASE, %d experts (not the full-size layer)" % args.experts,
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
        "vs_baseline": None, "dtype": "f32+f64", "data": "synthetic",
        "config": {"workload": ("one full-size routed-expert layer, NVFP4 with the weighted-SSE scale "
                                "search: gate_up bf16 [512,1536,2048] + down [512,2048,768]")
                   if args.experts == EXPERTS else
                   "PROFILING CASE, %d experts (not the full-size layer)" % args.experts,
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


def time_calls(calls, steps, warmup):
    """CUDA-event timing of `steps` passes over `calls` (callables issuing
    device work on the current stream) after `warmup` passes: mean step
    time, each call's mean time (ms) and the clock samples of the timed
    region."""
    for _ in range(warmup):
        for c in calls:
            c()
    torch.cuda.synchronize()
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in calls]
          for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device_uuid()) as clk:
        torch.cuda.synchronize()
        t0.record()
        for k in range(steps):
            for i, c in enumerate(calls):
                ev[k][i][0].record()
                c()
                ev[k][i][1].record()
        t1.record()
        torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    call_ms = [statistics.mean(ev[k][i][0].elapsed_time(ev[k][i][1]) for k in range(steps))
               for i in range(len(calls))]
    return ms, call_ms, clk.summary()


MX_BYTES = {"mxfp8": 2.0 + 1.0 + 1.0 / 32, "mxfp4": 2.0 + 0.5 + 1.0 / 32}   # per element, each pass


class MXStack:
    """One stack of equally shaped tensors, quantized to MX as a single
    [rows, cols] matrix (MX scales are per 32 values: no per-tensor state)
    and verified per tensor of `trows` rows."""

    def __init__(self, mxq, x2d, fmt, trows, device, layout="linear"):
        self.mxq, self.x, self.fmt, self.trows, self.layout = mxq, x2d, fmt, trows, layout
        self.R, self.C = x2d.shape
        self.nt = self.R // trows
        self.codes = torch.empty((self.R, self.C if fmt == "mxfp8" else self.C // 2), dtype=torch.uint8,
                                 device=device)
        self.scales = torch.empty(mxq.scale_bytes(fmt, layout, 1, self.R, self.C), dtype=torch.uint8,
                                  device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        ws = mxq.workspace_bytes("dequant_relerr", self.nt, trows, self.C)
        self.wsv = torch.empty(max(ws, 256), dtype=torch.uint8, device=device)
        self.err, self.ref, self.rel = (torch.empty(self.nt, dtype=torch.float64, device=device)
                                        for _ in range(3))

    def quantize(self):
        self.mxq.mxq_quantize_mx(self.x, self.R, self.C, self.fmt, 32, self.layout, self.codes, self.scales,
                                 self.status)

    def verify(self):
        # tiled: the stack was quantized as one matrix, so all its tensors share one scale matrix
        tps = 1 if self.layout == "linear" else self.nt
        self.mxq.mxq_dequant_relerr(self.x, self.codes, self.scales, None, self.fmt, self.layout, self.nt,
                                    self.trows, self.C, tps, self.err, self.ref, self.rel, self.wsv)


def mx_cpu_baseline(stacks, fmt, budget_s=15.0):
    """The oracle as it stands (single-threaded C) on whole tensors of the
    same stacks, quantize + verify, until about budget_s of CPU work."""
    import oracle
    from mxfp_block_scaled_b200 import workloads
    oracle.build()
    n_el, t_total, done = 0, 0.0, 0
    for k in range(max(s.nt for s in stacks)):
        for s in stacks:
            if k >= s.nt or t_total >= budget_s:
                continue
            xb = workloads.bf16_bits(s.x[k * s.trows:(k + 1) * s.trows])
            t0 = time.perf_counter()
            c, sc = oracle.quantize_mx(xb, fmt)
            oracle.dequant_relerr(xb, c, sc, None, fmt, 1, s.trows, s.C, 1)
            t_total += time.perf_counter() - t0
            n_el += xb.size
            done += 1
        if t_total >= budget_s:
            break
    return {"value": n_el * 2 * MX_BYTES[fmt] / t_total / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": "%d tensors (%.1fM elements), %s quantize + verify, %.1f s single-threaded C"
                      % (done, n_el / 1e6, fmt, t_total), "elements_per_s": n_el / t_total}


def run_mx(args, device):
    """MX quantize + verify.  mxfp8_shared: the shared-expert MXFP8 rewrite,
    48 layers x {dense, MTP-style padded} of gate/up [2560, 2048] and down
    [2048, 1280]; mxfp4_layer: one full-size routed-expert layer
    [512, 1536, 2048] + [512, 2048, 768] with the Student-t tail mix, as the
    MXFP4 layers of the mixed-format conversion."""
    from mxfp_block_scaled_b200 import mxq, workloads
    if args.workload == "mxfp8_shared":
        fmt, layers = "mxfp8", 48
        gus, dns = [], []
        for L in range(layers):
            for padded in (False, True):
                gu, dn = workloads.shared_expert_layer(seed=L, device=device, padded=padded)
                gus.append(gu)
                dns.append(dn)
        GU, DN = torch.stack(gus), torch.stack(dns)
        del gus, dns
        stacks = [MXStack(mxq, GU.view(-1, GU.shape[-1]), fmt, GU.shape[1] // 2, device, args.layout),
                  MXStack(mxq, DN.view(-1, DN.shape[-1]), fmt, DN.shape[1], device, args.layout)]
        workload = ("shared-expert MXFP8 rewrite, quantize + verify: 48 layers x {dense, padded} of "
                    "gate/up bf16 [2560,2048] + down [2048,1280] (gate and up verified separately)")
        check_pad = True
    else:
        fmt = "mxfp4"
        GU, DN = workloads.student_t_mix_layer(seed=0, device=device, experts=args.experts)
        stacks = [MXStack(mxq, GU.view(-1, GU.shape[-1]), fmt, GU.shape[1] // 2, device, args.layout),
                  MXStack(mxq, DN.view(-1, DN.shape[-1]), fmt, DN.shape[1], device, args.layout)]
        workload = ("one full-size routed-expert layer (Student-t tail mix), MXFP4 quantize + verify: "
                    "gate_up bf16 [%d,1536,2048] + down [%d,2048,768]" % (args.experts, args.experts))
        check_pad = False
    torch.cuda.synchronize()
    calls = [s.quantize for s in stacks] + [s.verify for s in stacks]
    ms, call_ms, clocks = time_calls(calls, args.steps, args.warmup)
    for s in stacks:
        if int(s.status.item()) != 0:
            raise RuntimeError("device status %#x" % int(s.status.item()))
    if check_pad:
        # the padded copies (odd stack entries) must quantize to exact zeros, codes and scale
        # bytes: gate rows [640, 1280) and up rows [1920, 2560) of gate/up, columns [640, 1280)
        # of down
        # (value codes in every layout; scale bytes where they are linear)
        cg = stacks[0].codes.view(GU.shape[0], GU.shape[1], -1)[1::2]
        cd = stacks[1].codes.view(DN.shape[0], DN.shape[1], -1)[1::2]
        zero = [cg[:, 640:1280], cg[:, 1920:], cd[:, :, 640:]]
        if args.layout == "linear":
            sg = stacks[0].scales.view(GU.shape[0], GU.shape[1], -1)[1::2]
            sd = stacks[1].scales.view(DN.shape[0], DN.shape[1], -1)[1::2]
            zero += [sg[:, 640:1280], sg[:, 1920:], sd[:, :, 20:]]
        if any(int(z.count_nonzero()) for z in zero):
            raise RuntimeError("padded regions did not quantize to zeros")
    n = sum(s.R * s.C for s in stacks)
    bpe = 2 * MX_BYTES[fmt]
    peak, peak_kind = measured_peak()
    value = n * bpe / (ms * 1e-3) / 1e9
    gu_n = stacks[0].R * stacks[0].C
    achieved = gu_n * MX_BYTES[fmt] / (call_ms[0] * 1e-3) / 1e9
    rel = torch.cat([s.rel for s in stacks]).cpu().numpy()
    names = ["quantize_gate_up", "quantize_down", "verify_gate_up", "verify_down"]
    result = {
        "metric": "%s quantize+verify HBM GB/s (1 GPU)" % fmt.upper(), "value": value, "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": workload, "scale_layout": args.layout, "elements_per_gpu": n,
                   "algorithmic_bytes_per_element": bpe,
                   "l2": "inputs %.1f GB, larger than L2; no flush" % (n * 2 / 1e9),
                   "fraction_of_peak": value / peak, "peak_gbs": peak, "peak_kind": peak_kind,
                   "call_ms": dict(zip(names, call_ms)),
                   "quality": {"relerr_mean": float(rel.mean()), "relerr_max": float(rel.max()),
                               "tensors": int(rel.size)}},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": None,
                     "kernel": "mx_quant_kernel<%s> (gate_up stack)" % fmt.upper(),
                     "algorithmic_bytes_per_launch": gu_n * MX_BYTES[fmt], "peak_kind": peak_kind},
        "gpu_launches": args.steps * (2 + 2 * KERNELS_PER_VERIFY),
        "clocks": clocks,
    }
    if not args.no_extras:
        result["cpu_baseline"] = mx_cpu_baseline(stacks, fmt, args.cpu_budget)
    return result


# Layer formats of the mixed-format conversion: layers 0, 2, 4, 6 NVFP4
# 4/6-optimal, layers 1, 3, 5, 7 MXFP4 (each with its verifier pass).
MIXED_FORMATS = ("nvfp4", "mxfp4") * 4


def mixed_bytes_per_layer(fmt, n_elems):
    """Algorithmic bytes of one layer's quantize + verify."""
    return n_elems * (STEP_BYTES_PER_ELEM if fmt == "nvfp4" else 2 * MX_BYTES[fmt])


def run_mixed8(args, device):
    """Mixed-format conversion of eight full-size routed-expert layers, values
    N(0, 0.02) with the Student-t(4) tail mix: every layer quantized (NVFP4
    4/6-optimal or MXFP4 by MIXED_FORMATS) and verified over all its unstacked
    tensors, all eight layers resident in HBM (38.7 GB of bf16 inputs)."""
    from mxfp_block_scaled_b200 import mxq, workloads
    calls, names, nv, mx = [], [], [], []
    n_total, bytes_total = 0, 0.0
    for L, fmt in enumerate(MIXED_FORMATS):
        gu, dn = workloads.student_t_mix_layer(seed=L, device=device, experts=args.experts)
        n = gu.numel() + dn.numel()
        if fmt == "nvfp4":
            lay = Layer(seed=L, device=device, experts=args.experts, tensors=(gu, dn), layout=args.layout)
            nv.append(lay)
            calls += [(lambda lay=lay, k=k, t=t: getattr(lay, k)(t)) for k, t in Layer.CALLS]
        else:
            st = [MXStack(mxq, gu.view(-1, gu.shape[-1]), fmt, gu.shape[1] // 2, device, args.layout),
                  MXStack(mxq, dn.view(-1, dn.shape[-1]), fmt, dn.shape[1], device, args.layout)]
            mx.append(st)
            calls += [st[0].quantize, st[1].quantize, st[0].verify, st[1].verify]
        names += ["L%d_%s_%s" % (L, k, t) for k, t in Layer.CALLS]
        n_total += n
        bytes_total += mixed_bytes_per_layer(fmt, n)
    torch.cuda.synchronize()
    ms, call_ms, clocks = time_calls(calls, args.steps, args.warmup)
    for lay in nv:
        for t in ("gu", "dn"):
            if int(lay.out[t]["status"].item()) != 0:
                raise RuntimeError("device status %#x" % int(lay.out[t]["status"].item()))
    for st in mx:
        for s in st:
            if int(s.status.item()) != 0:
                raise RuntimeError("device status %#x" % int(s.status.item()))
    peak, peak_kind = measured_peak()
    value = bytes_total / (ms * 1e-3) / 1e9
    # dominant kernel: the NVFP4 gate_up quantize launch (call 0 of each NVFP4 layer)
    q_ms = statistics.mean(call_ms[4 * L] for L, f in enumerate(MIXED_FORMATS) if f == "nvfp4")
    gu_elems = nv[0].gu.numel()
    achieved = gu_elems * Q_BYTES / (q_ms * 1e-3) / 1e9
    traffic = ncu_traffic_per_launch() if args.experts == EXPERTS and args.layout == "linear" else None
    rel_mx = torch.cat([s.rel for st in mx for s in st]).cpu().numpy()
    # after the timed region: the census of the NVFP4 layers, and (not in
    # profiling runs) those layers again with RTN scales for SSE vs RTN
    nv_census = nvfp4_census(nv, with_rtn=not args.no_extras)
    workload = ("mixed-format conversion of 8 full-size routed-expert layers (Student-t tail mix), "
                "quantize + verify: layers 0,2,4,6 NVFP4 4/6-optimal, layers 1,3,5,7 MXFP4; each "
                "gate_up bf16 [%d,1536,2048] + down [%d,2048,768]" % (args.experts, args.experts))
    result = {
        "metric": "mixed-format NVFP4 4/6 + MXFP4 quantize+verify HBM GB/s (1 GPU)", "value": value,
        "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": workload if args.experts == EXPERTS else
                   "PROFILING CASE, %d experts per layer (not the full-size workload)" % args.experts,
                   "layers": len(MIXED_FORMATS), "formats": list(MIXED_FORMATS), "scale_layout": args.layout,
                   "elements_per_gpu": n_total, "algorithmic_bytes_per_step": bytes_total,
                   "l2": "inputs %.1f GB, larger than L2; no flush" % (n_total * 2 / 1e9),
                   "fraction_of_peak": value / peak, "peak_gbs": peak, "peak_kind": peak_kind,
                   "call_ms": dict(zip(names, call_ms)),
                   "quality": {"nvfp4": nv_census,
                               "mxfp4": {"relerr_mean": float(rel_mx.mean()), "relerr_max": float(rel_mx.max()),
                                         "tensors": int(rel_mx.size)}}},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "traffic_note": "DRAM bytes of the same kernel on the same shape (routed-layer values); "
                                     "its traffic does not depend on the values",
                     "kernel": "nvfp4_fused_kernel (gate_up stacks of the NVFP4 layers)",
                     "algorithmic_bytes_per_launch": gu_elems * Q_BYTES, "peak_kind": peak_kind},
        "gpu_launches": args.steps * sum(
            2 * (KERNELS_PER_QUANTIZE_NVFP4 + KERNELS_PER_VERIFY) if f == "nvfp4" else 2 + 2 * KERNELS_PER_VERIFY
            for f in MIXED_FORMATS),
        "clocks": clocks,
    }
    if not args.no_extras:
        a = run_cpu_baseline(nv[0], args.cpu_budget / 2)
        b = mx_cpu_baseline(mx[0], "mxfp4", args.cpu_budget / 2)
        # CPU time of one step at the two measured element rates
        t_step = sum((lay.n_elems / a["elements_per_s"]) for lay in nv) + \
            sum(sum(s.R * s.C for s in st) / b["elements_per_s"] for st in mx)
        result["cpu_baseline"] = {"value": bytes_total / t_step / 1e9, "unit": "GB/s", "cores": 1,
                                  "kind": "oracle",
                                  "sample": "NVFP4: %s; MXFP4: %s; combined at the step's element mix"
                                            % (a["sample"], b["sample"])}
    return result


def time_loop(call, reps, warmup):
    """Mean time (us) of `reps` back-to-back calls on the current stream,
    CUDA events around the whole loop, and the clock samples."""
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device_uuid()) as clk:
        torch.cuda.synchronize()
        t0.record()
        for _ in range(reps):
            call()
        t1.record()
        torch.cuda.synchronize()
    return t0.elapsed_time(t1) * 1e3 / reps, clk.summary()


def time_graph(call, reps):
    """Mean device time (us) per call of `reps` calls captured in one CUDA
    graph (no host launch cost), or None where the capture is refused."""
    try:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            call()
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                call()
        g.replay()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        g.replay()
        t1.record()
        torch.cuda.synchronize()
        del g
        return t0.elapsed_time(t1) * 1e3 / reps
    except Exception as e:   # capture refused: report the stream timing only
        log("graph capture:", e)
        torch.cuda.synchronize()
        return None


ACT_T = (1, 16, 256, 4096, 65536)
ACT_BYTES = {"nvfp4": 2.0 + 0.5 + 1.0 / 16, "mxfp8": 2.0 + 1.0 + 1.0 / 32}   # quantize only


def run_act(args, device):
    """Dynamic activation quantization of token tiles [T, 2048] (N(0, 1),
    four outlier channels x 30): NVFP4 (input_scale = amax/2688, amax/6
    block scales, or the 4/6-optimal rule with --act-mode four_six) and
    MXFP8, each T timed as back-to-back calls on one
    stream (the latency of a call in a stream of calls)."""
    from mxfp_block_scaled_b200 import mxq, workloads
    H = HIDDEN
    sweep, launches = {}, 0
    clocks = None
    for T in ACT_T:
        x = workloads.activation_tile(T, seed=T, device=device)
        for fmt in ("nvfp4", "mxfp8"):
            blk = 16 if fmt == "nvfp4" else 32
            codes = torch.empty((T, H if fmt == "mxfp8" else H // 2), dtype=torch.uint8, device=device)
            scales = torch.empty(mxq.scale_bytes(fmt, args.layout, 1, T, H), dtype=torch.uint8, device=device)
            isc = torch.empty(1, dtype=torch.float32, device=device)
            st = torch.zeros(1, dtype=torch.int32, device=device)
            ws, _ = mxq._workspace("quantize_act", T, H, 0, device)
            mode = args.act_mode if fmt == "nvfp4" else "rtn"

            def call(x=x, fmt=fmt, codes=codes, scales=scales, isc=isc, st=st, ws=ws, T=T, mode=mode):
                mxq.mxq_quantize_act(x, T, H, fmt, mode, args.layout, codes, scales, isc, st, ws)

            reps = 2000 if T <= 256 else (400 if T <= 4096 else 50)
            us, clk = time_loop(call, reps, max(args.warmup, 3))
            us_graph = time_graph(call, reps)
            if int(st.item()) != 0:
                raise RuntimeError("device status %#x (T=%d, %s)" % (int(st.item()), T, fmt))
            best = min(us, us_graph) if us_graph is not None else us
            sweep["%s_T%d" % (fmt, T)] = {"us_per_call": us, "us_per_call_graph": us_graph,
                                          "gbs": T * H * ACT_BYTES[fmt] / (best * 1e-6) / 1e9}
            launches += reps
            if T == ACT_T[-1] and fmt == "nvfp4":
                clocks = clk
        del x
    peak, peak_kind = measured_peak()
    top = sweep["nvfp4_T%d" % ACT_T[-1]]
    n_top = ACT_T[-1] * H
    result = {
        "metric": "dynamic activation quantization GB/s, NVFP4 at T=65536 (1 GPU)",
        "value": top["gbs"], "unit": "GB/s", "n_gpus": 1, "steps": 1, "warmup": max(args.warmup, 3),
        "ms_per_step": n_top * ACT_BYTES["nvfp4"] / (top["gbs"] * 1e9) * 1e3, "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "token tiles bf16 [T,2048], T in {1,16,256,4096,65536}, N(0,1) with "
                               "channels 101/717/1333/1949 x30; NVFP4 (%s block scales, "
                               "input_scale = amax/2688) and MXFP8" %
                               ("RTN" if args.act_mode == "rtn" else "4/6-optimal"),
                   "nvfp4_scale_mode": args.act_mode, "scale_layout": args.layout,
                   "algorithmic_bytes_per_element": ACT_BYTES,
                   "l2": "T=65536 tile 268 MB, larger than L2; smaller tiles are L2-resident by design",
                   "sweep": sweep, "peak_gbs": peak, "peak_kind": peak_kind},
        "roofline": {"bound": "hbm", "achieved": top["gbs"], "peak": peak, "unit": "GB/s",
                     "frac": top["gbs"] / peak, "traffic": None,
                     "kernel": "mxq_quantize_act NVFP4 at T=65536 (group_amax_kernel + nvfp4_quant_kernel: "
                               "the tile is read twice, so the ceiling is 2.5625/4.5625 of the peak)",
                     "algorithmic_bytes_per_launch": n_top * ACT_BYTES["nvfp4"], "peak_kind": peak_kind},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if not args.no_extras:
        import oracle
        oracle.build()
        x = workloads.activation_tile(4096, seed=4096, device="cpu")
        xb = workloads.bf16_bits(x).reshape(1, 4096, H)
        n_el, t = 0, 0.0
        while t < args.cpu_budget / 2:
            t0 = time.perf_counter()
            oracle.quantize_nvfp4(xb, mode=0 if args.act_mode == "rtn" else 1)
            t += time.perf_counter() - t0
            n_el += xb.size
        result["cpu_baseline"] = {"value": n_el * ACT_BYTES["nvfp4"] / t / 1e9, "unit": "GB/s", "cores": 1,
                                  "kind": "oracle",
                                  "sample": "the T=4096 tile, NVFP4 quantize repeated for %.1f s "
                                            "single-threaded C" % t,
                                  "elements_per_s": n_el / t}
    return result


# ------------------------------------------------------------------ main --
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
                    choices=["nvfp4_layer", "fp8_requant", "nvfp4_weighted", "mxfp8_shared",
                             "mxfp4_layer", "act_sweep", "mixed8"],
                    help="nvfp4_layer: the headline quantize + verify step; fp8_requant: block-FP8 "
                         "-> MXFP4 requantization of the same layer; nvfp4_weighted: weighted-SSE "
                         "scale search; mxfp8_shared / mxfp4_layer: MX quantize + verify; act_sweep: "
                         "dynamic activation quantization over T; mixed8: 8 layers, NVFP4 4/6 and "
                         "MXFP4 alternating, quantize + verify")
    ap.add_argument("--layout", default="linear", choices=["linear", "swizzled_128x4"],
                    help="block-scale layout written by the quantizers and read by the verifier "
                         "(nvfp4_layer, mixed8, mxfp8_shared, mxfp4_layer)")
    ap.add_argument("--act-mode", default="rtn", choices=["rtn", "four_six"],
                    help="NVFP4 block-scale rule of the act_sweep workload")
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
    if args.workload in ("mxfp8_shared", "mxfp4_layer", "act_sweep", "mixed8"):
        if world > 1:
            raise SystemExit("--workload %s runs on one GPU" % args.workload)
        run = {"act_sweep": run_act, "mixed8": run_mixed8}.get(args.workload, run_mx)
        print(json.dumps(run(args, device)), flush=True)
        return 0

    layer = Layer(seed=rank, device=device, experts=args.experts, layout=args.layout)
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
    traffic = ncu_traffic_per_launch() if args.layout == "linear" else None
    # census of the layer's 1536 tensors, after the timed region; SSE(chosen) / SSE(RTN) - 1
    # (an RTN pass) is skipped by profiling runs, whose launch lists cover the measured step alone
    quality = nvfp4_census([layer], with_rtn=not args.no_extras)

    result = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": (WORKLOAD + ("" if args.layout == "linear" else
                                            "; block scales in the 128x4 tiled layout"))
                   if args.experts == EXPERTS else
                   "PROFILING CASE, %d experts (not the headline workload)" % args.experts,
                   "experts": args.experts, "hidden": HIDDEN, "inter": INTER, "scale_layout": args.layout,
                   "elements_per_gpu": layer.n_elems, "algorithmic_bytes_per_element": STEP_BYTES_PER_ELEM,
                   "l2": "inputs 4.8 GB per GPU, larger than L2; no flush",
                   "fraction_of_peak": value / peak, "peak_gbs": peak, "peak_kind": peak_kind,
                   "fraction_of_8tbs_nominal": value / 8000.0,
                   "call_ms": dict(zip(["quantize_gate_up", "quantize_down", "verify_gate_up",
                                        "verify_down"], call_ms)),
                   # algorithmic GB/s of every call of the step and its fraction of the peak
                   "call_gbs": {k: {"gbs": by / (t * 1e-3) / 1e9, "frac": by / (t * 1e-3) / 1e9 / peak}
                                for k, by, t in zip(["quantize_gate_up", "quantize_down", "verify_gate_up",
                                                     "verify_down"],
                                                    [gu_elems * Q_BYTES, layer.dn.numel() * Q_BYTES,
                                                     gu_elems * V_BYTES, layer.dn.numel() * V_BYTES],
                                                    call_ms)},
                   "quality": quality},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     **(ncu_traffic_split() if traffic is not None else {}),
                     "kernel": "nvfp4_fused_kernel (mxq_quantize_nvfp4 on the gate_up stack)",
                     "algorithmic_bytes_per_launch": gu_elems * Q_BYTES,
                     "peak_kind": peak_kind},
        "gpu_launches": args.steps * 2 * (KERNELS_PER_QUANTIZE_NVFP4 + KERNELS_PER_VERIFY),
        "clocks": clk.summary(),
    }
    if not args.no_extras:
        e2e = run_e2e(layer, args.e2e_steps, device, world=world)    # every rank: collectives inside
        if rank == 0:
            result["e2e"] = e2e
        if rank == 0 and world == 1:
            result["cpu_baseline"] = run_cpu_baseline(layer, args.cpu_budget)
            result["cpu_baseline_all_cores"] = run_cpu_parallel(layer)
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
