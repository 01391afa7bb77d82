"""Host logic of the multi-GPU benchmark on CPU with two gloo ranks.

The path shards into independent units (each rank converts its own layer;
no data-path collective), so the only cross-rank steps are the barrier
around the timed region and the max over ranks of the step time; the
reference arm runs on rank 0 alone."""
import json
import os
import socket
import subprocess
import sys
import types

from conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


WORKER = r"""
import os, sys, json
sys.path.insert(0, os.environ["ROOT"])
import torch.distributed as dist
import bench
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%s" % os.environ["PORT"],
                        rank=rank, world_size=world)
dist.barrier()
m = bench.max_over_ranks(1.0 + 1.5 * rank, world, "cpu")
dist.barrier()
print(json.dumps({"rank": rank, "max": m}))
dist.destroy_process_group()
"""


def test_step_time_is_the_max_over_two_gloo_ranks():
    port = str(_free_port())
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE="2", PORT=port, ROOT=ROOT)
        procs.append(subprocess.Popen([sys.executable, "-c", WORKER], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    assert sorted(o["rank"] for o in outs) == [0, 1]
    assert all(o["max"] == 2.5 for o in outs)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import bench
    args = types.SimpleNamespace(steps=1, warmup=0, gpus=2)
    assert bench.run_reference(args, rank=1, world=2) == 0
    assert capsys.readouterr().out == ""


E2E_WORKER = r"""
import os, sys, json, types
sys.path.insert(0, os.environ["ROOT"])
import torch, torch.distributed as dist
import bench
from mxfp_block_scaled_b200 import layers
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%s" % os.environ["PORT"],
                        rank=rank, world_size=world)

# CPU stand-ins for the device pieces: rank 1 cannot pin its host buffers
real_empty = torch.empty
def empty(*a, pin_memory=False, **k):
    if pin_memory and rank == 1 and os.environ["FAIL"] == "1":
        raise RuntimeError("pinned host memory refused")
    return real_empty(*a, **k)
class Ev:
    def record(self): pass
    def elapsed_time(self, other): return 10.0
class Conv:
    def __init__(self, *a, **k): pass
    def run(self, *a): pass
    def status(self): return 0
torch.empty = empty
torch.cuda.synchronize = lambda *a: None
torch.cuda.Event = lambda enable_timing=True: Ev()
layers.HostLayerConverter = Conv
layers.host_outputs = lambda gu, dn: {}
layer = types.SimpleNamespace(gu=real_empty((2, 4, 16), dtype=torch.bfloat16),
                              dn=real_empty((2, 16, 4), dtype=torch.bfloat16), n_elems=256)
res = bench.run_e2e(layer, 2, "cpu", world=world)
dist.barrier()
print(json.dumps({"rank": rank, "res": res}))
dist.destroy_process_group()
"""


def _run_e2e_ranks(fail):
    port = str(_free_port())
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE="2", PORT=port, ROOT=ROOT, FAIL=fail)
        procs.append(subprocess.Popen([sys.executable, "-c", E2E_WORKER], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    return {o["rank"]: o["res"] for o in outs}


def test_e2e_leg_failing_on_one_rank_reports_unavailable_without_hanging():
    """The e2e leg runs on every rank; a rank that cannot set it up still
    takes part in the barrier and the max over ranks, so no rank waits for
    another and the leg reports itself unavailable."""
    res = _run_e2e_ranks("1")
    assert all("unavailable" in r for r in res.values()), res
    assert "pinned host memory refused" in res[1]["unavailable"]


def test_e2e_leg_counts_every_rank():
    """Both ranks succeed: the step time is the max over ranks (10 ms over 2
    steps) and the value counts both ranks' elements."""
    import bench
    res = _run_e2e_ranks("0")
    for r in res.values():
        assert r["ms_per_step"] == 5.0
        assert abs(r["value"] - 256 * 2 * bench.STEP_BYTES_PER_ELEM / 5e-3 / 1e9) < 1e-12
