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
