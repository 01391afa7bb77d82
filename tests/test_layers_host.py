"""Layer statistics (mxfp_block_scaled_b200/layers.py) without a GPU: the
census figures are formed by the library (mxq_census_add); here a stand-in
for the device census checks what layers.census hands it per stack: the
verifier's per-tensor arrays, the RTN counterparts, and the M=4 counts with
their block counts (NVFP4 stacks only)."""
import torch

from mxfp_block_scaled_b200 import layers, mxq


class RecordingCensus:
    last = None

    def __init__(self, device=None, stream=None):
        self.adds = []
        RecordingCensus.last = self

    def add(self, **kw):
        self.adds.append(kw)

    def result(self):
        return {"mean_relerr": 0.0, "max_relerr": 0.0, "n_tensors": 0, "sse_vs_rtn": 0.0,
                "m4_fraction": 0.0}


def _stack(fmt, E, rows, cols, nt):
    s = {"fmt": fmt, "sum_sq_err": torch.arange(nt, dtype=torch.float64),
         "sum_sq_ref": torch.ones(nt, dtype=torch.float64), "relerr": torch.zeros(nt, dtype=torch.float64),
         "codes": torch.zeros((E, rows, cols if fmt == "mxfp8" else cols // 2), dtype=torch.uint8)}
    if fmt == "nvfp4":
        s["m4_count"] = torch.arange(E, dtype=torch.int32)
    return s


def test_census_marshalling(monkeypatch):
    monkeypatch.setattr(mxq, "Census", RecordingCensus)
    nv = {"gate_up": _stack("nvfp4", 2, 8, 32, 4), "down": _stack("nvfp4", 2, 16, 16, 2)}
    rtn = {"gate_up": _stack("nvfp4", 2, 8, 32, 4), "down": _stack("nvfp4", 2, 16, 16, 2)}
    mx = {"gate_up": _stack("mxfp8", 2, 8, 32, 4), "down": _stack("mxfp8", 2, 16, 32, 2)}
    layers.census([nv], [rtn])
    adds = RecordingCensus.last.adds
    assert [a["n_tensors"] for a in adds] == [4, 2]
    assert adds[0]["sum_sq_err"] is nv["gate_up"]["sum_sq_err"]
    assert adds[0]["sum_sq_err_rtn"] is rtn["gate_up"]["sum_sq_err"]
    assert adds[1]["sum_sq_err_rtn"] is rtn["down"]["sum_sq_err"]
    # gate_up: 8 rows x 32 cols = 16 blocks per expert; down: 16 x 16 = 16
    assert [(a["n_groups"], a["blocks_per_group"]) for a in adds] == [(2, 16), (2, 16)]
    assert adds[0]["m4_count"] is nv["gate_up"]["m4_count"]
    layers.census([mx])
    adds = RecordingCensus.last.adds
    assert [(a["n_groups"], a["m4_count"], a["sum_sq_err_rtn"]) for a in adds] == [(0, None, None)] * 2
