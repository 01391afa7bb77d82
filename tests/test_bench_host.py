"""Host-side logic of bench.py that the reported numbers depend on, checked
without a GPU: the clock-sample summary (median loaded clock, throttle
reasons of the right GPU only) and the DRAM traffic record (used only while
the kernel source it was captured from is unchanged)."""
import os

import bench


def _write(tmp_path, lines):
    p = tmp_path / "clocks.csv"
    p.write_text("\n".join(lines) + "\n")
    return str(p)


def test_clock_summary_median_and_reasons(tmp_path):
    rows = [
        # index, uuid, sm, max, power, active, hw_slowdown, hw_thermal, sw_thermal, sw_power_cap
        "0, GPU-a, 1965, 1965, 800, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, GPU-a, 1950, 1965, 990, 0x4, Not Active, Not Active, Not Active, Active",
        "0, GPU-a, 1965, 1965, 900, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, GPU-a, 300, 1965, 100, 0x0, Not Active, Not Active, Not Active, Not Active",  # idle tail
        "1, GPU-b, 900, 1965, 400, 0x8, Active, Not Active, Not Active, Not Active",      # other GPU
    ]
    s = bench.ClockSampler("GPU-a")
    s.path = _write(tmp_path, rows)
    out = s.summary()
    assert out["sm_max_mhz"] == 1965.0
    assert out["sm_mhz"] == 1965.0              # median of the loaded samples (> half the max)
    assert out["reasons"] == ["sw_power_cap"]   # GPU-b's hw_slowdown is not ours
    assert out["samples"] == 4
    assert not os.path.exists(s.path)


def test_clock_summary_without_samples(tmp_path):
    s = bench.ClockSampler("GPU-a")
    s.path = _write(tmp_path, ["garbage"])
    assert s.summary() is None


def test_traffic_record_follows_the_kernel_source(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    rec = prof / "nvfp4_quant_gate_up_fullsize_traffic.txt"
    sha = bench.kernel_source_sha()
    rec.write_text("# comment\nsource_sha %s\ndram_bytes_per_call 1234\n" % sha)
    real_join = os.path.join

    def join(*parts):
        if len(parts) >= 3 and parts[1] == "profiles":
            return real_join(str(tmp_path), *parts[1:])
        return real_join(*parts)

    monkeypatch.setattr(bench.os.path, "join", join)
    assert bench.ncu_traffic_per_launch() == 1234.0
    rec.write_text("source_sha 0000000000000000\ndram_bytes_per_call 1234\n")
    assert bench.ncu_traffic_per_launch() is None


def test_algorithmic_bytes_per_element():
    assert bench.Q_BYTES == 2.5625 and bench.STEP_BYTES_PER_ELEM == 5.125
    assert bench.MX_BYTES == {"mxfp8": 3.03125, "mxfp4": 2.53125}
    assert bench.ACT_BYTES["nvfp4"] == 2.5625


def test_mixed_format_layers_and_bytes():
    # layers 0, 2, 4, 6 NVFP4 4/6-optimal, layers 1, 3, 5, 7 MXFP4
    assert bench.MIXED_FORMATS == ("nvfp4", "mxfp4", "nvfp4", "mxfp4", "nvfp4", "mxfp4", "nvfp4", "mxfp4")
    n = 512 * 1536 * 2048 + 512 * 2048 * 768
    step = sum(bench.mixed_bytes_per_layer(f, n) for f in bench.MIXED_FORMATS)
    assert step == 4 * n * (5.125 + 5.0625)          # about 98.45 GB per step


class FakeCensus:
    """Stands in for mxq.Census on the CPU: keeps the arrays each add() got,
    so the test sees which buffers the bench hands to the census."""
    made = []

    def __init__(self, device=None, stream=None):
        self.adds = []
        FakeCensus.made.append(self)

    def add(self, **kw):
        self.adds.append({k: (v.clone() if hasattr(v, "clone") else v) for k, v in kw.items()})

    def result(self):
        err = sum(float(a["sum_sq_err"].sum()) for a in self.adds)
        rtn = [a["sum_sq_err_rtn"] for a in self.adds]
        return {"mean_relerr": 0.0, "max_relerr": 0.0, "n_tensors": sum(a["n_tensors"] for a in self.adds),
                "m4_fraction": 0.0,
                "sse_vs_rtn": (err / sum(float(r.sum()) for r in rtn) - 1.0) if all(r is not None for r in rtn)
                else float("nan")}


def test_census_pass(monkeypatch):
    import torch
    from mxfp_block_scaled_b200 import mxq
    monkeypatch.setattr(bench.torch.cuda, "synchronize", lambda *a: None)
    monkeypatch.setattr(mxq, "Census", FakeCensus)

    class FakeLayer:
        """err holds the 4/6 sums until the RTN quantize + verify rewrites them."""
        def __init__(self, e46, ertn):
            self.gu = torch.zeros(1)
            self.out = {t: {"err": torch.tensor(e46[t], dtype=torch.float64),
                            "ref": torch.ones(len(e46[t]), dtype=torch.float64),
                            "rel": torch.zeros(len(e46[t]), dtype=torch.float64),
                            "m4": torch.tensor([1], dtype=torch.int32), "nt": len(e46[t]), "G": 1,
                            "R": 4, "C": 16} for t in ("gu", "dn")}
            self.ertn, self.mode = ertn, None

        def quantize(self, t, mode="four_six"):
            self.mode = mode

        def verify(self, t):
            assert self.mode == "rtn"
            self.out[t]["err"] = torch.tensor(self.ertn[t], dtype=torch.float64)

    a = FakeLayer({"gu": [1.0, 2.0], "dn": [1.0]}, {"gu": [2.0, 2.0], "dn": [4.0]})
    b = FakeLayer({"gu": [0.5], "dn": [0.5]}, {"gu": [1.0], "dn": [1.0]})
    r = bench.nvfp4_census([a, b])
    assert abs(r["sse_vs_rtn"] - (5.0 / 10.0 - 1.0)) < 1e-15
    c = FakeCensus.made[-1]
    # the 4/6 error sums were saved before the RTN pass rewrote the buffers
    assert [a_["sum_sq_err"].tolist() for a_ in c.adds] == [[1.0, 2.0], [1.0], [0.5], [0.5]]
    assert [a_["sum_sq_err_rtn"].tolist() for a_ in c.adds] == [[2.0, 2.0], [4.0], [1.0], [1.0]]
    assert all(a_["blocks_per_group"] == 4 and a_["n_groups"] == 1 for a_ in c.adds)
    # without the RTN pass, no RTN sums reach the census
    r = bench.nvfp4_census([FakeLayer({"gu": [1.0], "dn": [1.0]}, {})], with_rtn=False)
    assert "sse_vs_rtn" not in r and FakeCensus.made[-1].adds[0]["sum_sq_err_rtn"] is None

    class Broken(FakeLayer):
        def verify(self, t):
            raise RuntimeError("device status 0x2")

    r = bench.nvfp4_census([Broken({"gu": [1.0], "dn": [1.0]}, {})])
    assert "unavailable" in r["sse_vs_rtn"] and "0x2" in r["sse_vs_rtn"]["unavailable"]
