"""Buffer checks of the Python binding, without a GPU.  The C ABI sees only
pointers, so mxq.py refuses, before anything is enqueued, a buffer that is
not contiguous or is smaller than the call reads or writes (the sizes of
include/mxq.h).  The compute entry points are replaced by a recorder; the
size functions (mxq_scale_bytes, mxq_workspace_bytes) are the library's own.
Host tensors stand in for device tensors: only the sizes matter here."""
import ctypes

import pytest
import torch

from mxfp_block_scaled_b200 import mxq

SWZ = "swizzled_128x4"


class _Recorder:
    def __init__(self, real):
        self.real = real
        self.calls = []

    def __getattr__(self, name):
        if name in ("mxq_scale_bytes", "mxq_workspace_bytes"):
            return getattr(self.real, name)

        def fn(*args):
            self.calls.append((name, args))
            return 0
        return fn


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder(mxq.load())
    monkeypatch.setattr(mxq, "load", lambda *a, **k: r)
    monkeypatch.setattr(mxq, "_p", lambda t: None if t is None else ctypes.c_void_p(t.data_ptr()))
    monkeypatch.setattr(mxq, "_stream", lambda s: None)
    return r


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


@pytest.mark.parametrize("layout", ["linear", SWZ])
def test_allocating_wrappers_pass_the_checks(rec, layout):
    G, R, C = 3, 40, 64
    x = _bf16(G, R, C)
    q = mxq.quantize_nvfp4(x, layout=layout)
    mxq.quantize_nvfp4_weighted(x, torch.ones(C), layout=layout)
    mxq.quantize_nvfp4_weighted(x, torch.ones(G, C), layout=layout)
    # gate_up style verification: 2G tensors of R/2 rows, two per scale matrix
    mxq.dequant_relerr(x, q["codes"], q["scales"], q["s2"], "nvfp4", 2 * G, R // 2, C, 2, layout=layout)
    for fmt in ("mxfp8", "mxfp4"):
        m = mxq.quantize_mx(x, fmt, layout=layout)
        # the stack quantized as one matrix: every tensor in one scale matrix
        mxq.dequant_relerr(x, m["codes"], m["scales"], None, fmt, G, R, C, G, layout=layout)
        mxq.requant_fp8_mx(torch.zeros((130, 96), dtype=torch.uint8), torch.ones((2, 3)), 128, 32, fmt,
                           layout=layout)
    for fmt, mode in (("nvfp4", "rtn"), ("nvfp4", "four_six"), ("mxfp8", "rtn"), ("mxfp4", "rtn")):
        mxq.quantize_act(_bf16(5, C), fmt, mode=mode, layout=layout)
    mxq.quantize_nvfp4_s2(x, torch.ones(G), layout=layout)
    mxq.global_scale_nvfp4(x)
    names = [c[0] for c in rec.calls]
    assert names.count("mxq_quantize_nvfp4_s2") == 1 and names.count("mxq_global_scale_nvfp4") == 1
    assert names.count("mxq_quantize_nvfp4") == 1 and names.count("mxq_quantize_nvfp4_weighted") == 2
    assert names.count("mxq_quantize_mx") == 2 and names.count("mxq_requant_fp8_mx") == 2
    assert names.count("mxq_quantize_act") == 4 and names.count("mxq_dequant_relerr") == 3


def test_hand_built_exact_buffers_pass(rec):
    """Exact-size views into larger buffers (canary padding) and the
    no-workspace verifier with its linear scales."""
    G, R, C = 2, 32, 64
    n = G * R * C
    x = _bf16(G, R, C)
    codes = torch.zeros(n // 2 + 512, dtype=torch.uint8)
    scales = torch.zeros(n // 16 + 512, dtype=torch.uint8)
    s2 = torch.zeros(G + 64)
    mb = torch.zeros((n // 16) // 32 + 64, dtype=torch.int32)
    m4 = torch.zeros(G + 64, dtype=torch.int32)
    st = torch.zeros(1, dtype=torch.int32)
    ws, _ = mxq._workspace("quantize_nvfp4", G, R, C, "cpu")
    mxq.mxq_quantize_nvfp4(x, G, R, C, "four_six", "linear", codes[256:256 + n // 2],
                           scales[256:256 + n // 16], s2[:G], mb[:(n // 16) // 32], m4[:G], st, ws)
    err = torch.zeros(2 * G, dtype=torch.float64)
    mxq.mxq_dequant_relerr_noalloc(x, codes[256:256 + n // 2], scales[256:256 + n // 16], s2[:G], "nvfp4",
                                   2 * G, R // 2, C, 2, err, err.clone(), None)
    assert [c[0] for c in rec.calls] == ["mxq_quantize_nvfp4", "mxq_dequant_relerr_noalloc"]


def _nvfp4_args(G=2, R=32, C=64):
    n = G * R * C
    return dict(x=_bf16(G, R, C), n_groups=G, rows=R, cols=C, mode="four_six", layout="linear",
                codes=torch.zeros(n // 2, dtype=torch.uint8), scales=torch.zeros(n // 16, dtype=torch.uint8),
                s2=torch.zeros(G), mbits=torch.zeros((n // 16 + 31) // 32, dtype=torch.int32),
                m4_count=torch.zeros(G, dtype=torch.int32), status=torch.zeros(1, dtype=torch.int32),
                workspace=mxq._workspace("quantize_nvfp4", G, R, C, "cpu")[0])


@pytest.mark.parametrize("field,bad,match", [
    ("codes", lambda a: a["codes"][1:], "codes holds"),
    ("scales", lambda a: a["scales"][:-1], "scales holds"),
    ("s2", lambda a: a["s2"][:1], "s2 holds"),
    ("mbits", lambda a: a["mbits"][:-1], "mbits holds"),
    ("m4_count", lambda a: a["m4_count"][:1], "m4_count holds"),
    ("x", lambda a: a["x"][:, 1:], "x must be contiguous"),
    ("codes", lambda a: a["codes"].view(64, -1).t(), "codes must be contiguous"),
    ("status", lambda a: torch.zeros(0, dtype=torch.int32), "status holds"),
])
def test_short_or_strided_buffers_are_refused_before_any_call(rec, field, bad, match):
    a = _nvfp4_args()
    a[field] = bad(a)
    with pytest.raises(ValueError, match=match):
        mxq.mxq_quantize_nvfp4(**a)
    assert rec.calls == []


def test_tiled_scales_need_the_tiled_size(rec):
    a = _nvfp4_args()
    a["layout"] = SWZ                          # the linear-size scales are too small when tiled
    with pytest.raises(ValueError, match="scales holds"):
        mxq.mxq_quantize_nvfp4(**a)
    a["scales"] = torch.zeros(mxq.scale_bytes("nvfp4", SWZ, 2, 32, 64), dtype=torch.uint8)
    mxq.mxq_quantize_nvfp4(**a)
    assert len(rec.calls) == 1


def test_verifier_sizes(rec):
    G, R, C = 3, 32, 64
    x = _bf16(G, R, C)
    n = G * R * C
    codes = torch.zeros(n // 2, dtype=torch.uint8)
    scales = torch.zeros(n // 16, dtype=torch.uint8)
    out = [torch.zeros(2 * G, dtype=torch.float64) for _ in range(3)]
    ws, _ = mxq._workspace("dequant_relerr", 2 * G, R // 2, C, "cpu")
    # s2 is read at t / tensors_per_scale: 5 tensors two per scale read 3 values
    with pytest.raises(ValueError, match="s2 holds"):
        mxq.mxq_dequant_relerr(x, codes, scales, torch.zeros(2), "nvfp4", "linear", 5, R // 2, C, 2,
                               *out, ws)
    mxq.mxq_dequant_relerr(x, codes, scales, torch.zeros(3), "nvfp4", "linear", 5, R // 2, C, 2, *out, ws)
    with pytest.raises(ValueError, match="relerr holds"):
        mxq.mxq_dequant_relerr(x, codes, scales, torch.zeros(G), "nvfp4", "linear", 2 * G, R // 2, C, 2,
                               out[0], out[1], out[2][:1], ws)
    with pytest.raises(ValueError, match="x holds"):
        mxq.mxq_dequant_relerr(x[:1], codes, scales, torch.zeros(G), "nvfp4", "linear", 2 * G, R // 2, C,
                               2, *out, ws)
    # tiled scales with a shorter last run: two full matrices of 2 x 16 rows plus one of 16 rows
    need = mxq.scale_bytes("nvfp4", SWZ, 2, 2 * (R // 2), C) + mxq.scale_bytes("nvfp4", SWZ, 1, R // 2, C)
    tiled = torch.zeros(need, dtype=torch.uint8)
    mxq.mxq_dequant_relerr(x, codes, tiled, torch.zeros(3), "nvfp4", SWZ, 5, R // 2, C, 2, *out, ws)
    with pytest.raises(ValueError, match="scales holds"):
        mxq.mxq_dequant_relerr(x, codes, tiled[:-1], torch.zeros(3), "nvfp4", SWZ, 5, R // 2, C, 2, *out, ws)
    assert [c[0] for c in rec.calls] == ["mxq_dequant_relerr"] * 2


def test_other_entry_points_refuse_short_outputs(rec):
    x = _bf16(64, 64)
    st = torch.zeros(1, dtype=torch.int32)
    with pytest.raises(ValueError, match="codes holds"):
        mxq.mxq_quantize_mx(x, 64, 64, "mxfp8", 32, "linear", torch.zeros(64 * 32, dtype=torch.uint8),
                            torch.zeros(128, dtype=torch.uint8), st)
    with pytest.raises(ValueError, match="bscale holds"):
        mxq.mxq_requant_fp8_mx(torch.zeros((130, 64), dtype=torch.uint8), torch.ones(1), 130, 64, 128, 64,
                               "mxfp4", "linear", torch.zeros(130 * 32, dtype=torch.uint8),
                               torch.zeros(130 * 2, dtype=torch.uint8), st)
    with pytest.raises(ValueError, match="input_scale holds"):
        mxq.mxq_quantize_act(x, 64, 64, "nvfp4", "rtn", "linear", torch.zeros(64 * 32, dtype=torch.uint8),
                             torch.zeros(64 * 4, dtype=torch.uint8), torch.zeros(0), st,
                             mxq._workspace("quantize_act", 64, 64, 0, "cpu")[0])
    with pytest.raises(ValueError, match="h holds"):
        mxq.mxq_quantize_nvfp4_weighted(_bf16(2, 16, 64), 2, 16, 64, torch.ones(64), 2, "linear",
                                        torch.zeros(1024, dtype=torch.uint8), torch.zeros(128, dtype=torch.uint8),
                                        torch.zeros(2), st, torch.zeros(4096, dtype=torch.uint8))
    assert rec.calls == []


def test_workspace_is_passed_in_bytes(rec):
    a = _nvfp4_args()
    a["workspace"] = torch.zeros(1000, dtype=torch.float32)
    mxq.mxq_quantize_nvfp4(**a)
    assert rec.calls[0][1][-2] == 4000


def test_s2_and_census_buffers_are_checked(rec):
    G, R, C = 3, 16, 32
    x = _bf16(G, R, C)
    with pytest.raises(ValueError):
        mxq.quantize_nvfp4_s2(x, torch.ones(G - 1))                      # one scale short
    cen = torch.zeros(len(mxq.CENSUS_FIELDS), dtype=torch.float64)
    mxq.mxq_census_reset(cen)
    arr = torch.zeros(4, dtype=torch.float64)
    mxq.mxq_census_add(cen, 4, arr, arr, arr, None, 2, torch.zeros(2, dtype=torch.int32), 8)
    with pytest.raises(ValueError):
        mxq.mxq_census_add(cen, 5, arr, arr, arr, None, 0, None, 0)      # arrays shorter than n_tensors
    with pytest.raises(ValueError):
        mxq.mxq_census_reset(cen[:12])                                    # struct is 13 fields
    names = [c[0] for c in rec.calls]
    assert names == ["mxq_census_reset", "mxq_census_add"]
