"""Thin Python binding of libmxq.so (include/mxq.h).

Argument marshalling only: every step of the quantizer and the verifier
runs in the CUDA library.  Torch provides device memory and the current
CUDA stream; tensors are passed by data pointer.  There is no fallback: if
the library is missing the first call raises.

Low-level functions carry the C names (``mxq_quantize_nvfp4`` ...) and take
tensors for every buffer.  ``quantize_nvfp4``, ``quantize_mx``,
``quantize_act`` and ``dequant_relerr`` allocate the outputs and workspace
with torch and return them.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmxq.so")

MXQ_OK = 0
STATUS_NAMES = {0: "ok", 1: "invalid argument", 2: "shape", 3: "align", 4: "workspace",
                5: "cuda", 6: "unsupported"}
DEV_NONFINITE_INPUT = 0x1
DEV_WAIT_TIMEOUT = 0x2
DEV_INVALID_SCALE = 0x4

FMT = {"nvfp4": 0, "mxfp4": 1, "mxfp8": 2}
SCALE_MODE = {"rtn": 0, "four_six": 1}
LAYOUT = {"linear": 0, "swizzled_128x4": 1}
OP = {"quantize_nvfp4": 0, "quantize_act": 1, "dequant_relerr": 2}

EXPORTED = ("mxq_version", "mxq_status_string", "mxq_scale_bytes", "mxq_workspace_bytes",
            "mxq_quantize_nvfp4", "mxq_global_scale_nvfp4", "mxq_quantize_nvfp4_s2", "mxq_quantize_nvfp4_weighted",
            "mxq_quantize_mx", "mxq_requant_fp8_mx", "mxq_quantize_act", "mxq_dequant_relerr",
            "mxq_dequant_relerr_noalloc", "mxq_census_reset", "mxq_census_add")

# Fields of struct mxq_census (include/mxq.h), in order, each 8 bytes.
CENSUS_FIELDS = ("sum_relerr", "max_relerr", "sum_sq_err", "sum_sq_ref", "sum_sq_err_rtn",
                 "n_tensors", "n_tensors_rtn", "blocks", "blocks_m4",
                 "mean_relerr", "sse_vs_rtn", "m4_fraction", "reserved")
_CENSUS_INTS = ("n_tensors", "n_tensors_rtn", "blocks", "blocks_m4")


class MxqError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__("%s failed: %s (%d)" % (fn, STATUS_NAMES.get(code, "?"), code))
        self.code = code


_lib = None


def load(path=LIB_PATH):
    """Load libmxq.so and declare its signatures (raises if missing)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("libmxq.so is not built (%s): run `python -m mxfp_block_scaled_b200.build`"
                           % path)
    L = ctypes.CDLL(path)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    L.mxq_version.restype = i32
    L.mxq_version.argtypes = []
    L.mxq_status_string.restype = ctypes.c_char_p
    L.mxq_status_string.argtypes = [i32]
    L.mxq_scale_bytes.restype = sz
    L.mxq_scale_bytes.argtypes = [i32, i32, i64, i64, i64]
    L.mxq_workspace_bytes.restype = sz
    L.mxq_workspace_bytes.argtypes = [i32, i64, i64, i64]
    L.mxq_quantize_nvfp4.restype = i32
    L.mxq_quantize_nvfp4.argtypes = [vp, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.mxq_global_scale_nvfp4.restype = i32
    L.mxq_global_scale_nvfp4.argtypes = [vp, i64, i64, i64, vp, vp, vp]
    L.mxq_quantize_nvfp4_s2.restype = i32
    L.mxq_quantize_nvfp4_s2.argtypes = [vp, i64, i64, i64, vp, i32, i32, vp, vp, vp, vp, vp, vp]
    L.mxq_census_reset.restype = i32
    L.mxq_census_reset.argtypes = [vp, vp]
    L.mxq_census_add.restype = i32
    L.mxq_census_add.argtypes = [vp, i64, vp, vp, vp, vp, i64, vp, i64, vp]
    L.mxq_quantize_nvfp4_weighted.restype = i32
    L.mxq_quantize_nvfp4_weighted.argtypes = [vp, i64, i64, i64, vp, i64, i32, vp, vp, vp, vp, vp, sz,
                                              vp]
    L.mxq_quantize_mx.restype = i32
    L.mxq_quantize_mx.argtypes = [vp, i64, i64, i32, i32, i32, vp, vp, vp, vp]
    L.mxq_requant_fp8_mx.restype = i32
    L.mxq_requant_fp8_mx.argtypes = [vp, vp, i64, i64, i64, i64, i32, i32, vp, vp, vp, vp]
    L.mxq_quantize_act.restype = i32
    L.mxq_quantize_act.argtypes = [vp, i64, i64, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp]
    L.mxq_dequant_relerr.restype = i32
    L.mxq_dequant_relerr.argtypes = [vp, vp, vp, vp, i32, i32, i64, i64, i64, i64, vp, vp, vp, vp, sz,
                                     vp]
    L.mxq_dequant_relerr_noalloc.restype = i32
    L.mxq_dequant_relerr_noalloc.argtypes = [vp, vp, vp, vp, i32, i64, i64, i64, i64, vp, vp, vp, vp]
    L.mxq_test_stall_next_single_pass.restype = None
    L.mxq_test_stall_next_single_pass.argtypes = [i32]
    if path == LIB_PATH:
        _lib = L
    return L


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmxq takes device tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, rc):
    if rc != MXQ_OK:
        raise MxqError(fn, rc)


def scale_bytes(fmt, layout, n_matrices, rows, cols):
    return load().mxq_scale_bytes(FMT[fmt], LAYOUT[layout], n_matrices, rows, cols)


def workspace_bytes(op, n, rows, cols):
    return load().mxq_workspace_bytes(OP[op], n, rows, cols)


def _workspace(op, n, rows, cols, device):
    nbytes = workspace_bytes(op, n, rows, cols)
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device), nbytes


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def _need(name, t, nbytes):
    """The library sees only a pointer, so a buffer that is not contiguous or
    is smaller than the call reads or writes is refused here, before anything
    is enqueued (the kernels would otherwise touch memory past its end).
    Sizes the library rejects (negative, misaligned shapes) give nbytes <= 0
    here and are left to its status code."""
    if t is None:
        return
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if _nbytes(t) < nbytes:
        raise ValueError("%s holds %d bytes; the call needs %d" % (name, _nbytes(t), nbytes))


def _verify_scale_need(fmt, layout, n_tensors, rows, cols, tps):
    """Scale bytes the verifier reads: n_tensors * rows * cols / block when
    linear; tiled, each run of tps tensors is one scale matrix (the last run
    may be shorter)."""
    if layout == "linear" or tps < 1:
        return scale_bytes(fmt, "linear", n_tensors, rows, cols)
    full, rem = divmod(n_tensors, tps)
    return (scale_bytes(fmt, layout, full, rows * tps, cols)
            + (scale_bytes(fmt, layout, 1, rows * rem, cols) if rem else 0))


def _code_bytes(fmt, n):
    return n if fmt == "mxfp8" else n // 2


# ---------------------------------------------------------------- C names --
def mxq_quantize_nvfp4(x, n_groups, rows, cols, mode, layout, codes, scales, s2, mbits, m4_count,
                       status, workspace, stream=None):
    n = n_groups * rows * cols
    _need("x", x, 2 * n)
    _need("codes", codes, n // 2)
    _need("scales", scales, scale_bytes("nvfp4", layout, n_groups, rows, cols))
    _need("s2", s2, 4 * n_groups)
    _need("mbits", mbits, 4 * ((n // 16 + 31) // 32))
    _need("m4_count", m4_count, 4 * n_groups)
    _need("status", status, 4)
    rc = load().mxq_quantize_nvfp4(_p(x), n_groups, rows, cols, SCALE_MODE[mode], LAYOUT[layout],
                                   _p(codes),
                                   _p(scales), _p(s2), _p(mbits), _p(m4_count), _p(status),
                                   _p(workspace), _nbytes(workspace), _stream(stream))
    _check("mxq_quantize_nvfp4", rc)


def mxq_global_scale_nvfp4(x, n_groups, rows, cols, s2, status, stream=None):
    _need("x", x, 2 * n_groups * rows * cols)
    _need("s2", s2, 4 * n_groups)
    _need("status", status, 4)
    rc = load().mxq_global_scale_nvfp4(_p(x), n_groups, rows, cols, _p(s2), _p(status), _stream(stream))
    _check("mxq_global_scale_nvfp4", rc)


def mxq_quantize_nvfp4_s2(x, n_groups, rows, cols, s2_in, mode, layout, codes, scales, mbits, m4_count,
                          status, stream=None):
    n = n_groups * rows * cols
    _need("x", x, 2 * n)
    _need("s2_in", s2_in, 4 * n_groups)
    _need("codes", codes, n // 2)
    _need("scales", scales, scale_bytes("nvfp4", layout, n_groups, rows, cols))
    _need("mbits", mbits, 4 * ((n // 16 + 31) // 32))
    _need("m4_count", m4_count, 4 * n_groups)
    _need("status", status, 4)
    rc = load().mxq_quantize_nvfp4_s2(_p(x), n_groups, rows, cols, _p(s2_in), SCALE_MODE[mode],
                                      LAYOUT[layout], _p(codes), _p(scales), _p(mbits), _p(m4_count),
                                      _p(status), _stream(stream))
    _check("mxq_quantize_nvfp4_s2", rc)


def mxq_census_reset(census, stream=None):
    _need("census", census, 8 * len(CENSUS_FIELDS))
    _check("mxq_census_reset", load().mxq_census_reset(_p(census), _stream(stream)))


def mxq_census_add(census, n_tensors, sum_sq_err, sum_sq_ref, relerr, sum_sq_err_rtn, n_groups,
                   m4_count, blocks_per_group, stream=None):
    _need("census", census, 8 * len(CENSUS_FIELDS))
    for name, t in (("sum_sq_err", sum_sq_err), ("sum_sq_ref", sum_sq_ref), ("relerr", relerr),
                    ("sum_sq_err_rtn", sum_sq_err_rtn)):
        _need(name, t, 8 * n_tensors)
    _need("m4_count", m4_count, 4 * n_groups)
    rc = load().mxq_census_add(_p(census), n_tensors, _p(sum_sq_err), _p(sum_sq_ref), _p(relerr),
                               _p(sum_sq_err_rtn), n_groups, _p(m4_count), blocks_per_group,
                               _stream(stream))
    _check("mxq_census_add", rc)


def mxq_quantize_nvfp4_weighted(x, n_groups, rows, cols, h, h_groups, layout, codes, scales, s2,
                                status, workspace, stream=None):
    n = n_groups * rows * cols
    _need("x", x, 2 * n)
    _need("h", h, 4 * h_groups * cols)
    _need("codes", codes, n // 2)
    _need("scales", scales, scale_bytes("nvfp4", layout, n_groups, rows, cols))
    _need("s2", s2, 4 * n_groups)
    _need("status", status, 4)
    rc = load().mxq_quantize_nvfp4_weighted(_p(x), n_groups, rows, cols, _p(h), h_groups,
                                            LAYOUT[layout], _p(codes), _p(scales), _p(s2), _p(status),
                                            _p(workspace), _nbytes(workspace), _stream(stream))
    _check("mxq_quantize_nvfp4_weighted", rc)


def mxq_quantize_mx(x, rows, cols, fmt, block, layout, codes, scales, status, stream=None):
    n = rows * cols
    _need("x", x, 2 * n)
    _need("codes", codes, _code_bytes(fmt, n))
    _need("scales", scales, scale_bytes(fmt, layout, 1, rows, cols))
    _need("status", status, 4)
    rc = load().mxq_quantize_mx(_p(x), rows, cols, FMT[fmt], block, LAYOUT[layout], _p(codes),
                                _p(scales), _p(status), _stream(stream))
    _check("mxq_quantize_mx", rc)


def mxq_requant_fp8_mx(fp8, bscale, rows, cols, brows, bcols, fmt, layout, codes, scales, status,
                       stream=None):
    n = rows * cols
    _need("fp8", fp8, n)
    if brows > 0 and bcols > 0:
        _need("bscale", bscale, 4 * (-(-rows // brows)) * (-(-cols // bcols)))
    _need("codes", codes, _code_bytes(fmt, n))
    _need("scales", scales, scale_bytes(fmt, layout, 1, rows, cols))
    _need("status", status, 4)
    rc = load().mxq_requant_fp8_mx(_p(fp8), _p(bscale), rows, cols, brows, bcols, FMT[fmt],
                                   LAYOUT[layout], _p(codes), _p(scales), _p(status), _stream(stream))
    _check("mxq_requant_fp8_mx", rc)


def mxq_quantize_act(tokens, T, hidden, fmt, mode, layout, codes, scales, input_scale, status,
                     workspace, stream=None):
    n = T * hidden
    _need("tokens", tokens, 2 * n)
    _need("codes", codes, _code_bytes(fmt, n))
    _need("scales", scales, scale_bytes(fmt, layout, 1, T, hidden))
    _need("input_scale", input_scale, 4 if fmt == "nvfp4" else 0)
    _need("status", status, 4)
    rc = load().mxq_quantize_act(_p(tokens), T, hidden, FMT[fmt], SCALE_MODE[mode], LAYOUT[layout],
                                 _p(codes), _p(scales),
                                 _p(input_scale), _p(status), _p(workspace),
                                 _nbytes(workspace), _stream(stream))
    _check("mxq_quantize_act", rc)


def _need_verify(x, codes, scales, s2, fmt, layout, n_tensors, rows, cols, tps, err, ref, rel):
    n = n_tensors * rows * cols
    _need("x", x, 2 * n)
    _need("codes", codes, _code_bytes(fmt, n))
    _need("scales", scales, _verify_scale_need(fmt, layout, n_tensors, rows, cols, tps))
    if fmt == "nvfp4" and tps >= 1:
        _need("s2", s2, 4 * (-(-n_tensors // tps)))
    for name, t in (("sum_sq_err", err), ("sum_sq_ref", ref), ("relerr", rel)):
        _need(name, t, 8 * n_tensors)


def mxq_dequant_relerr(x, codes, scales, s2, fmt, layout, n_tensors, rows, cols,
                       tensors_per_scale, sum_sq_err, sum_sq_ref, relerr, workspace, stream=None):
    _need_verify(x, codes, scales, s2, fmt, layout, n_tensors, rows, cols, tensors_per_scale,
                 sum_sq_err, sum_sq_ref, relerr)
    rc = load().mxq_dequant_relerr(_p(x), _p(codes), _p(scales), _p(s2), FMT[fmt], LAYOUT[layout],
                                   n_tensors, rows, cols, tensors_per_scale, _p(sum_sq_err), _p(sum_sq_ref),
                                   _p(relerr), _p(workspace), _nbytes(workspace), _stream(stream))
    _check("mxq_dequant_relerr", rc)


def mxq_dequant_relerr_noalloc(x, codes, scales, s2, fmt, n_tensors, rows, cols,
                               tensors_per_scale, sum_sq_err, sum_sq_ref, relerr, stream=None):
    """The verifier without a workspace, for callers that cannot allocate
    device memory: its partial sums live in a fixed 2 MiB array inside the
    library (at most 131072 chunks of 16384 elements per call).  Calls whose
    GPU work overlaps in time share that array and race."""
    _need_verify(x, codes, scales, s2, fmt, "linear", n_tensors, rows, cols, tensors_per_scale,
                 sum_sq_err, sum_sq_ref, relerr)
    rc = load().mxq_dequant_relerr_noalloc(_p(x), _p(codes), _p(scales), _p(s2), FMT[fmt],
                                           n_tensors, rows, cols, tensors_per_scale,
                                           _p(sum_sq_err), _p(sum_sq_ref), _p(relerr),
                                           _stream(stream))
    _check("mxq_dequant_relerr_noalloc", rc)


# ------------------------------------------------------------ allocating --
def _bf16(x):
    if x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise ValueError("expected a contiguous bf16 tensor")
    return x


def quantize_nvfp4(x, mode="four_six", with_mbits=True, stream=None, layout="linear"):
    """x: bf16 [G, R, C] on the device.  Returns a dict of device tensors:
    codes [G,R,C/2] u8, scales ([G,R,C/16] u8 when linear, the flat tiled
    bytes of G matrices when layout="swizzled_128x4"), s2 [G] f32, mbits u32
    words, m4_count [G] i32-view of u32, status [1]."""
    _bf16(x)
    G, R, C = x.shape
    dev = x.device
    out = {
        "codes": torch.empty((G, R, C // 2), dtype=torch.uint8, device=dev),
        "scales": torch.empty((G, R, C // 16), dtype=torch.uint8, device=dev) if layout == "linear"
        else torch.empty(max(scale_bytes("nvfp4", layout, G, R, C), 1), dtype=torch.uint8, device=dev),
        "s2": torch.empty(G, dtype=torch.float32, device=dev),
        "mbits": torch.empty(((G * R * C // 16) + 31) // 32 or 1, dtype=torch.int32, device=dev)
        if with_mbits else None,
        "m4_count": torch.empty(max(G, 1), dtype=torch.int32, device=dev),
        "status": torch.zeros(1, dtype=torch.int32, device=dev),
    }
    ws, _ = _workspace("quantize_nvfp4", G, R, C, dev)
    mxq_quantize_nvfp4(x, G, R, C, mode, layout, out["codes"], out["scales"], out["s2"],
                       out["mbits"], out["m4_count"], out["status"], ws, stream)
    return out


def quantize_nvfp4_s2(x, s2_in, mode="four_six", with_mbits=True, stream=None, layout="linear"):
    """x: bf16 [G, R, C]; s2_in: fp32 [G] global scales on the device (gate
    and up held apart pass the scale they share).  Returns a dict of device
    tensors: codes, scales, mbits, m4_count, status (as quantize_nvfp4,
    without s2)."""
    _bf16(x)
    G, R, C = x.shape
    if s2_in.dtype != torch.float32 or not s2_in.is_contiguous() or s2_in.numel() < G:
        raise ValueError("expected contiguous fp32 global scales [G]")
    dev = x.device
    out = {
        "codes": torch.empty((G, R, C // 2), dtype=torch.uint8, device=dev),
        "scales": torch.empty((G, R, C // 16), dtype=torch.uint8, device=dev) if layout == "linear"
        else torch.empty(max(scale_bytes("nvfp4", layout, G, R, C), 1), dtype=torch.uint8, device=dev),
        "mbits": torch.empty(((G * R * C // 16) + 31) // 32 or 1, dtype=torch.int32, device=dev)
        if with_mbits else None,
        "m4_count": torch.empty(max(G, 1), dtype=torch.int32, device=dev),
        "status": torch.zeros(1, dtype=torch.int32, device=dev),
    }
    mxq_quantize_nvfp4_s2(x, G, R, C, s2_in, mode, layout, out["codes"], out["scales"], out["mbits"],
                          out["m4_count"], out["status"], stream)
    return out


def global_scale_nvfp4(x, stream=None):
    """x: bf16 [G, R, C].  Returns (s2 [G] fp32, status [1]) on the device:
    s2 = RN32(amax_g / 2688) per group."""
    _bf16(x)
    G, R, C = x.shape
    s2 = torch.empty(max(G, 1), dtype=torch.float32, device=x.device)
    status = torch.zeros(1, dtype=torch.int32, device=x.device)
    mxq_global_scale_nvfp4(x, G, R, C, s2, status, stream)
    return s2[:G], status


class Census:
    """A device-resident struct mxq_census: reset on creation, filled by
    add() (mxq_census_add), read by result() (one small device -> host
    copy, after which the struct's fields come back as a dict)."""

    def __init__(self, device="cuda", stream=None):
        self.buf = torch.empty(len(CENSUS_FIELDS), dtype=torch.float64, device=device)
        mxq_census_reset(self.buf, stream)

    def add(self, n_tensors=0, sum_sq_err=None, sum_sq_ref=None, relerr=None, sum_sq_err_rtn=None,
            n_groups=0, m4_count=None, blocks_per_group=0, stream=None):
        mxq_census_add(self.buf, n_tensors, sum_sq_err, sum_sq_ref, relerr, sum_sq_err_rtn, n_groups,
                       m4_count, blocks_per_group, stream)

    def result(self):
        raw = self.buf.cpu()
        ints = raw.view(torch.int64)
        return {k: (int(ints[i]) if k in _CENSUS_INTS else float(raw[i]))
                for i, k in enumerate(CENSUS_FIELDS) if k != "reserved"}


def quantize_nvfp4_weighted(x, h, stream=None, layout="linear"):
    """x: bf16 [G, R, C]; h: fp32 weights per input channel, [C] (shared) or
    [G, C].  Returns dict codes, scales, s2, status."""
    _bf16(x)
    G, R, C = x.shape
    if h.dtype != torch.float32 or not h.is_contiguous() or h.shape[-1] != C:
        raise ValueError("expected contiguous fp32 weights [C] or [G, C]")
    hg = 1 if h.dim() == 1 else h.shape[0]
    dev = x.device
    out = {
        "codes": torch.empty((G, R, C // 2), dtype=torch.uint8, device=dev),
        "scales": torch.empty((G, R, C // 16), dtype=torch.uint8, device=dev) if layout == "linear"
        else torch.empty(max(scale_bytes("nvfp4", layout, G, R, C), 1), dtype=torch.uint8, device=dev),
        "s2": torch.empty(max(G, 1), dtype=torch.float32, device=dev),
        "status": torch.zeros(1, dtype=torch.int32, device=dev),
    }
    ws, _ = _workspace("quantize_nvfp4", G, R, C, dev)
    mxq_quantize_nvfp4_weighted(x, G, R, C, h, hg, layout, out["codes"], out["scales"], out["s2"],
                                out["status"], ws, stream)
    return out


def quantize_mx(x, fmt, stream=None, layout="linear"):
    """x: bf16 [..., C], quantized as one [rows, C] matrix.  Returns dict
    codes, scales (tiled bytes of that one matrix when layout is
    "swizzled_128x4"), status."""
    _bf16(x)
    C = x.shape[-1]
    R = x.numel() // C if C else 0
    dev = x.device
    out = {
        "codes": torch.empty(x.shape[:-1] + ((C // 2) if fmt == "mxfp4" else C,), dtype=torch.uint8,
                             device=dev),
        "scales": torch.empty(x.shape[:-1] + (C // 32,), dtype=torch.uint8, device=dev)
        if layout == "linear"
        else torch.empty(max(scale_bytes(fmt, layout, 1, R, C), 1), dtype=torch.uint8, device=dev),
        "status": torch.zeros(1, dtype=torch.int32, device=dev),
    }
    mxq_quantize_mx(x, R, C, fmt, 32, layout, out["codes"], out["scales"], out["status"], stream)
    return out


def requant_fp8_mx(fp8, bscale, brows, bcols, fmt, stream=None, layout="linear"):
    """fp8: uint8 E4M3 codes [R, C] on the device; bscale: fp32
    [ceil(R/brows), ceil(C/bcols)].  Returns dict codes, scales, status."""
    if fp8.dtype != torch.uint8 or not fp8.is_contiguous() or fp8.dim() != 2:
        raise ValueError("expected a contiguous uint8 [rows, cols] tensor of E4M3 codes")
    if bscale.dtype != torch.float32 or not bscale.is_contiguous():
        raise ValueError("expected contiguous fp32 block scales")
    R, C = fp8.shape
    dev = fp8.device
    out = {
        "codes": torch.empty((R, (C // 2) if fmt == "mxfp4" else C), dtype=torch.uint8, device=dev),
        "scales": torch.empty((R, C // 32), dtype=torch.uint8, device=dev) if layout == "linear"
        else torch.empty(max(scale_bytes(fmt, layout, 1, R, C), 1), dtype=torch.uint8, device=dev),
        "status": torch.zeros(1, dtype=torch.int32, device=dev),
    }
    mxq_requant_fp8_mx(fp8, bscale, R, C, brows, bcols, fmt, layout, out["codes"], out["scales"],
                       out["status"], stream)
    return out


def quantize_act(tokens, fmt, stream=None, mode="rtn", layout="linear"):
    """tokens: bf16 [T, hidden].  NVFP4 returns input_scale too; mode
    "four_six" applies the 4/6-optimal block scales to the tile."""
    _bf16(tokens)
    T, H = tokens.shape
    dev = tokens.device
    blk = 16 if fmt == "nvfp4" else 32
    out = {
        "codes": torch.empty((T, H if fmt == "mxfp8" else H // 2), dtype=torch.uint8, device=dev),
        "scales": torch.empty((T, H // blk), dtype=torch.uint8, device=dev) if layout == "linear"
        else torch.empty(max(scale_bytes(fmt, layout, 1, T, H), 1), dtype=torch.uint8, device=dev),
        "input_scale": torch.empty(1, dtype=torch.float32, device=dev),
        "status": torch.zeros(1, dtype=torch.int32, device=dev),
    }
    ws, _ = _workspace("quantize_act", T, H, 0, dev)
    mxq_quantize_act(tokens, T, H, fmt, mode, layout, out["codes"], out["scales"],
                     out["input_scale"], out["status"], ws, stream)
    return out


def dequant_relerr(x, codes, scales, s2, fmt, n_tensors, rows, cols, tensors_per_scale=1,
                   stream=None, layout="linear"):
    """Per-tensor fp64 (sum_sq_err, sum_sq_ref, relerr) on the device."""
    dev = x.device
    err = torch.empty(max(n_tensors, 1), dtype=torch.float64, device=dev)
    ref = torch.empty_like(err)
    rel = torch.empty_like(err)
    ws, _ = _workspace("dequant_relerr", n_tensors, rows, cols, dev)
    mxq_dequant_relerr(x, codes, scales, s2, fmt, layout, n_tensors, rows, cols, tensors_per_scale,
                       err, ref, rel, ws, stream)
    return err[:n_tensors], ref[:n_tensors], rel[:n_tensors]
