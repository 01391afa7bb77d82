"""ctypes front end of the C oracle (test infrastructure only).

Numpy arrays in, numpy arrays out.  Inputs are bf16 bit patterns held in
``uint16`` arrays, the same bits the CUDA path reads.
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mxq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# No FMA contraction, no fast-math, denormals kept: every float operation
# in the oracle is one correctly rounded IEEE operation.
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
          "-fPIC", "-shared", "-Wall", "-Wextra"]

GLOBAL_DIVISOR = 2688.0  # 6 * 448: weight_scale_2 and input_scale


def build(force=False):
    """Compile the oracle into oracle/liboracle.so (gcc)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + ".tmp%d" % os.getpid()
    subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = load_library(_LIB)
    return _lib


def load_library(path):
    """Load a build of mxq_oracle.c and declare its signatures (the mutation
    tests load deliberately broken copies this way)."""
    L = ctypes.CDLL(path)
    d, u, i, i64, vp = (ctypes.c_double, ctypes.c_uint, ctypes.c_int,
                        ctypes.c_int64, ctypes.c_void_p)
    L.oracle_e2m1_value.restype = d
    L.oracle_e2m1_value.argtypes = [u]
    L.oracle_e4m3_value.restype = d
    L.oracle_e4m3_value.argtypes = [u]
    L.oracle_ue8m0_value.restype = d
    L.oracle_ue8m0_value.argtypes = [u]
    L.oracle_e2m1_encode.restype = u
    L.oracle_e2m1_encode.argtypes = [d]
    L.oracle_e4m3_encode.restype = u
    L.oracle_e4m3_encode.argtypes = [d]
    L.oracle_mx_exponent.restype = i
    L.oracle_mx_exponent.argtypes = [d, d]
    L.oracle_quantize_nvfp4.restype = i
    L.oracle_quantize_nvfp4.argtypes = [vp, i64, i64, i64, i, d, vp, vp, vp, vp]
    L.oracle_quantize_nvfp4_s2.restype = i
    L.oracle_quantize_nvfp4_s2.argtypes = [vp, i64, i64, i64, i, vp, vp, vp, vp]
    L.oracle_quantize_mx.restype = i
    L.oracle_quantize_mx.argtypes = [vp, i64, i64, i, vp, vp]
    L.oracle_quantize_nvfp4_weighted.restype = i
    L.oracle_quantize_nvfp4_weighted.argtypes = [vp, i64, i64, i64, vp, i64, vp, vp, vp]
    L.oracle_requant_fp8_mx.restype = i
    L.oracle_requant_fp8_mx.argtypes = [vp, vp, i64, i64, i64, i64, i, vp, vp]
    L.oracle_dequant_relerr.restype = i
    L.oracle_dequant_relerr.argtypes = [vp, vp, vp, vp, i, i64, i64, i64, i64, vp, vp]
    return L


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def e2m1_value(code):
    return lib().oracle_e2m1_value(int(code))


def e4m3_value(code):
    return lib().oracle_e4m3_value(int(code))


def ue8m0_value(code):
    return lib().oracle_ue8m0_value(int(code))


def e2m1_encode(v):
    return lib().oracle_e2m1_encode(float(v))


def e4m3_encode(v):
    return lib().oracle_e4m3_encode(float(v))


def mx_exponent(amax, qmax):
    return lib().oracle_mx_exponent(float(amax), float(qmax))


def _as_bits(x):
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (uint16)")
    return x


def quantize_nvfp4(x_bits, mode=1, global_div=GLOBAL_DIVISOR):
    """x_bits: uint16 [G, R, C].  Returns codes [G,R,C/2], scales [G,R,C/16],
    s2 [G] float32, m4 [G, R*C/16] uint8 (1 = the M=4 plan won)."""
    x = _as_bits(x_bits)
    G, R, C = x.shape
    codes = np.zeros((G, R, C // 2), np.uint8)
    scales = np.zeros((G, R, C // 16), np.uint8)
    s2 = np.zeros(G, np.float32)
    m4 = np.zeros((G, R * C // 16), np.uint8)
    rc = lib().oracle_quantize_nvfp4(_ptr(x), G, R, C, int(mode), float(global_div),
                                     _ptr(codes), _ptr(scales), _ptr(s2), _ptr(m4))
    if rc != 0:
        raise RuntimeError("oracle_quantize_nvfp4 failed: %d" % rc)
    return codes, scales, s2, m4


def quantize_nvfp4_s2(x_bits, s2_in, mode=1):
    """x_bits: uint16 [G, R, C]; s2_in: float32 [G] caller-given global
    scales.  Returns codes [G,R,C/2], scales [G,R,C/16], m4 [G, R*C/16]."""
    x = _as_bits(x_bits)
    G, R, C = x.shape
    s2a = np.ascontiguousarray(s2_in, np.float32)
    codes = np.zeros((G, R, C // 2), np.uint8)
    scales = np.zeros((G, R, C // 16), np.uint8)
    m4 = np.zeros((G, R * C // 16), np.uint8)
    rc = lib().oracle_quantize_nvfp4_s2(_ptr(x), G, R, C, int(mode), _ptr(s2a), _ptr(codes),
                                        _ptr(scales), _ptr(m4))
    if rc != 0:
        raise RuntimeError("oracle_quantize_nvfp4_s2 failed: %d" % rc)
    return codes, scales, m4


def quantize_mx(x_bits, fmt):
    """fmt: 'mxfp4' or 'mxfp8'.  x_bits uint16 [R, C] (or any shape whose
    last dim is C).  Returns codes, scales."""
    x = _as_bits(x_bits)
    C = x.shape[-1]
    R = x.size // C if C else 0
    f = {"mxfp4": 1, "mxfp8": 2}[fmt]
    codes = np.zeros(x.shape[:-1] + ((C // 2) if f == 1 else C,), np.uint8)
    scales = np.zeros(x.shape[:-1] + (C // 32,), np.uint8)
    rc = lib().oracle_quantize_mx(_ptr(x), R, C, f, _ptr(codes), _ptr(scales))
    if rc != 0:
        raise RuntimeError("oracle_quantize_mx failed: %d" % rc)
    return codes, scales


def quantize_nvfp4_weighted(x_bits, h):
    """x_bits: uint16 [G, R, C]; h: float32 [C] (shared) or [G, C].
    Returns codes [G,R,C/2], scales [G,R,C/16], s2 [G]."""
    x = _as_bits(x_bits)
    G, R, C = x.shape
    hh = np.ascontiguousarray(h, np.float32)
    hg = 1 if hh.ndim == 1 else hh.shape[0]
    codes = np.zeros((G, R, C // 2), np.uint8)
    scales = np.zeros((G, R, C // 16), np.uint8)
    s2 = np.zeros(G, np.float32)
    rc = lib().oracle_quantize_nvfp4_weighted(_ptr(x), G, R, C, _ptr(hh), hg, _ptr(codes),
                                              _ptr(scales), _ptr(s2))
    if rc != 0:
        raise RuntimeError("oracle_quantize_nvfp4_weighted failed: %d" % rc)
    return codes, scales, s2


def requant_fp8_mx(fp8, bscale, brows, bcols, fmt):
    """fp8: uint8 E4M3 codes [R, C]; bscale: float32 [ceil(R/brows), ceil(C/bcols)].
    Returns MX codes and scales of the fp32-dequantized source."""
    q = np.ascontiguousarray(fp8, np.uint8)
    R, C = q.shape
    sc = np.ascontiguousarray(bscale, np.float32)
    f = {"mxfp4": 1, "mxfp8": 2}[fmt]
    codes = np.zeros((R, (C // 2) if f == 1 else C), np.uint8)
    scales = np.zeros((R, C // 32), np.uint8)
    rc = lib().oracle_requant_fp8_mx(_ptr(q), _ptr(sc), R, C, brows, bcols, f, _ptr(codes),
                                     _ptr(scales))
    if rc != 0:
        raise RuntimeError("oracle_requant_fp8_mx failed: %d" % rc)
    return codes, scales


def dequant_relerr(x_bits, codes, scales, s2, fmt, n_tensors, rows, cols,
                   tensors_per_scale=1):
    """Per-tensor (sum_sq_err, sum_sq_ref) as float64 arrays [n_tensors]."""
    x = _as_bits(x_bits)
    f = {"nvfp4": 0, "mxfp4": 1, "mxfp8": 2}[fmt]
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    s2a = np.ascontiguousarray(s2, np.float32) if s2 is not None else None
    err = np.zeros(n_tensors, np.float64)
    ref = np.zeros(n_tensors, np.float64)
    rc = lib().oracle_dequant_relerr(_ptr(x), _ptr(codes), _ptr(scales), _ptr(s2a), f,
                                     n_tensors, rows, cols, tensors_per_scale,
                                     _ptr(err), _ptr(ref))
    if rc != 0:
        raise RuntimeError("oracle_dequant_relerr failed: %d" % rc)
    return err, ref


def relerr_from_sums(err, ref):
    """rel = sqrt(sum_sq_err) / sqrt(sum_sq_ref); 0 for an all-zero tensor
    reproduced exactly."""
    err = np.asarray(err, np.float64)
    ref = np.asarray(ref, np.float64)
    out = np.zeros_like(err)
    nz = ref > 0
    out[nz] = np.sqrt(err[nz]) / np.sqrt(ref[nz])
    out[(~nz) & (err > 0)] = np.inf
    return out


def census(err, ref, err_rtn=None, m4_blocks=0, blocks=0):
    """The census figures of a set of tensors, by their definitions
    (dabsLabs/Qwen3.8-Flash-Next-NVFP4, metric table: mean and max relative
    error over the tensors; "What makes this build different": total squared
    error against plain RTN, share of 16-blocks that took M=4), from the
    oracle's per-tensor sums: plain binary64 sums in tensor order.
    Returns a dict with mean_relerr, max_relerr, n_tensors, sum_sq_err,
    sum_sq_ref, sse_vs_rtn (None without err_rtn) and m4_fraction."""
    err = [float(v) for v in np.asarray(err, np.float64).reshape(-1)]
    ref = [float(v) for v in np.asarray(ref, np.float64).reshape(-1)]
    rel = [float(v) for v in relerr_from_sums(err, ref)]
    n = len(rel)
    tot_err = tot_ref = tot_rel = 0.0
    for k in range(n):
        tot_err += err[k]
        tot_ref += ref[k]
        tot_rel += rel[k]
    out = {"n_tensors": n, "mean_relerr": tot_rel / n if n else 0.0, "max_relerr": max(rel) if n else 0.0,
           "sum_sq_err": tot_err, "sum_sq_ref": tot_ref, "sse_vs_rtn": None,
           "m4_fraction": m4_blocks / blocks if blocks else 0.0}
    if err_rtn is not None:
        tot_rtn = 0.0
        for v in np.asarray(err_rtn, np.float64).reshape(-1):
            tot_rtn += float(v)
        out["sse_vs_rtn"] = tot_err / tot_rtn - 1.0
    return out
