"""The C-ABI library loads and exports every entry point the headers under
include/ declare; host-side argument checks answer before any CUDA work (these
calls need no GPU)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT


@pytest.fixture(scope="module")
def lib():
    from mxfp_block_scaled_b200 import build, mxq
    build.build()
    return mxq.load()


def declared_functions():
    """Every entry point the headers under include/ declare."""
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            with open(os.path.join(ROOT, "include", h)) as f:
                names += re.findall(r"MXQ_API\s+[\w\s\*]+?\b(mxq_\w+)\s*\(", f.read())
    return names


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("mxq_quantize_nvfp4", "mxq_quantize_mx", "mxq_quantize_act", "mxq_dequant_relerr",
              "mxq_workspace_bytes", "mxq_status_string", "mxq_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from mxfp_block_scaled_b200 import mxq
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(mxq.EXPORTED) <= set(declared_functions())


def test_version_and_status_strings(lib):
    assert lib.mxq_version() >= 10000
    for code in range(7):
        s = lib.mxq_status_string(code)
        assert s and isinstance(s, bytes)
    assert lib.mxq_status_string(99) == b"unknown status"


def test_workspace_sizes(lib):
    # amax bits + per-group, per-CTA amax slots (256 x 8 bytes), each padded
    # to 256 bytes
    assert lib.mxq_workspace_bytes(0, 512, 1536, 2048) == 2048 + 512 * 256 * 8
    assert lib.mxq_workspace_bytes(0, 1, 16, 16) == 256 + 2048
    assert lib.mxq_workspace_bytes(1, 4096, 2048, 0) == 256 + 2048
    # verifier: 16 bytes per chunk of 16384 elements per tensor
    cpt = -(-768 * 2048 // 16384)
    assert lib.mxq_workspace_bytes(2, 1024, 768, 2048) == (1024 * cpt * 16 + 255) // 256 * 256
    assert lib.mxq_workspace_bytes(0, -1, 4, 16) == 0
    assert lib.mxq_workspace_bytes(0, 1 << 40, 1 << 20, 1 << 20) == 0   # overflow


def test_host_argument_errors_return_before_any_launch(lib):
    vp = ctypes.c_void_p
    fake = vp(0x1000)           # never dereferenced: every call below fails its checks first
    # NVFP4: cols not a multiple of 16
    assert lib.mxq_quantize_nvfp4(fake, 1, 4, 24, 1, 0, fake, fake, fake, None, None, fake, fake,
                                  4096, None) == 2
    # negative sizes, bad mode
    assert lib.mxq_quantize_nvfp4(fake, -1, 4, 16, 1, 0, fake, fake, fake, None, None, fake, fake,
                                  4096, None) == 1
    assert lib.mxq_quantize_nvfp4(fake, 1, 4, 16, 7, 0, fake, fake, fake, None, None, fake, fake,
                                  4096, None) == 1
    # null output / status
    assert lib.mxq_quantize_nvfp4(fake, 1, 4, 16, 1, 0, None, fake, fake, None, None, fake, fake,
                                  4096, None) == 1
    assert lib.mxq_quantize_nvfp4(fake, 1, 4, 16, 1, 0, fake, fake, fake, None, None, None, fake,
                                  4096, None) == 1
    # misaligned input
    assert lib.mxq_quantize_nvfp4(vp(0x1002), 1, 4, 16, 1, 0, fake, fake, fake, None, None, fake,
                                  fake, 4096, None) == 3
    # workspace too small
    assert lib.mxq_quantize_nvfp4(fake, 1, 4, 16, 1, 0, fake, fake, fake, None, None, fake, fake,
                                  8, None) == 4
    # MX: block size other than 32, bad format, bad shape
    assert lib.mxq_quantize_mx(fake, 4, 64, 2, 16, 0, fake, fake, None, None) == 6
    assert lib.mxq_quantize_mx(fake, 4, 64, 0, 32, 0, fake, fake, None, None) == 1
    assert lib.mxq_quantize_mx(fake, 4, 48, 2, 32, 0, fake, fake, None, None) == 2
    # verifier: missing s2 for NVFP4, tensors_per_scale < 1
    assert lib.mxq_dequant_relerr(fake, fake, fake, None, 0, 0, 2, 4, 16, 1, fake, fake, None, fake,
                                  4096, None) == 1
    assert lib.mxq_dequant_relerr(fake, fake, fake, fake, 0, 0, 2, 4, 16, 0, fake, fake, None, fake,
                                  4096, None) == 1
    # unknown layout / mode values
    assert lib.mxq_quantize_nvfp4(fake, 1, 4, 16, 1, 5, fake, fake, fake, None, None, fake, fake,
                                  4096, None) == 1
    assert lib.mxq_quantize_mx(fake, 4, 64, 2, 32, 9, fake, fake, None, None) == 1
    assert lib.mxq_dequant_relerr(fake, fake, fake, None, 2, 3, 2, 4, 64, 1, fake, fake, None, fake,
                                  4096, None) == 1
    assert lib.mxq_quantize_act(fake, 4, 64, 0, 2, 0, fake, fake, fake, fake, fake, 4096, None) == 1
    # MX activations have no 4/6 mode
    assert lib.mxq_quantize_act(fake, 4, 64, 2, 1, 0, fake, fake, None, fake, None, 0, None) == 6
    # tiled layout: a scale matrix needs at least one tensor
    assert lib.mxq_dequant_relerr(fake, fake, fake, None, 2, 1, 2, 4, 64, 0, fake, fake, None, fake,
                                  4096, None) == 1
    # weighted search: weight rows neither 1 nor n_groups, cols % 16, misaligned weights
    assert lib.mxq_quantize_nvfp4_weighted(fake, 2, 4, 16, fake, 3, 0, fake, fake, fake, fake, fake,
                                           4096, None) == 1
    assert lib.mxq_quantize_nvfp4_weighted(fake, 2, 4, 24, fake, 1, 0, fake, fake, fake, fake, fake,
                                           4096, None) == 2
    assert lib.mxq_quantize_nvfp4_weighted(fake, 2, 4, 16, vp(0x1004), 1, 0, fake, fake, fake, fake,
                                           fake, 4096, None) == 3
    assert lib.mxq_quantize_nvfp4_weighted(None, 0, 4, 16, None, 1, 0, None, None, None, None, None,
                                           0, None) == 0
    # FP8 -> MX requantization: source block width not a multiple of 32, bad block, bad format
    assert lib.mxq_requant_fp8_mx(fake, fake, 4, 64, 128, 48, 1, 0, fake, fake, None, None) == 2
    assert lib.mxq_requant_fp8_mx(fake, fake, 4, 64, 0, 128, 1, 0, fake, fake, None, None) == 1
    assert lib.mxq_requant_fp8_mx(fake, fake, 4, 64, 128, 128, 0, 0, fake, fake, None, None) == 1
    assert lib.mxq_requant_fp8_mx(fake, fake, 4, 48, 128, 128, 1, 0, fake, fake, None, None) == 2
    assert lib.mxq_requant_fp8_mx(None, fake, 4, 64, 128, 128, 1, 0, fake, fake, None, None) == 1
    assert lib.mxq_requant_fp8_mx(None, None, 0, 64, 128, 128, 1, 0, None, None, None, None) == 0
    # activation: status required; NVFP4 needs input_scale
    assert lib.mxq_quantize_act(fake, 4, 64, 0, 0, 0, fake, fake, fake, None, fake, 4096, None) == 1
    assert lib.mxq_quantize_act(fake, 4, 64, 0, 0, 0, fake, fake, None, fake, fake, 4096, None) == 1


def test_scale_bytes(lib):
    # linear: one byte per block; tiled: rows padded to 128, blocks per row to 4
    assert lib.mxq_scale_bytes(0, 0, 512, 1536, 2048) == 512 * 1536 * 128
    assert lib.mxq_scale_bytes(0, 1, 512, 1536, 2048) == 512 * 1536 * 128
    assert lib.mxq_scale_bytes(0, 1, 2, 130, 80) == 2 * 256 * 8        # 5 blocks -> 8
    assert lib.mxq_scale_bytes(2, 1, 1, 1, 32) == 128 * 4
    assert lib.mxq_scale_bytes(1, 0, 3, 7, 64) == 3 * 7 * 2
    assert lib.mxq_scale_bytes(0, 0, 1, 4, 24) == 0                      # cols % 16
    assert lib.mxq_scale_bytes(0, 2, 1, 4, 16) == 0                      # unknown layout
    assert lib.mxq_scale_bytes(7, 0, 1, 4, 32) == 0                      # unknown format


def test_empty_inputs_are_no_ops(lib):
    # zero groups / zero rows: nothing to do, success without touching memory
    assert lib.mxq_quantize_nvfp4(None, 0, 4, 16, 1, 0, None, None, None, None, None, None, None, 0,
                                  None) == 0
    assert lib.mxq_quantize_mx(None, 0, 64, 2, 32, 0, None, None, None, None) == 0
    assert lib.mxq_dequant_relerr(None, None, None, None, 2, 0, 0, 4, 64, 1, None, None, None, None, 0,
                                  None) == 0


def test_maximum_sizes_are_refused_before_any_launch(lib):
    vp = ctypes.c_void_p
    fake = vp(0x1000)
    # element count beyond int64 / 4
    assert lib.mxq_quantize_nvfp4(fake, 1 << 30, 1 << 20, 1 << 20, 1, 0, fake, fake, fake, None, None,
                                  fake, fake, 4096, None) == 2
    # tiled scales: a group of 2^32 blocks does not fit the 32-bit tile offsets
    assert lib.mxq_quantize_nvfp4(fake, 1, 1 << 22, 1 << 14, 1, 1, fake, fake, fake, None, None, fake,
                                  fake, 4096, None) == 2
    assert lib.mxq_quantize_mx(fake, 1 << 22, 1 << 15, 2, 32, 1, fake, fake, None, None) == 2
    # the verifier indexes its chunks in 32 bits
    assert lib.mxq_dequant_relerr(fake, fake, fake, fake, 0, 0, 1 << 31, 16, 1024, 1, fake, fake, None,
                                  fake, 1 << 40, None) == 2
    # the largest layer of the workloads is accepted by the same checks (the workspace sizes agree)
    assert lib.mxq_workspace_bytes(0, 512, 1536, 2048) > 0
    assert lib.mxq_workspace_bytes(2, 1536, 768, 2048) > 0


def test_groups_without_elements_still_need_their_scales(lib):
    vp = ctypes.c_void_p
    fake = vp(0x1000)
    # no elements: x, codes, scales and the workspace may be NULL, but s2 and status are written
    assert lib.mxq_quantize_nvfp4(None, 3, 0, 32, 1, 0, None, None, None, None, None, fake, None, 0,
                                  None) == 1
    assert lib.mxq_quantize_nvfp4(None, 3, 0, 32, 1, 0, None, None, fake, None, None, None, None, 0,
                                  None) == 1
    assert lib.mxq_global_scale_nvfp4(None, 3, 0, 32, None, fake, None) == 1
    assert lib.mxq_quantize_nvfp4_s2(None, 3, 0, 32, None, 1, 0, None, None, None, None, fake, None) == 1
    assert lib.mxq_quantize_nvfp4(None, 3, 0, 32, 1, 0, None, None, vp(0x1002), None, None, fake, None,
                                  0, None) == 3


def test_product_path_refuses_to_run_without_the_library(tmp_path):
    from mxfp_block_scaled_b200 import mxq
    with pytest.raises(RuntimeError, match="not built"):
        mxq.load(str(tmp_path / "missing.so"))
