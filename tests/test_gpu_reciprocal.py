"""The refined reciprocal of the NVFP4 fast path (rcp2_rn_mid, and its
one-lane form rcp_rn_mid of the weighted search: hardware approximation +
one Newton-Raphson step) equals CUDA's correctly rounded
reciprocal for every significand at every exponent of [2^-60, 2^60], both
signs: the range every block-scale divisor of the fast path lies in."""
import os
import shutil
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "mxfp_block_scaled_b200", "csrc")


def test_refined_reciprocal_is_correctly_rounded_exhaustively(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = str(tmp_path / "rcp_check")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-I", CSRC, "-o", exe, os.path.join(HERE, "csrc", "rcp_check.cu")], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=300).stdout
    assert out.startswith("mismatches 0 "), out
