"""CPU oracle of the block-scaled microscaling quantizer.

TEST INFRASTRUCTURE ONLY.  The C oracle (``mxq_oracle.c``), the exact
rational micro-oracle (``micro.py``) and the scale-layout permutation
(``layout.py``) are the checkers the CUDA library is compared against.  Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package; the product library
neither imports nor links it, and the two share no code.
"""
from .capi import (  # noqa: F401
    build,
    lib,
    e2m1_value,
    e4m3_value,
    ue8m0_value,
    e2m1_encode,
    e4m3_encode,
    mx_exponent,
    quantize_nvfp4,
    quantize_nvfp4_s2,
    quantize_nvfp4_weighted,
    quantize_mx,
    requant_fp8_mx,
    dequant_relerr,
    relerr_from_sums,
    census,
)
