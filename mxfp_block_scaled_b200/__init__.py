"""B200-native block-scaled microscaling quantizer (NVFP4 4/6-optimal,
MXFP4, MXFP8) with a fused dequantize + relative-error verifier.

The compute path is the C-ABI CUDA library ``libmxq.so`` (declared in
``include/mxq.h``); ``mxfp_block_scaled_b200.mxq`` is its thin Python binding.
"""
__all__ = ["mxq", "workloads"]
