"""fp8_block_scaled_11_b200 -- FP8 (e4m3) dynamic quantization and scaled GEMM
for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libfp8bs.so`` (declared in
``include/fp8bs.h``); ``fp8_block_scaled_11_b200.ops`` is its thin Python
binding (argument marshalling only).  Importing the package does not load the
library; the first op call does, and raises if it is missing.
"""
__all__ = ["ops", "inputs"]
