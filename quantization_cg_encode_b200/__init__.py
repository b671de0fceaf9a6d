"""B200-native Codec-Gauge cache-coordinate codec.

The compute path is the CUDA library ``libcg.so`` (C ABI declared in
``include/cg.h``); ``quantization_cg_encode_b200.cg`` is its thin Python binding.
"""
