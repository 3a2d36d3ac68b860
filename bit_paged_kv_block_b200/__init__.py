"""SAW-INT4 paged INT4 KV-cache compression for NVIDIA B200 (sm_100a).

The product is libsaw.so (CUDA kernels behind the C ABI in include/saw.h); ``saw`` is its thin
Python binding and ``synth`` draws seeded synthetic inputs.  Import ``saw`` explicitly:

    from bit_paged_kv_block_b200 import saw
"""
__all__ = ["saw", "synth", "build"]
