"""B200-native MXFP8 training hot path: block-32 casts, scaled grouped GEMM, linear.

The compute lives in the C-ABI library ``libmx.so`` (sm_100a CUDA, built from
``csrc/``). ``mxfp8_block_scaled_cast_b200.mx`` is the thin ctypes binding
over it; importing this package does not load the library, so the seeded
input generators in ``synthetic`` also work on a machine without a GPU.
"""
__all__ = ["mx", "synthetic"]
