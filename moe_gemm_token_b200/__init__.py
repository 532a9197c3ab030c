"""B200-native FP8 fast-math linear layer: per-token E4M3 quantizer, tcgen05
W8A8 GEMM with per-token x per-channel scales, the W8A16 decode path and the
routed-expert grouped GEMM.

The compute lives in ``libmetis_fp8.so`` (CUDA, sm_100a) behind a C ABI
declared in ``include/metis_fp8.h``; :mod:`moe_gemm_token_b200.metis` is the
thin ctypes binding with the same entry-point names. Importing this package
loads nothing; the library is loaded on first use of the binding.
"""
__version__ = "0.1.0"
