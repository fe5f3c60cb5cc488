"""CSA2 (Compressed Sparse Attention 2) over an FP4 main KV cache on NVIDIA B200.

The compute path is libcsa2.so (hand-written sm_100a CUDA kernels behind the C ABI in
include/csa2.h); ``fp4_kv_cache_04_b200.csa2`` is its ctypes binding and
``fp4_kv_cache_04_b200.synth`` draws the seeded synthetic workloads.
"""
__all__ = ["csa2", "synth"]
