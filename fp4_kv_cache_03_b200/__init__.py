"""CSA2 attention step over an FP4 global KV cache, for B200 (sm_100a).

The compute lives in ``libcsa2.so`` (hand-written CUDA behind a C ABI,
declared in ``include/csa2.h``); ``fp4_kv_cache_03_b200.csa2`` is a thin
ctypes binding with the same names.
"""
