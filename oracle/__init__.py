"""CPU oracle for the CSA2 step over an FP4 global KV cache.

Test infrastructure only: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline of ``bench.py`` use it; the product path never does.  It shares no
code with the CUDA library.
"""
