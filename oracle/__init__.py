"""CPU oracle for the asymmetric-bit KV cache (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA library never uses it and
shares no code with it.
"""
