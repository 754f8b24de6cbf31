"""B200 (sm_100a) asymmetric 2/4/8-bit KV cache with fused decode attention.

The CUDA library (``lib/libkvq.so``, C ABI in ``include/kvq.h``) does all the
work; :mod:`asymmetric_bit_kv_b200.kvq` is a thin ctypes binding over it.
"""

from .kvq import CacheConfig, KVCache, KvqError, load_library, required_bytes  # noqa: F401
