"""paged_kv_cache_433_b200: paged KV-cache decode attention for B200 (sm_100a).

The compute path lives in ``libkvpaged.so`` (hand-written CUDA + host C++),
reached through the C ABI declared in ``include/kvpaged.h``. ``kvpaged`` is a
thin ctypes binding with the same names. Importing this package does not load
the library; the first call does, and fails loudly if it has not been built.
"""
__all__ = ["kvpaged", "workloads"]
