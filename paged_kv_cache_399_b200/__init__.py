"""B200-native paged KV-cache hot path: cache write and PagedAttention decode.

The compute runs in hand-written sm_100a CUDA kernels behind the C ABI declared
in ``include/pa.h`` (``libpa_b200.so``). ``paged_kv_cache_399_b200.pa`` is the
thin ctypes binding (argument marshalling only); it raises if the CUDA library
is missing -- there is no CPU fallback. ``workloads`` builds seeded synthetic
inputs.
"""

__all__ = ["pa", "workloads"]
