"""Centroid-residual low-bit KV-cache compression and compressed-history
attention for NVIDIA B200 (sm_100a).

The compute lives in libkvq.so (C ABI in include/kvq.h); ``kvq`` is its thin
ctypes binding and ``synth`` draws the seeded synthetic workloads.  Import
``kv_cache_compression_head_b200.kvq`` explicitly: it loads the CUDA library
and raises if it is missing."""

__all__ = ["kvq", "synth"]
