"""B200-native (sm_100a) Universal Attention hot path: prefill forward/backward with the
content-aware decay bias, and the self-pruning KV-cache decode step.

The compute lives in ``libua.so`` (hand-written CUDA, C ABI declared in ``include/ua.h``);
``kv_cache_compression_ua_b200.ua`` is the thin ctypes binding.  Importing this package
does not load the library; the first call into ``ua`` does, and raises if it is missing.
"""
