"""kvq: a B200-native quantized KV cache (cache write + int8-KV attention).

The compute lives in ``libkvq.so`` (CUDA, sm_100a) behind a C ABI declared in
``include/kvq.h``; ``quantized_kv_cache_20_b200.kvq`` is the thin ctypes binding.
"""
