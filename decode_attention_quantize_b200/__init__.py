"""KV-cache quantize-on-append and quantized decode attention for B200 (sm_100a).

The work runs in ``libkvq.so`` (C ABI, ``include/kvq.h``); ``kvq`` is its ctypes binding.
"""
from .kvq import (  # noqa: F401
    CacheSpec, KvqDesc, KvqError, QuantizedKVCache, kvq_cache_bytes, kvq_decode_attention,
    kvq_decode_workspace_bytes, kvq_dequantize, kvq_get_device_status, kvq_quantize_append, lib,
)
