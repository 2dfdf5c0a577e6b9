"""B200-native int4 KV-cache quantization and decode attention on the packed
cache (compressed-domain attention).  The compute path is libtq.so (CUDA,
sm_100a) behind the C ABI of include/tq.h; this package is its binding.
"""
from ._lib import (TQError, decode_chunk_tokens, decode_workspace_bytes, load,
                   quantize_append, sdpa_int4_decode, status_string)
from .cache import CodebookKVCache, Int4KVCache, UniformKVCache

__all__ = ["CodebookKVCache", "Int4KVCache", "UniformKVCache", "TQError", "decode_chunk_tokens", "decode_workspace_bytes", "load",
           "quantize_append", "sdpa_int4_decode", "status_string"]
