"""kvq: group-quantized KV cache and decode attention over the packed cache,
for NVIDIA B200 (sm_100a).  The computation lives in libkvq.so (CUDA, C ABI
declared in include/kvq.h); ``kvq`` is its Python binding.

Attributes resolve lazily so that ``quantized_kv_cache_12_b200.build`` can be
imported before the library exists; touching any binding name without a
built libkvq.so raises ImportError (there is no fallback path).
"""
_BINDING_NAMES = (
    "QuantizedKVCache", "KvqError", "alloc_workspace", "workspace_error_word",
    "kvq_chunk_assign", "kvq_chunk_reorder", "kvq_decode_attention", "kvq_decode_partials",
    "kvq_decode_merge", "kvq_decode_attention_noalloc",
    "kvq_decode_workspace_bytes", "kvq_kv_elements", "kvq_plane_bytes",
    "kvq_quantize_append", "kvq_status_string", "kvq_version",
)


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import kvq
        return getattr(kvq, name)
    raise AttributeError(name)
