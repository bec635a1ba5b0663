"""B200-native paged KV-cache decode hot path.

PagedAttention's data-parallel hot path: single-query decode attention over
a KV cache stored in fixed-size physical blocks reached through a block
table, plus the cache write and the copy-on-write block copy that maintain
that cache, and a host block manager; and causal prefill / chunked-prefill
attention over the same cache on the tensor cores.  All device work runs in the CUDA
library ``libpagedkv.so`` (sm_100a) behind a C ABI; the Python names below
only marshal arguments into it (see ``binding.py``).

Importing this package loads nothing; the library is opened on first use
and a missing library is an error, never a fallback.
"""

__all__ = [
    "paged_attention_decode", "paged_attention_decode_append", "paged_attention_decode_fp8kv",
    "paged_attention_decode_noalloc", "paged_attention_prefill",
    "reshape_and_cache_fp8kv", "paged_attention_workspace_size", "paged_attention_partition_size",
    "reshape_and_cache", "copy_blocks", "swap_blocks", "read_device_errors", "set_wait_limit", "BlockManager",
    "load_library",
    "PagedKVError", "OutOfBlocks", "default_workspace",
]


def __getattr__(name):
    if name in __all__:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
