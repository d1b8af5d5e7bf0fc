"""Paged KV-cache decode attention for NVIDIA B200 (sm_100a).

The compute runs in ``libpagedkv.so`` (C ABI in ``include/pagedkv.h``);
``binding`` is its ctypes wrapper. The names below are resolved from
``binding`` on first use, which raises ImportError when the library has not
been built (``python -m paged_kv_cache_440_b200.build``). There is no fallback.
"""
_EXPORTS = (
    "KVPool", "PagedKVError", "PrefixCache", "default_ctas", "kv_append", "kv_block_copy",
    "kv_quantize", "make_workspace", "paged_attn_decode", "paged_attn_decode_append",
    "paged_attn_decode_static", "paged_attn_partition_append", "paged_attn_decode_cascade",
    "cascade_workspace_bytes", "make_cascade_workspace",
    "paged_attn_merge", "paged_attn_prefill",
    "paged_attn_partition", "required_bytes", "selftest_wait_timeout", "version",
    "workspace_bytes",
)
__all__ = list(_EXPORTS)


def __getattr__(name):
    if name in _EXPORTS:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
