"""Exact long-context attention on B200 (sm_100a): tcgen05/TMEM prefill, split-KV decode with
an exact log-sum-exp merge, FP8 KV dequantisation in the tile load, and a host streamer that
feeds (query block, key chunk) sub-tasks under a device-memory budget.

The compute lives in libattn.so (C ABI, include/attn.h); ``attn`` is its thin binding.
Importing the package does not load the library; the first call does, and fails loudly
if it is missing.
"""

_API = ("attn_prefill", "attn_decode_splitkv", "attn_decode_splitkv_noalloc", "attn_decode_paged", "attn_prefill_varlen", "attn_decode_multi", "attn_decode_workspace_bytes", "attn_decode_num_splits",
        "attn_merge_lse", "attn_chunked_stream", "attn_stream_plan", "attn_stream_task", "attn_device_status",
        "attn_set_wait_limit_ns", "attn_debug_wait_probe", "attn_debug_inject", "attn_status_string", "AttnError")

__all__ = list(_API)


def __getattr__(name):
    if name in _API:
        from . import attn as _b
        return getattr(_b, name)
    raise AttributeError(name)
