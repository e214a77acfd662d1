"""Paged KV cache for the decode oracle — test infrastructure only (tests, the smoke check and the
benchmark's CPU baseline use it; the library never does).

LLM-CoOpt summary, "Opt-Pa": a sequence is cut into fixed-size pages (e.g. 512 tokens) and only
the pages that are mapped are touched.  A paged decode computes exactly the decode of the cache
the page table describes, so the oracle is that definition: gather each sequence's mapped pages
back into a contiguous cache (plain indexing), then run the decode oracle.
"""
from __future__ import annotations

import numpy as np
import torch

from . import attention as A


def gather(pool, page_table, kv_lens, page_size: int):
    """Contiguous [B, max_pages * page_size, ...] view of a paged pool: sequence b's token t is
    pool[page_table[b, t // page_size], t % page_size].  Positions at or past kv_lens[b] are NaN
    (the decode must never use them); every page below a length must be mapped."""
    pool = torch.as_tensor(pool)
    table = torch.as_tensor(page_table).long()
    lens = torch.as_tensor(kv_lens).long()
    B, max_pages = table.shape
    out = torch.full((B, max_pages * page_size) + tuple(pool.shape[2:]), float("nan"), dtype=torch.float64)
    for b in range(B):
        n = int(lens[b])
        for i in range((n + page_size - 1) // page_size):
            pg = int(table[b, i])
            assert 0 <= pg < pool.shape[0], f"sequence {b} page {i} is not mapped"
            lo = i * page_size
            hi = min(n, lo + page_size)
            out[b, lo:hi] = pool[pg, : hi - lo].to(torch.float64)
    return out


def decode_paged(q, k_pool, v_pool, page_table, kv_lens, page_size: int, *, scale: float,
                 k_scale_pool=None, v_scale_pool=None):
    """Decode over a paged cache (values already dequantised when FP8: pass code values as the
    pools and the scale pools separately).  Returns (o [B, Hq, D], lse [B, Hq]) in float64."""
    k = gather(k_pool, page_table, kv_lens, page_size)
    v = gather(v_pool, page_table, kv_lens, page_size)
    ks = None if k_scale_pool is None else gather(k_scale_pool, page_table, kv_lens, page_size)
    vs = None if v_scale_pool is None else gather(v_scale_pool, page_table, kv_lens, page_size)
    return A.decode(q, k, v, kv_lens, scale=scale, k_scale=ks, v_scale=vs)
