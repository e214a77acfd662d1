"""Oracle for the streamed decomposition of causal attention into independent sub-tasks.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Stream-CQSA (summary, "Methodology", items 2-3) splits attention into
sub-attention tasks over sub-sequences that together cover every (query, key)
position pair exactly once, runs each task independently, and recombines the
partial results into the exact full result.  The summary gives no cyclic-quorum
construction, so the reading taken here is the plain partition of the
(query, key) plane into (query block, key chunk) rectangles, keeping a rectangle
when it holds at least one visible pair; partial results are recombined by the
log-sum-exp merge.
"""
from __future__ import annotations

import numpy as np

from .attention import attention, merge_lse


def block_tasks(S: int, T: int, Bq: int, Ck: int, causal: bool, q_pos0: int = 0, kv_pos0: int = 0):
    """Every (query block, key chunk) rectangle that contains a visible pair."""
    out = []
    for qb in range(0, S, Bq):
        q_last = q_pos0 + min(S, qb + Bq) - 1
        for kc in range(0, T, Ck):
            if causal and kv_pos0 + kc > q_last:
                continue
            out.append((qb, kc))
    return out


def coverage(tasks, S: int, T: int, Bq: int, Ck: int, causal: bool):
    """Count, for every visible (i, j) pair, how many tasks contain it.

    Returns (counts [S, T] int, visible [S, T] bool).  An exact cover has
    counts == visible (each visible pair exactly once, nothing else).
    """
    counts = np.zeros((S, T), dtype=np.int64)
    for qb, kc in tasks:
        counts[qb:qb + Bq, kc:kc + Ck] += 1
    i = np.arange(S)[:, None]
    j = np.arange(T)[None, :]
    visible = (j <= i) if causal else np.ones((S, T), dtype=bool)
    return counts * visible, visible


def chunked_attention(q, k, v, *, scale: float, causal: bool, Bq: int, Ck: int):
    """Run each (query block, key chunk) task as its own exact attention call with
    absolute position offsets, then merge the partials of each query block."""
    B, S, Hq, D = q.shape
    T = k.shape[1]
    o = np.zeros((B, S, Hq, D))
    lse = np.full((B, Hq, S), -np.inf)
    for qb in range(0, S, Bq):
        q_blk = q[:, qb:qb + Bq]
        parts_o, parts_l = [], []
        for (qb2, kc) in block_tasks(S, T, Bq, Ck, causal):
            if qb2 != qb:
                continue
            po, pl = attention(q_blk, k[:, kc:kc + Ck], v[:, kc:kc + Ck], scale=scale, causal=causal,
                               q_pos0=qb, kv_pos0=kc)
            parts_o.append(po)
            parts_l.append(pl.transpose(0, 2, 1))  # LSE rows aligned with o's [B, R, Hq]
        mo, ml = merge_lse(np.stack(parts_o), np.stack(parts_l))
        o[:, qb:qb + Bq] = mo
        lse[:, :, qb:qb + Bq] = ml.transpose(0, 2, 1)
    return o, lse
