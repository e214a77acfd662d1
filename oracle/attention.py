"""Float64 CPU oracle for exact grouped-query attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  It shares no code with the
CUDA path and must never be used as a fallback for it.

What it computes is the plain definition the pages state: attention is
``A = softmax(Q K^T) V`` (Stream-CQSA summary, "Methodology", item 2), with the
1/sqrt(d) scale, a causal mask and grouped-query heads (LLM-CoOpt summary,
"Opt-GQA"), and the row log-sum-exp that the ORT CPU GQA analysis uses to merge
Flash-Decoding partials ("Flash Decoding" section).  The full score row is
formed explicitly: no tiling, no online softmax, no blocking beyond looping over
(batch, head) and chunks of query rows.

Readings of points the pages leave open:
  * query row i of a call sits at absolute position q_pos0 + i and key j at
    kv_pos0 + j; the causal mask keeps j when kv_pos0 + j <= q_pos0 + i
    (the packed-QSA analysis computes positions as past length + local index);
  * query head h reads KV head h // (Hq / Hkv);
  * keys at or beyond kv_lens[b] are invisible;
  * a row with no visible key has O = 0 and LSE = -inf;
  * LSE is the natural-log log-sum-exp of the scaled scores.
"""
from __future__ import annotations

import numpy as np


def as_f64(x) -> np.ndarray:
    """Exact widening of a torch tensor (any float dtype) or array to float64."""
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if x.dtype != __import__("torch").float64:
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def attention(q, k, v, *, scale: float, causal: bool, q_pos0: int = 0, kv_pos0: int = 0,
              kv_lens=None, rows=None, k_scale=None, v_scale=None, row_chunk: int = 256):
    """Exact attention rows by the definition.

    q: [B, S, Hq, D]; k, v: [B, T, Hkv, D] (values, or FP8 values already decoded);
    k_scale, v_scale: optional [B, T, Hkv] multipliers (per-token dequant scales).
    kv_lens: optional [B] visible lengths (default T).
    rows: optional list of query indices to evaluate (default all S).
    Returns (o [B, R, Hq, D] float64, lse [B, Hq, R] float64), R = len(rows).
    """
    q = as_f64(q)
    B, S, Hq, D = q.shape
    T, Hkv = k.shape[1], k.shape[2]
    assert Hq % Hkv == 0, "query heads must be a multiple of KV heads"
    G = Hq // Hkv
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    lens = np.full(B, T, dtype=np.int64) if kv_lens is None else np.asarray(as_f64(kv_lens), dtype=np.int64)
    R = len(rows)
    o = np.zeros((B, R, Hq, D))
    lse = np.full((B, Hq, R), -np.inf)
    for b in range(B):
        L = int(min(lens[b], T))
        if L <= 0:
            continue
        for kvh in range(Hkv):
            K = as_f64(k[b, :L, kvh, :])
            V = as_f64(v[b, :L, kvh, :])
            if k_scale is not None:
                K = K * as_f64(k_scale[b, :L, kvh])[:, None]
            if v_scale is not None:
                V = V * as_f64(v_scale[b, :L, kvh])[:, None]
            key_pos = kv_pos0 + np.arange(L)
            for h in range(kvh * G, (kvh + 1) * G):
                for r0 in range(0, R, row_chunk):
                    rr = rows[r0:r0 + row_chunk]
                    Qr = as_f64(q[b, rr, h, :])
                    s = scale * (Qr @ K.T)  # [r, L] full score rows
                    if causal:
                        visible = key_pos[None, :] <= (q_pos0 + rr)[:, None]
                        s = np.where(visible, s, -np.inf)
                    mx = s.max(axis=1)
                    has = np.isfinite(mx)
                    mx_safe = np.where(has, mx, 0.0)
                    e = np.exp(s - mx_safe[:, None])
                    tot = e.sum(axis=1)
                    with np.errstate(divide="ignore"):
                        row_lse = np.where(has, mx_safe + np.log(tot), -np.inf)
                    w = np.where(has[:, None], e / np.where(has, tot, 1.0)[:, None], 0.0)
                    o[b, r0:r0 + len(rr), h, :] = w @ V
                    lse[b, h, r0:r0 + len(rr)] = row_lse
    return o, lse


def decode(q, k, v, kv_lens, *, scale: float, k_scale=None, v_scale=None):
    """Single-token decode: query of sequence b sits at position len_b - 1 and sees
    every key below len_b (the causal reading with q_pos0 = len_b - 1).

    q: [B, Hq, D]; k, v: [B, Tmax, Hkv, D]; kv_lens [B].
    Returns (o [B, Hq, D], lse [B, Hq]).
    """
    q = as_f64(q)
    B = q.shape[0]
    o, lse = attention(q[:, None], k, v, scale=scale, causal=False, kv_lens=kv_lens,
                       k_scale=k_scale, v_scale=v_scale)
    return o[:, 0], lse[:, :, 0]


def decode_multi(q, k, v, kv_lens, *, scale: float, k_scale=None, v_scale=None):
    """Multi-token decode: the cache already holds the n_q new tokens, so token i of sequence b
    is at position len_b - n_q + i (past length + index among the new tokens, as the ORT CUDA
    packed sparse attention analysis positions packed tokens in "Code analysis" 1 and verifies
    several new tokens against one key state in "Code analysis" 2) and attends causally to the
    cache.

    q: [B, n_q, Hq, D]; k, v: [B, Tmax, Hkv, D]; kv_lens [B].
    Returns (o [B, n_q, Hq, D], lse [B, n_q, Hq]).
    """
    q = as_f64(q)
    B, n_q, Hq, D = q.shape
    lens = [int(x) for x in np.asarray(kv_lens).reshape(-1)]
    o = np.zeros((B, n_q, Hq, D))
    lse = np.full((B, n_q, Hq), -np.inf)
    for b in range(B):
        ks = None if k_scale is None else k_scale[b:b + 1]
        vs = None if v_scale is None else v_scale[b:b + 1]
        ob, lb = attention(q[b:b + 1], k[b:b + 1], v[b:b + 1], scale=scale, causal=True, q_pos0=lens[b] - n_q,
                           kv_pos0=0, kv_lens=[lens[b]], k_scale=ks, v_scale=vs)
        o[b] = ob[0]
        lse[b] = np.asarray(lb[0]).T
    return o, lse


def prefill_varlen(q, k, v, cu_q, cu_k, *, scale: float, causal: bool):
    """Packed variable-length prefill (ORT packed-QSA analysis, "Code analysis 1"): sequence b's
    queries are rows cu_q[b]..cu_q[b+1]-1 of q and its keys rows cu_k[b]..cu_k[b+1]-1 of k, v; a
    query's position is the past length (keys - queries) plus its index among the queries.

    q: [total_q, Hq, D]; k, v: [total_k, Hkv, D].  Returns (o [total_q, Hq, D], lse [total_q, Hq]).
    """
    q = as_f64(q)
    cu_q = [int(x) for x in np.asarray(cu_q).reshape(-1)]
    cu_k = [int(x) for x in np.asarray(cu_k).reshape(-1)]
    total_q, Hq, D = q.shape
    o = np.zeros((total_q, Hq, D))
    lse = np.full((total_q, Hq), -np.inf)
    for b in range(len(cu_q) - 1):
        qs, qe, ks, ke = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        if qe <= qs:
            continue
        ob, lb = attention(q[None, qs:qe], k[None, ks:ke], v[None, ks:ke], scale=scale, causal=causal,
                           q_pos0=(ke - ks) - (qe - qs), kv_pos0=0)
        o[qs:qe] = ob[0]
        lse[qs:qe] = np.asarray(lb[0]).T
    return o, lse


def merge_lse(o_parts, lse_parts):
    """Exact merge of partial attention results over disjoint key sets.

    For parts k with (o_k, lse_k): lse = log sum_k exp(lse_k) and
    o = sum_k exp(lse_k - lse) o_k; parts with lse = -inf contribute nothing and
    an all-empty row gives o = 0, lse = -inf.  This is the log-sum-exp reduce of
    Flash-Decoding partials (ORT CPU GQA analysis, "Flash Decoding") and the
    recombination of independent sub-attention tasks (Stream-CQSA summary,
    "Methodology", items 2-3).

    o_parts: [P, ..., D]; lse_parts: [P, ...].  Returns (o [..., D], lse [...]).
    """
    o_parts = as_f64(o_parts)
    lse_parts = as_f64(lse_parts)
    mx = lse_parts.max(axis=0)
    has = np.isfinite(mx)
    mx_safe = np.where(has, mx, 0.0)
    w = np.exp(lse_parts - mx_safe[None])  # exp(-inf) = 0 for empty parts
    tot = w.sum(axis=0)
    with np.errstate(divide="ignore"):
        lse = np.where(has, mx_safe + np.log(np.where(has, tot, 1.0)), -np.inf)
    wn = np.where(has[None], w / np.where(has, tot, 1.0)[None], 0.0)
    o = (wn[..., None] * o_parts).sum(axis=0)
    return o, lse
