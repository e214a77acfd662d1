"""Pins for the float64 oracle: facts fixed by the pages and by mathematics, not by the
oracle itself.  Each pin takes the oracle's attention module as an argument so that
the mutation test can run the same pins against copies of the oracle with planted
mistakes.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _arr(x):
    return np.array(_floatify(x), dtype=np.float64)


def _floatify(x):
    if isinstance(x, list):
        return [_floatify(v) for v in x]
    return float(x)


def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def rng(seed):
    return np.random.default_rng(seed)


def brute_force(q, k, v, scale, causal, q_pos0=0, kv_pos0=0, kv_lens=None):
    """Scalar loops with math.exp: the definition spelled out element by element."""
    B, S, Hq, D = q.shape
    T, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    o = np.zeros((B, S, Hq, D))
    lse = np.full((B, Hq, S), -math.inf)
    for b in range(B):
        L = T if kv_lens is None else int(kv_lens[b])
        for h in range(Hq):
            kvh = h // G
            for i in range(S):
                scores = []
                for j in range(L):
                    if causal and kv_pos0 + j > q_pos0 + i:
                        continue
                    dot = 0.0
                    for d in range(D):
                        dot += q[b, i, h, d] * k[b, j, kvh, d]
                    scores.append((j, scale * dot))
                if not scores:
                    continue
                mx = max(s for _, s in scores)
                tot = sum(math.exp(s - mx) for _, s in scores)
                lse[b, h, i] = mx + math.log(tot)
                for j, s in scores:
                    w = math.exp(s - lse[b, h, i])
                    for d in range(D):
                        o[b, i, h, d] += w * v[b, j, kvh, d]
    return o, lse


# --------------------------------------------------------------------------- pins

def pin_golden(A):
    g = golden()
    for name in ("two_keys", "uniform_causal", "gqa_two_heads_one_kv"):
        ex = g[name]
        o, lse = A.attention(_arr(ex["q"]), _arr(ex["k"]), _arr(ex["v"]), scale=ex["scale"],
                             causal=ex["causal"])
        np.testing.assert_allclose(o, _arr(ex["o"]), rtol=0, atol=1e-12, err_msg=name)
        np.testing.assert_allclose(lse, _arr(ex["lse"]), rtol=0, atol=1e-12, err_msg=name)
    ex = g["merge_two_parts"]
    o, lse = A.merge_lse(_arr(ex["o_parts"]), _arr(ex["lse_parts"]))
    np.testing.assert_allclose(o, _arr(ex["o"]), atol=1e-12)
    np.testing.assert_allclose(lse, _arr(ex["lse"]), atol=1e-12)


def pin_brute_force(A):
    r = rng(1)
    cases = [
        dict(B=1, S=5, T=5, Hq=2, Hkv=1, D=3, causal=True, q_pos0=0, kv_pos0=0),
        dict(B=2, S=4, T=6, Hq=4, Hkv=2, D=2, causal=True, q_pos0=2, kv_pos0=0),
        dict(B=1, S=3, T=7, Hq=3, Hkv=3, D=4, causal=False, q_pos0=0, kv_pos0=0),
        dict(B=1, S=4, T=4, Hq=2, Hkv=2, D=2, causal=True, q_pos0=0, kv_pos0=2),  # early rows see nothing
    ]
    for c in cases:
        q = r.standard_normal((c["B"], c["S"], c["Hq"], c["D"]))
        k = r.standard_normal((c["B"], c["T"], c["Hkv"], c["D"]))
        v = r.standard_normal((c["B"], c["T"], c["Hkv"], c["D"]))
        scale = 1 / math.sqrt(c["D"])
        lens = None
        if c["B"] == 2:
            lens = np.array([6, 3])
        o, lse = A.attention(q, k, v, scale=scale, causal=c["causal"], q_pos0=c["q_pos0"],
                             kv_pos0=c["kv_pos0"], kv_lens=lens)
        ob, lb = brute_force(q, k, v, scale, c["causal"], c["q_pos0"], c["kv_pos0"], lens)
        np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
        np.testing.assert_array_equal(np.isinf(lse), np.isinf(lb))
        fin = np.isfinite(lb)
        np.testing.assert_allclose(lse[fin], lb[fin], rtol=0, atol=1e-12)


def pin_sdpa(A):
    """Library special case: torch's CPU scaled_dot_product_attention in float64."""
    g = torch.Generator().manual_seed(7)
    for (B, S, T, Hq, Hkv, D, causal) in [(2, 33, 33, 8, 2, 16, True), (1, 17, 40, 4, 4, 8, False)]:
        q = torch.randn(B, S, Hq, D, generator=g, dtype=torch.float64)
        k = torch.randn(B, T, Hkv, D, generator=g, dtype=torch.float64)
        v = torch.randn(B, T, Hkv, D, generator=g, dtype=torch.float64)
        scale = 1 / math.sqrt(D)
        # torch's is_causal aligns the mask to the top-left corner, i.e. q_pos0 = kv_pos0 = 0
        ref = torch.nn.functional.scaled_dot_product_attention(
            q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2), is_causal=causal, scale=scale,
            enable_gqa=True).transpose(1, 2)
        o, lse = A.attention(q.numpy(), k.numpy(), v.numpy(), scale=scale, causal=causal)
        np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
        # LSE against torch.logsumexp over explicitly masked scores
        G = Hq // Hkv
        kk = k.repeat_interleave(G, dim=2)
        s = torch.einsum("bshd,bthd->bhst", q, kk) * scale
        if causal:
            s = s.masked_fill(torch.ones(S, T, dtype=torch.bool).triu(1), float("-inf"))
        np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12)


def pin_uniform_scores(A):
    """Q = 0: every visible score is 0, so O_i = mean(V[0..i]) and LSE_i = ln(i+1)."""
    r = rng(2)
    B, S, Hq, Hkv, D = 1, 40, 4, 2, 8
    q = np.zeros((B, S, Hq, D))
    k = r.standard_normal((B, S, Hkv, D))
    v = r.standard_normal((B, S, Hkv, D))
    o, lse = A.attention(q, k, v, scale=0.3, causal=True)
    G = Hq // Hkv
    for h in range(Hq):
        cm = np.cumsum(v[0, :, h // G, :], axis=0) / np.arange(1, S + 1)[:, None]
        np.testing.assert_allclose(o[0, :, h, :], cm, atol=1e-12)
        np.testing.assert_allclose(lse[0, h], np.log(np.arange(1, S + 1)), atol=1e-12)


def pin_dominant_key(A):
    """One key aligned with the query with a score gap >= delta over all others:
    ||O - V_j*||_inf <= (n-1) e^{-delta} * 2 max|V|."""
    r = rng(3)
    D, T, delta = 16, 50, 30.0
    qv = r.standard_normal(D)
    jstar = 17
    k = r.standard_normal((1, T, 1, D)) * 0.01
    k[0, jstar, 0] = (delta + 5.0) * qv / (qv @ qv)  # score delta+5 at scale 1, others |s| << 5
    v = r.standard_normal((1, T, 1, D))
    o, lse = A.attention(qv.reshape(1, 1, 1, D), k, v, scale=1.0, causal=False)
    s = k[0, :, 0] @ qv
    gap = s[jstar] - np.max(np.delete(s, jstar))
    assert gap >= delta
    bound = (T - 1) * math.exp(-gap) * 2 * np.abs(v).max()
    assert np.abs(o[0, 0, 0] - v[0, jstar, 0]).max() <= bound + 1e-15
    assert abs(lse[0, 0, 0] - s[jstar]) <= (T - 1) * math.exp(-gap) + 1e-15


def pin_single_visible_key(A):
    """Causal row 0 sees only key 0: O_0 = V_0 and LSE_0 = scale <q_0, k_0>."""
    r = rng(4)
    q = r.standard_normal((1, 6, 2, 8))
    k = r.standard_normal((1, 6, 1, 8))
    v = r.standard_normal((1, 6, 1, 8))
    o, lse = A.attention(q, k, v, scale=0.25, causal=True)
    for h in range(2):
        np.testing.assert_allclose(o[0, 0, h], v[0, 0, 0], atol=1e-14)
        assert abs(lse[0, h, 0] - 0.25 * (q[0, 0, h] @ k[0, 0, 0])) < 1e-14


def pin_merge_splits(A):
    """Merging the partials of any split of the key range (empty parts included) gives the
    unsplit result; the merge is order-independent and associative."""
    r = rng(5)
    B, Hq, Hkv, D, T = 2, 4, 2, 8, 37
    q = r.standard_normal((B, 1, Hq, D))
    k = r.standard_normal((B, T, Hkv, D))
    v = r.standard_normal((B, T, Hkv, D))
    o_ref, l_ref = A.attention(q, k, v, scale=0.35, causal=False)
    for cuts in ([0, 10, 10, 25, 37], [0, 37], [0, 1, 2, 3, 36, 37], [0, 0, 37, 37]):
        po, pl = [], []
        for a, bnd in zip(cuts[:-1], cuts[1:]):
            o, lse = A.attention(q, k[:, a:bnd], v[:, a:bnd], scale=0.35, causal=False)
            po.append(o)
            pl.append(lse.transpose(0, 2, 1))  # [B, Hq, R] -> [B, R, Hq], the rows of o
        mo, ml = A.merge_lse(np.stack(po), np.stack(pl))
        np.testing.assert_allclose(mo, o_ref, atol=1e-12)
        np.testing.assert_allclose(ml, l_ref.transpose(0, 2, 1), atol=1e-12)
        perm = r.permutation(len(po))
        mo2, ml2 = A.merge_lse(np.stack([po[i] for i in perm]), np.stack([pl[i] for i in perm]))
        np.testing.assert_allclose(mo2, mo, atol=1e-12)
        np.testing.assert_allclose(ml2, ml, atol=1e-12)
        if len(po) >= 3:
            ao, al = A.merge_lse(np.stack(po[:2]), np.stack(pl[:2]))
            bo, bl = A.merge_lse(np.stack([ao] + po[2:]), np.stack([al] + pl[2:]))
            np.testing.assert_allclose(bo, mo, atol=1e-12)
            np.testing.assert_allclose(bl, ml, atol=1e-12)
    # all-empty rows
    mo, ml = A.merge_lse(np.zeros((3, 2, 4)), np.full((3, 2), -np.inf))
    assert np.all(mo == 0) and np.all(np.isneginf(ml))


def pin_gqa_equals_mha(A):
    r = rng(6)
    B, S, Hq, Hkv, D = 1, 9, 6, 2, 4
    q = r.standard_normal((B, S, Hq, D))
    k = r.standard_normal((B, S, Hkv, D))
    v = r.standard_normal((B, S, Hkv, D))
    o, lse = A.attention(q, k, v, scale=0.5, causal=True)
    G = Hq // Hkv
    o2, lse2 = A.attention(q, np.repeat(k, G, axis=2), np.repeat(v, G, axis=2), scale=0.5, causal=True)
    np.testing.assert_allclose(o, o2, atol=1e-13)
    np.testing.assert_allclose(lse, lse2, atol=1e-13)


def pin_affine_v(A):
    r = rng(7)
    q = r.standard_normal((1, 7, 2, 4))
    k = r.standard_normal((1, 7, 2, 4))
    v = r.standard_normal((1, 7, 2, 4))
    o, lse = A.attention(q, k, v, scale=0.5, causal=True)
    o2, lse2 = A.attention(q, k, 3.0 * v - 1.25, scale=0.5, causal=True)
    np.testing.assert_allclose(o2, 3.0 * o - 1.25, atol=1e-12)
    np.testing.assert_allclose(lse2, lse, atol=0)


def pin_decode_is_last_prefill_row(A):
    r = rng(8)
    B, T, Hq, Hkv, D = 2, 11, 4, 2, 8
    q = r.standard_normal((B, T, Hq, D))
    k = r.standard_normal((B, T, Hkv, D))
    v = r.standard_normal((B, T, Hkv, D))
    op, lp = A.attention(q, k, v, scale=0.3, causal=True)
    for t in (0, 5, T - 1):
        od, ld = A.decode(q[:, t], k, v, np.array([t + 1] * B), scale=0.3)
        np.testing.assert_allclose(od, op[:, t], atol=1e-12)
        np.testing.assert_allclose(ld, lp[:, :, t], atol=1e-12)


def pin_empty_sequence(A):
    r = rng(9)
    q = r.standard_normal((2, 4, 8))
    k = r.standard_normal((2, 5, 2, 8))
    v = r.standard_normal((2, 5, 2, 8))
    o, lse = A.decode(q, k, v, np.array([0, 5]), scale=0.3)
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(lse[1]))


def pin_dequant_scales(A):
    """Per-token scales multiply K and V rows; scale on K is a score factor per key."""
    r = rng(10)
    q = r.standard_normal((1, 3, 2, 4))
    k = r.standard_normal((1, 5, 1, 4))
    v = r.standard_normal((1, 5, 1, 4))
    ks = r.uniform(0.5, 2.0, (1, 5, 1))
    vs = r.uniform(0.5, 2.0, (1, 5, 1))
    o, lse = A.attention(q, k, v, scale=0.5, causal=False, k_scale=ks, v_scale=vs)
    o2, lse2 = A.attention(q, k * ks[..., None], v * vs[..., None], scale=0.5, causal=False)
    np.testing.assert_allclose(o, o2, atol=1e-13)
    np.testing.assert_allclose(lse, lse2, atol=1e-13)


ATTENTION_PINS = [pin_golden, pin_brute_force, pin_sdpa, pin_uniform_scores, pin_dominant_key,
                  pin_single_visible_key, pin_merge_splits, pin_gqa_equals_mha, pin_affine_v,
                  pin_decode_is_last_prefill_row, pin_empty_sequence, pin_dequant_scales]
