"""Pins of the packed variable-length prefill oracle."""
import math

import numpy as np
import torch

from exact_long_context_tmem_b200 import inputs as I
from oracle import attention as O


def _packed(pairs, Hq, Hkv, D, seed):
    g = I.generator(seed)
    tq, tk = sum(p[0] for p in pairs), sum(p[1] for p in pairs)
    q = I.randn_bf16((tq, Hq, D), g)
    k = I.randn_bf16((tk, Hkv, D), g)
    v = I.randn_bf16((tk, Hkv, D), g)
    cu_q = np.concatenate([[0], np.cumsum([p[0] for p in pairs])]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum([p[1] for p in pairs])]).astype(np.int32)
    return q, k, v, cu_q, cu_k


def test_brute_force_scalar_loops():
    pairs = [(3, 5), (2, 2), (0, 3), (4, 4), (2, 0)]
    Hq, Hkv, D = 4, 2, 4
    q, k, v, cu_q, cu_k = _packed(pairs, Hq, Hkv, D, 3)
    scale = 0.37
    o, lse = O.prefill_varlen(q, k, v, cu_q, cu_k, scale=scale, causal=True)
    qf, kf, vf = q.double().numpy(), k.double().numpy(), v.double().numpy()
    for b, (sq, sk) in enumerate(pairs):
        for i in range(sq):
            row = cu_q[b] + i
            pos = sk - sq + i
            for h in range(Hq):
                kvh = h // (Hq // Hkv)
                vis = [j for j in range(sk) if j <= pos]
                if not vis:
                    assert np.all(o[row, h] == 0) and lse[row, h] == -np.inf
                    continue
                s = [scale * sum(qf[row, h, d] * kf[cu_k[b] + j, kvh, d] for d in range(D)) for j in vis]
                mx = max(s)
                den = sum(math.exp(x - mx) for x in s)
                assert abs(lse[row, h] - (mx + math.log(den))) < 1e-12
                for d in range(D):
                    num = sum(math.exp(x - mx) * vf[cu_k[b] + j, kvh, d] for x, j in zip(s, vis))
                    assert abs(o[row, h, d] - num / den) < 1e-12


def test_order_of_sequences_does_not_matter():
    pairs = [(5, 9), (3, 3), (7, 12)]
    q, k, v, cu_q, cu_k = _packed(pairs, 4, 2, 8, 5)
    o, lse = O.prefill_varlen(q, k, v, cu_q, cu_k, scale=0.3, causal=True)
    order = [2, 0, 1]
    qs = torch.cat([q[cu_q[b]:cu_q[b + 1]] for b in order])
    ks = torch.cat([k[cu_k[b]:cu_k[b + 1]] for b in order])
    vs = torch.cat([v[cu_k[b]:cu_k[b + 1]] for b in order])
    cq = np.concatenate([[0], np.cumsum([pairs[b][0] for b in order])])
    ck = np.concatenate([[0], np.cumsum([pairs[b][1] for b in order])])
    o2, l2 = O.prefill_varlen(qs, ks, vs, cq, ck, scale=0.3, causal=True)
    o_back = np.concatenate([o[cu_q[b]:cu_q[b + 1]] for b in order])
    l_back = np.concatenate([lse[cu_q[b]:cu_q[b + 1]] for b in order])
    np.testing.assert_array_equal(o2, o_back)
    np.testing.assert_array_equal(l2, l_back)


def test_single_sequence_is_dense_prefill_with_past():
    q, k, v, cu_q, cu_k = _packed([(6, 10)], 4, 4, 8, 9)
    o, lse = O.prefill_varlen(q, k, v, cu_q, cu_k, scale=0.25, causal=True)
    od, ld = O.attention(q[None], k[None], v[None], scale=0.25, causal=True, q_pos0=4)
    np.testing.assert_array_equal(o, np.asarray(od)[0])
    np.testing.assert_array_equal(lse, np.asarray(ld)[0].T)
