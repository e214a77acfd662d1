"""Pins of the multi-token decode oracle against single-token decodes of the same cache."""
import numpy as np
import torch

from exact_long_context_tmem_b200 import inputs as I
from oracle import attention as O
from oracle import fp8 as F


def _case(lens, Tmax, n_q, fp8=False, Hq=8, Hkv=2, seed=13):
    w = I.Workload("multi_small", "decode", B=len(lens), Hq=Hq, Hkv=Hkv, D=16, kv_fp8=fp8, seed=seed)
    d = I.decode_inputs(w, lens=torch.tensor(lens, dtype=torch.int32), Tmax=Tmax)
    g = I.generator(seed + 1)
    q = I.randn_bf16((len(lens), n_q, Hq, 16), g)
    return w, d, q


def test_one_token_is_decode():
    w, d, q = _case([50, 7, 64], 64, 1)
    o1, l1 = O.decode_multi(q, d["k"], d["v"], d["kv_lens"], scale=w.scale)
    o2, l2 = O.decode(q[:, 0], d["k"], d["v"], d["kv_lens"], scale=w.scale)
    np.testing.assert_array_equal(o1[:, 0], np.asarray(o2))
    np.testing.assert_array_equal(l1[:, 0], np.asarray(l2))


def test_each_token_is_a_decode_over_its_prefix():
    n_q = 4
    w, d, q = _case([50, 9, 64], 64, n_q)
    o, lse = O.decode_multi(q, d["k"], d["v"], d["kv_lens"], scale=w.scale)
    for i in range(n_q):
        lens_i = d["kv_lens"] - n_q + i + 1
        oi, li = O.decode(q[:, i], d["k"], d["v"], lens_i, scale=w.scale)
        np.testing.assert_allclose(o[:, i], np.asarray(oi), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[:, i], np.asarray(li), rtol=1e-12, atol=1e-12)


def test_fp8_scales_follow_the_tokens():
    n_q = 2
    w, d, q = _case([40, 33], 48, n_q, fp8=True)
    k, v = F.e4m3_decode(d["k_codes"]), F.e4m3_decode(d["v_codes"])
    o, lse = O.decode_multi(q, k, v, d["kv_lens"], scale=w.scale, k_scale=d["k_scale"], v_scale=d["v_scale"])
    for i in range(n_q):
        oi, li = O.decode(q[:, i], k, v, d["kv_lens"] - n_q + i + 1, scale=w.scale,
                          k_scale=d["k_scale"], v_scale=d["v_scale"])
        np.testing.assert_allclose(o[:, i], np.asarray(oi), rtol=1e-12, atol=1e-12)


def test_token_without_keys_is_empty():
    w, d, q = _case([1, 0], 8, 2)
    o, lse = O.decode_multi(q, d["k"], d["v"], d["kv_lens"], scale=w.scale)
    assert np.all(o[0, 0] == 0) and np.all(np.isneginf(lse[0, 0]))   # position -1: nothing visible
    assert np.all(np.isfinite(lse[0, 1]))                           # position 0 sees key 0
    assert np.all(o[1] == 0) and np.all(np.isneginf(lse[1]))
