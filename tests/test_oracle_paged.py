"""Pins of the paged-decode oracle (LLM-CoOpt summary, "Opt-Pa") against things it must equal."""
import math

import numpy as np
import pytest
import torch

from exact_long_context_tmem_b200 import inputs as I
from oracle import attention as O
from oracle import fp8 as F
from oracle import paged as PG


def _small(fp8=False, lens=(700, 0, 1, 512, 1024), Tmax=1100, seed=5):
    w = I.Workload("paged_small", "decode", B=len(lens), Hq=8, Hkv=2, D=16, kv_fp8=fp8, seed=seed)
    return w, I.decode_inputs(w, lens=torch.tensor(lens, dtype=torch.int32), Tmax=Tmax)


def test_gather_by_hand():
    # two sequences, page size 2; pool pages hold their own index in every slot
    pool = torch.arange(5, dtype=torch.float64)[:, None, None, None].expand(5, 2, 1, 1).clone()
    table = torch.tensor([[3, 0, -1], [4, 1, 2]])
    got = PG.gather(pool, table, torch.tensor([3, 6]), 2)
    assert got[0, :3, 0, 0].tolist() == [3, 3, 0]
    assert torch.isnan(got[0, 3:]).all()
    assert got[1, :, 0, 0].tolist() == [4, 4, 1, 1, 2, 2]


@pytest.mark.parametrize("page_size", [128, 512])
def test_identity_table_equals_contiguous(page_size):
    w, d = _small()
    B, Tmax = d["k"].shape[:2]
    mp = (Tmax + page_size - 1) // page_size
    pad = torch.full((B, mp * page_size - Tmax) + tuple(d["k"].shape[2:]), float("nan"), dtype=d["k"].dtype)
    kp = torch.cat([d["k"], pad], 1).reshape(B * mp, page_size, *d["k"].shape[2:])
    vp = torch.cat([d["v"], pad], 1).reshape(B * mp, page_size, *d["v"].shape[2:])
    table = torch.arange(B * mp, dtype=torch.int32).reshape(B, mp)
    o1, l1 = PG.decode_paged(d["q"], kp, vp, table, d["kv_lens"], page_size, scale=w.scale)
    o2, l2 = O.decode(d["q"], d["k"], d["v"], d["kv_lens"], scale=w.scale)
    np.testing.assert_array_equal(np.asarray(o1), np.asarray(o2))
    np.testing.assert_array_equal(np.asarray(l1), np.asarray(l2))


@pytest.mark.parametrize("fp8", [False, True])
def test_permuted_pool_equals_contiguous(fp8):
    w, d = _small(fp8=fp8)
    pd = I.paged_inputs(d, 128, seed=11)
    assert (pd["page_table"] >= -1).all() and pd["num_pages"] > int((pd["page_table"] >= 0).sum())
    if fp8:
        o1, l1 = PG.decode_paged(pd["q"], F.e4m3_decode(pd["k_codes"]), F.e4m3_decode(pd["v_codes"]),
                                 pd["page_table"], pd["kv_lens"], 128, scale=w.scale,
                                 k_scale_pool=pd["k_scale"], v_scale_pool=pd["v_scale"])
        o2, l2 = O.decode(d["q"], F.e4m3_decode(d["k_codes"]), F.e4m3_decode(d["v_codes"]), d["kv_lens"],
                          scale=w.scale, k_scale=d["k_scale"], v_scale=d["v_scale"])
    else:
        o1, l1 = PG.decode_paged(pd["q"], pd["k"], pd["v"], pd["page_table"], pd["kv_lens"], 128, scale=w.scale)
        o2, l2 = O.decode(d["q"], d["k"], d["v"], d["kv_lens"], scale=w.scale)
    # spare pages and padding are NaN: a read of any of them would show here
    assert np.isfinite(np.asarray(o1)).all()
    np.testing.assert_array_equal(np.asarray(o1), np.asarray(o2))
    np.testing.assert_array_equal(np.asarray(l1), np.asarray(l2))


def test_swapped_entries_change_the_result():
    w, d = _small(lens=(600,), Tmax=640)
    pd = I.paged_inputs(d, 128, seed=3)
    t2 = pd["page_table"].clone()
    t2[0, 0], t2[0, 1] = pd["page_table"][0, 1], pd["page_table"][0, 0]
    o1, _ = PG.decode_paged(pd["q"], pd["k"], pd["v"], pd["page_table"], pd["kv_lens"], 128, scale=w.scale)
    o2, _ = PG.decode_paged(pd["q"], pd["k"], pd["v"], t2, pd["kv_lens"], 128, scale=w.scale)
    # the softmax over a permuted key set is the same; K and V pages move together, so swap only K
    o3, _ = PG.decode_paged(pd["q"], pd["k"], pd["v"], pd["page_table"], pd["kv_lens"], 128, scale=w.scale)
    np.testing.assert_allclose(np.asarray(o1), np.asarray(o2), rtol=1e-12, atol=1e-12)
    k_only = PG.gather(pd["k"], t2, pd["kv_lens"], 128)
    v_ref = PG.gather(pd["v"], pd["page_table"], pd["kv_lens"], 128)
    o4, _ = O.decode(pd["q"], k_only, v_ref, pd["kv_lens"], scale=w.scale)
    assert np.abs(np.asarray(o4) - np.asarray(o3)).max() > 1e-3


def test_unmapped_page_below_length_is_an_error():
    w, d = _small(lens=(300,), Tmax=384)
    pd = I.paged_inputs(d, 128, seed=1)
    pd["page_table"][0, 1] = -1
    with pytest.raises(AssertionError):
        PG.gather(pd["k"], pd["page_table"], pd["kv_lens"], 128)
