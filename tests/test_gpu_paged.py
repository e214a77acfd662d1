"""GPU parity of the paged decode (LLM-CoOpt summary, "Opt-Pa") against the paged oracle, and
bit-equality with the contiguous-cache kernel on the same data."""
import numpy as np
import pytest
import torch

from exact_long_context_tmem_b200 import attn as A
from exact_long_context_tmem_b200 import inputs as I
from oracle import fp8 as F
from oracle import paged as PG
from tests.parity import assert_lse_close, assert_o_close, device_clean

pytestmark = pytest.mark.gpu


def _case(lens, Tmax, fp8, Hq=32, Hkv=8, seed=41):
    w = I.Workload("paged_gpu", "decode", B=len(lens), Hq=Hq, Hkv=Hkv, D=128, kv_fp8=fp8, seed=seed)
    return w, I.decode_inputs(w, lens=torch.tensor(lens, dtype=torch.int32), Tmax=Tmax)


def _run_paged(pd, dev, splits):
    q, lens, table = pd["q"].to(dev), pd["kv_lens"].to(dev), pd["page_table"].to(dev)
    if "k_codes" in pd:
        return A.attn_decode_paged(q, pd["k_codes"].to(dev), pd["v_codes"].to(dev), table, lens,
                                   k_scale=pd["k_scale"].to(dev), v_scale=pd["v_scale"].to(dev), num_splits=splits)
    return A.attn_decode_paged(q, pd["k"].to(dev), pd["v"].to(dev), table, lens, num_splits=splits)


def _run_contig(d, dev, splits):
    q, lens = d["q"].to(dev), d["kv_lens"].to(dev)
    if "k_codes" in d:
        return A.attn_decode_splitkv(q, d["k_codes"].to(dev), d["v_codes"].to(dev), lens,
                                     k_scale=d["k_scale"].to(dev), v_scale=d["v_scale"].to(dev), num_splits=splits)
    return A.attn_decode_splitkv(q, d["k"].to(dev), d["v"].to(dev), lens, num_splits=splits)


def _ref(pd, w):
    ps = pd["page_size"]
    if "k_codes" in pd:
        return PG.decode_paged(pd["q"], F.e4m3_decode(pd["k_codes"]), F.e4m3_decode(pd["v_codes"]), pd["page_table"],
                               pd["kv_lens"], ps, scale=w.scale, k_scale_pool=pd["k_scale"], v_scale_pool=pd["v_scale"])
    return PG.decode_paged(pd["q"], pd["k"], pd["v"], pd["page_table"], pd["kv_lens"], ps, scale=w.scale)


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("page_size", [128, 512])
def test_paged_matches_oracle_and_contiguous(cuda_device, fp8, page_size):
    lens = [3000, 0, 1, 512, 1024, 2049]
    w, d = _case(lens, 3072, fp8)
    pd = I.paged_inputs(d, page_size, seed=page_size + int(fp8))
    ro, rl = _ref(pd, w)
    for splits in (1, 3, 0):
        o, lse = _run_paged(pd, cuda_device, splits)
        torch.cuda.synchronize()
        assert_o_close(o, ro)
        assert_lse_close(lse, rl)
        assert torch.all(o[1] == 0) and torch.all(torch.isneginf(lse[1]))
        oc, lc = _run_contig(d, cuda_device, splits)
        torch.cuda.synchronize()
        # same splits, same arithmetic: only the addresses differ
        assert torch.equal(o, oc) and torch.equal(lse, lc)
    device_clean()


def test_paged_fp8_many_items(cuda_device):
    """More (split, head, sequence) items than SMs, so each persistent CTA walks several
    sequences and their pages back to back."""
    g = np.random.default_rng(9)
    lens = g.integers(0, 2049, size=48).tolist()
    lens[:3] = [0, 2048, 129]
    w, d = _case(lens, 2048, True, Hq=16, Hkv=4, seed=9)
    pd = I.paged_inputs(d, 512, seed=2)
    ro, rl = _ref(pd, w)
    o, lse = _run_paged(pd, cuda_device, 4)
    torch.cuda.synchronize()
    assert_o_close(o, ro)
    assert_lse_close(lse, rl)
    device_clean()


@pytest.mark.parametrize("fp8", [False, True])
def test_bad_page_entry_reads_zeros_and_is_reported(cuda_device, fp8):
    w, d = _case([1000], 1024, fp8)
    pd = I.paged_inputs(d, 128, seed=4)
    pd["page_table"][0, 2] = pd["num_pages"] + 5  # outside the pool: never dereferenced
    o, lse = _run_paged(pd, cuda_device, 1)
    torch.cuda.synchronize()
    st, site = A.attn_device_status(reset=True)
    assert st == A.ATTN_ERR_INVALID_ARG and site == 44
    assert torch.isfinite(o).all()
