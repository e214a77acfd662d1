"""GPU parity of multi-token decode (n_q query tokens per sequence over one cache pass)."""
import numpy as np
import pytest
import torch

from exact_long_context_tmem_b200 import attn as A
from exact_long_context_tmem_b200 import inputs as I
from oracle import attention as O
from oracle import fp8 as F
from tests.parity import assert_lse_close, assert_o_close, device_clean

pytestmark = pytest.mark.gpu


def _case(lens, Tmax, n_q, fp8, Hq, Hkv, seed):
    w = I.Workload("multi_gpu", "decode", B=len(lens), Hq=Hq, Hkv=Hkv, D=128, kv_fp8=fp8, seed=seed)
    d = I.decode_inputs(w, lens=torch.tensor(lens, dtype=torch.int32), Tmax=Tmax)
    q = I.randn_bf16((len(lens), n_q, Hq, 128), I.generator(seed + 100))
    return w, d, q


def _run(d, q, dev, splits):
    lens = d["kv_lens"].to(dev)
    if "k_codes" in d:
        return A.attn_decode_multi(q.to(dev), d["k_codes"].to(dev), d["v_codes"].to(dev), lens,
                                   k_scale=d["k_scale"].to(dev), v_scale=d["v_scale"].to(dev), num_splits=splits)
    return A.attn_decode_multi(q.to(dev), d["k"].to(dev), d["v"].to(dev), lens, num_splits=splits)


def _ref(w, d, q):
    if "k_codes" in d:
        return O.decode_multi(q, F.e4m3_decode(d["k_codes"]), F.e4m3_decode(d["v_codes"]), d["kv_lens"],
                              scale=w.scale, k_scale=d["k_scale"], v_scale=d["v_scale"])
    return O.decode_multi(q, d["k"], d["v"], d["kv_lens"], scale=w.scale)


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("n_q,Hq,Hkv", [(2, 32, 8), (4, 32, 8), (2, 64, 8), (3, 12, 4), (16, 8, 8)])
def test_multi_token_decode(cuda_device, fp8, n_q, Hq, Hkv):
    lens = [2049, 1, 0, 700, n_q, 128]
    w, d, q = _case(lens, 2100, n_q, fp8, Hq, Hkv, seed=7 * n_q + Hq)
    ro, rl = _ref(w, d, q)
    for splits in (1, 3, 0):
        o, lse = _run(d, q, cuda_device, splits)
        torch.cuda.synchronize()
        assert_o_close(o, ro)
        assert_lse_close(lse, rl)
    device_clean()


@pytest.mark.parametrize("fp8", [False, True])
def test_last_token_matches_single_token_decode(cuda_device, fp8):
    n_q = 4
    w, d, q = _case([3000, 1500, 64], 3072, n_q, fp8, 32, 8, seed=3)
    o, lse = _run(d, q, cuda_device, 0)
    lens = d["kv_lens"].to(cuda_device)
    qs = q[:, -1].contiguous().to(cuda_device)
    if fp8:
        o1, l1 = A.attn_decode_splitkv(qs, d["k_codes"].to(cuda_device), d["v_codes"].to(cuda_device), lens,
                                       k_scale=d["k_scale"].to(cuda_device), v_scale=d["v_scale"].to(cuda_device))
    else:
        o1, l1 = A.attn_decode_splitkv(qs, d["k"].to(cuda_device), d["v"].to(cuda_device), lens)
    torch.cuda.synchronize()
    assert (o[:, -1].float() - o1.float()).abs().max().item() <= 2e-2
    assert (lse[:, -1] - l1).abs().max().item() <= 1e-3
    device_clean()
