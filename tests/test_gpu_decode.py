"""GPU parity of the split-KV decode kernels (bf16 and FP8 E4M3 caches) against the oracle."""
import math

import numpy as np
import pytest
import torch

from exact_long_context_tmem_b200 import attn as A
from exact_long_context_tmem_b200 import inputs as I
from oracle import attention as O
from oracle import fp8 as F
from tests.parity import assert_lse_close, assert_o_close, device_clean

pytestmark = pytest.mark.gpu


def _run(d, dev, num_splits=0, fp8=False):
    q = d["q"].to(dev)
    lens = d["kv_lens"].to(dev)
    if fp8:
        o, lse = A.attn_decode_splitkv(q, d["k_codes"].to(dev), d["v_codes"].to(dev), lens,
                                       k_scale=d["k_scale"].to(dev), v_scale=d["v_scale"].to(dev),
                                       num_splits=num_splits)
    else:
        o, lse = A.attn_decode_splitkv(q, d["k"].to(dev), d["v"].to(dev), lens, num_splits=num_splits)
    torch.cuda.synchronize()
    return o, lse


def _ref(d, scale, fp8=False):
    if fp8:
        return O.decode(d["q"], F.e4m3_decode(d["k_codes"]), F.e4m3_decode(d["v_codes"]), d["kv_lens"],
                        scale=scale, k_scale=d["k_scale"], v_scale=d["v_scale"])
    return O.decode(d["q"], d["k"], d["v"], d["kv_lens"], scale=scale)


def _small(B, Hq, Hkv, lens, Tmax, seed, fp8=False):
    w = I.Workload("decode_small", "decode", B=B, Hq=Hq, Hkv=Hkv, D=128, kv_fp8=fp8, seed=seed)
    return w, I.decode_inputs(w, lens=torch.tensor(lens, dtype=torch.int32), Tmax=Tmax)


@pytest.mark.parametrize("splits", [1, 3, 0])
def test_decode_bf16_ragged_with_nan_padding(cuda_device, splits):
    w, d = _small(3, 8, 2, [1000, 0, 777], 1024, seed=21)
    o, lse = _run(d, cuda_device, splits)
    ro, rl = _ref(d, w.scale)
    assert_o_close(o, ro)
    assert_lse_close(lse, rl)
    assert torch.all(o[1] == 0) and torch.all(torch.isneginf(lse[1]))
    device_clean()


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (16, 16), (12, 1), (6, 3), (64, 8), (32, 2)])
def test_decode_bf16_groups(cuda_device, Hq, Hkv):
    w, d = _small(2, Hq, Hkv, [1, 2049], 2100, seed=Hq * 10 + Hkv)
    for splits in (1, 5):
        o, lse = _run(d, cuda_device, splits)
        ro, rl = _ref(d, w.scale)
        assert_o_close(o, ro)
        assert_lse_close(lse, rl)
    device_clean()


@pytest.mark.parametrize("splits", [1, 4, 0])
def test_decode_fp8_small(cuda_device, splits):
    w, d = _small(2, 32, 8, [513, 1024], 1024, seed=31, fp8=True)
    o, lse = _run(d, cuda_device, splits, fp8=True)
    ro, rl = _ref(d, w.scale, fp8=True)
    assert_o_close(o, ro)
    assert_lse_close(lse, rl)
    device_clean()


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (16, 16), (12, 1), (6, 3), (64, 8), (32, 2)])
def test_decode_fp8_groups(cuda_device, Hq, Hkv):
    w, d = _small(2, Hq, Hkv, [1, 2049], 2100, seed=Hq * 10 + Hkv + 500, fp8=True)
    for splits in (1, 5):
        o, lse = _run(d, cuda_device, splits, fp8=True)
        ro, rl = _ref(d, w.scale, fp8=True)
        assert_o_close(o, ro)
        assert_lse_close(lse, rl)
    device_clean()


def test_decode_fp8_many_items_ragged(cuda_device):
    """More (split, head, sequence) items than SMs: each persistent CTA runs several items back to
    back, with empty, one-token and exact-tile splits among them."""
    g = np.random.default_rng(77)
    lens = g.integers(0, 1501, size=40)
    lens[:6] = [0, 1, 1500, 128, 129, 0]
    w, d = _small(40, 8, 2, lens.tolist(), 1500, seed=77, fp8=True)
    for splits in (4, 1):
        o, lse = _run(d, cuda_device, splits, fp8=True)
        ro, rl = _ref(d, w.scale, fp8=True)
        assert_o_close(o, ro)
        assert_lse_close(lse, rl)
        assert torch.all(o[0] == 0) and torch.all(torch.isneginf(lse[0]))
    device_clean()


@pytest.mark.parametrize("fp8", [False, True])
def test_decode_rescale_ramp(cuda_device, fp8):
    """Key magnitudes grow along the sequence, so the running maximum rises by more than the lazy
    threshold on almost every tile and O^T is rescaled again and again."""
    Tmax = 2000
    w, d = _small(2, 32, 8, [2000, 1700], Tmax, seed=91, fp8=fp8)
    ramp = 1.0 + torch.arange(Tmax, dtype=torch.float32) / 32.0
    if fp8:
        d["k_scale"] = d["k_scale"] * ramp[None, :, None]
    else:
        d["k"] = (d["k"].float() * ramp[None, :, None, None]).to(torch.bfloat16)
    for splits in (1, 3):
        o, lse = _run(d, cuda_device, splits, fp8=fp8)
        ro, rl = _ref(d, w.scale, fp8=fp8)
        assert_o_close(o, ro)
        assert_lse_close(lse, rl)
    device_clean()


def test_decode_matches_prefill_last_row(cuda_device):
    """Decode of token t equals row t of a causal prefill over the same cache."""
    g = I.generator(41)
    T, Hq, Hkv, D = 700, 8, 2, 128
    q = I.randn_bf16((1, T, Hq, D), g)
    k = I.randn_bf16((1, T, Hkv, D), g)
    v = I.randn_bf16((1, T, Hkv, D), g)
    po, pl = A.attn_prefill(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), causal=True)
    lens = torch.tensor([T], dtype=torch.int32, device=cuda_device)
    do_, dl = A.attn_decode_splitkv(q[:, T - 1].contiguous().to(cuda_device), k.to(cuda_device),
                                    v.to(cuda_device), lens, num_splits=3)
    torch.cuda.synchronize()
    np.testing.assert_allclose(do_.float().cpu().numpy(), po[:, T - 1].float().cpu().numpy(), atol=2e-2, rtol=2e-2)
    np.testing.assert_allclose(dl.cpu().numpy(), pl[:, T - 1].cpu().numpy(), atol=1e-3)
    device_clean()


@pytest.mark.slow
def test_decode_b4_ragged_64k_128k_full(cuda_device):
    w = I.WORKLOADS["decode_b4_h32g8_d128_ragged64k_128k"]
    d = I.decode_inputs(w)
    o, lse = _run(d, cuda_device, 0)
    ro, rl = _ref(d, w.scale)
    assert_o_close(o, ro)
    assert_lse_close(lse, rl)
    device_clean()


@pytest.mark.slow
def test_decode_fp8_b16_t32768_full(cuda_device):
    w = I.WORKLOADS["decode_fp8_b16_h32g8_d128_t32768"]
    d = I.decode_inputs(w)
    o, lse = _run(d, cuda_device, 0, fp8=True)
    ro, rl = _ref(d, w.scale, fp8=True)
    assert_o_close(o, ro)
    assert_lse_close(lse, rl)
    device_clean()
