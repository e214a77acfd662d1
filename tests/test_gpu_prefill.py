"""GPU parity of the tcgen05 prefill kernel against the float64 oracle."""
import math

import numpy as np
import pytest
import torch

from exact_long_context_tmem_b200 import attn as A
from exact_long_context_tmem_b200 import inputs as I
from oracle import attention as O
from tests.parity import assert_lse_close, assert_o_close, device_clean, to_np

pytestmark = pytest.mark.gpu


def _gen(B, S, T, Hq, Hkv, D, seed):
    g = I.generator(seed)
    q = I.randn_bf16((B, S, Hq, D), g)
    k = I.randn_bf16((B, T, Hkv, D), g)
    v = I.randn_bf16((B, T, Hkv, D), g)
    return q, k, v


def _check(q, k, v, dev, causal, q_pos0=0, kv_pos0=0, rows=None, out_dtype=torch.bfloat16, scale=None):
    D = q.shape[-1]
    scale = 1 / math.sqrt(D) if scale is None else scale
    o, lse = A.attn_prefill(q.to(dev), k.to(dev), v.to(dev), causal=causal, q_pos0=q_pos0, kv_pos0=kv_pos0,
                            out_dtype=out_dtype, scale=scale)
    torch.cuda.synchronize()
    ro, rl = O.attention(q, k, v, scale=scale, causal=causal, q_pos0=q_pos0, kv_pos0=kv_pos0, rows=rows)
    go, gl = o, lse
    if rows is not None:
        go, gl = o[:, rows], lse[:, rows]
    eo = assert_o_close(go, ro)
    el = assert_lse_close(to_np(gl).transpose(0, 2, 1), rl)
    device_clean()
    return eo, el


def test_prefill_small_causal_gqa_d64(cuda_device):
    w = I.WORKLOADS["prefill_b1_h4g2_d64_s256"]
    q, k, v = I.prefill_inputs(w)
    _check(q, k, v, cuda_device, causal=True)


@pytest.mark.parametrize("B,S,T,Hq,Hkv,D,causal", [
    (1, 300, 300, 8, 2, 128, True),     # ragged tail tile, group 4
    (2, 200, 333, 4, 4, 128, False),    # non-causal, MHA (group 1: consecutive query tiles pair up)
    (1, 129, 129, 6, 2, 64, True),      # group 3 (odd), one row in the last tile
    (1, 1, 1, 2, 1, 128, True),         # single query, single key
    (2, 64, 700, 2, 2, 64, False),      # fewer queries than one tile, several key tiles
    (1, 640, 640, 16, 8, 128, True),    # five query tiles, group 2
])
def test_prefill_shapes(cuda_device, B, S, T, Hq, Hkv, D, causal):
    q, k, v = _gen(B, S, T, Hq, Hkv, D, seed=S * 7 + T)
    _check(q, k, v, cuda_device, causal)


def test_prefill_position_offsets(cuda_device):
    """Queries at positions 256..511 over keys 0..511 (a later query block against one chunk)."""
    q, k, v = _gen(1, 256, 512, 8, 2, 128, seed=5)
    _check(q, k, v, cuda_device, causal=True, q_pos0=256, kv_pos0=0)
    # a key chunk that starts after some queries: early rows see nothing (O = 0, LSE = -inf)
    _check(q, k, v, cuda_device, causal=True, q_pos0=100, kv_pos0=200)


def test_prefill_f32_out_and_scale(cuda_device):
    q, k, v = _gen(1, 384, 384, 4, 2, 128, seed=6)
    _check(q, k, v, cuda_device, causal=True, out_dtype=torch.float32, scale=0.05)


def test_prefill_no_keys(cuda_device):
    q, k, v = _gen(1, 130, 1, 4, 2, 128, seed=7)
    o, lse = A.attn_prefill(q.to(cuda_device), k[:, :0].contiguous().to(cuda_device),
                            v[:, :0].contiguous().to(cuda_device), causal=True)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
    device_clean()


def test_prefill_large_rescale(cuda_device):
    """Scores that grow along the key axis force the lazy O rescale many times."""
    q, k, v = _gen(1, 256, 1024, 4, 2, 128, seed=8)
    ramp = torch.linspace(0.1, 6.0, 1024).view(1, 1024, 1, 1)
    k = (k.float() * ramp).to(torch.bfloat16)
    q = (q.float() * 2).to(torch.bfloat16)
    _check(q, k, v, cuda_device, causal=False)


@pytest.mark.slow
def test_prefill_b2_h32_d128_s8192_sampled(cuda_device):
    """The full-size causal prefill workload, checked on sampled rows (all heads)."""
    w = I.WORKLOADS["prefill_b2_h32g8_d128_s8192"]
    q, k, v = I.prefill_inputs(w)
    rows = I.sample_rows(w.S, 48, seed=77, edges=(0, 1, 127, 128, 4095, 4096, 8191))
    _check(q, k, v, cuda_device, causal=True, rows=rows)
