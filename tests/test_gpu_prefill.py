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


def _check_views(qv, kv, vv, dev, causal=True, o=None, scale=None):
    """attn_prefill on strided views (read in place through the strides argument) against the
    oracle on packed copies of the same values."""
    D = qv.shape[-1]
    scale = 1 / math.sqrt(D) if scale is None else scale
    o, lse = A.attn_prefill(qv, kv, vv, causal=causal, o=o, scale=scale)
    torch.cuda.synchronize()
    ro, rl = O.attention(qv.cpu().contiguous(), kv.cpu().contiguous(), vv.cpu().contiguous(), scale=scale,
                         causal=causal)
    assert_o_close(o, ro)
    assert_lse_close(to_np(lse).transpose(0, 2, 1), rl)
    device_clean()
    return o


def test_prefill_fused_qkv_views(cuda_device):
    """Q, K and V as slices of one fused [B, S, Hq + 2 Hkv, D] tensor (packed QKV), ragged length."""
    B, S, Hq, Hkv, D = 2, 300, 8, 2, 128
    g = I.generator(21)
    qkv = I.randn_bf16((B, S, Hq + 2 * Hkv, D), g).to(cuda_device)
    q, k, v = qkv[:, :, :Hq], qkv[:, :, Hq:Hq + Hkv], qkv[:, :, Hq + Hkv:]
    assert not q.is_contiguous() and not k.is_contiguous()
    _check_views(q, k, v, cuda_device)


def test_prefill_head_subset_and_bhsd_views(cuda_device):
    """Every other head of a wider tensor (head stride 2D), and K/V stored [B, H, T, D] and seen as
    [B, T, H, D] (token stride D, head stride T*D); D = 64, non-causal, 5 key tiles."""
    B, S, T, Hq, Hkv, D = 1, 200, 600, 4, 2, 64
    g = I.generator(22)
    qw = I.randn_bf16((B, S, 2 * Hq, D), g).to(cuda_device)
    k_bhsd = I.randn_bf16((B, Hkv, T, D), g).to(cuda_device)
    v_bhsd = I.randn_bf16((B, Hkv, T, D), g).to(cuda_device)
    q = qw[:, :, ::2]
    k, v = k_bhsd.transpose(1, 2), v_bhsd.transpose(1, 2)
    _check_views(q, k, v, cuda_device, causal=False)


def test_prefill_strided_output_leaves_neighbours(cuda_device):
    """O written into a head slice of a wider buffer (bf16 and float32): the slice matches the
    oracle and the heads around it keep their sentinel values."""
    B, S, Hq, Hkv, D = 1, 257, 4, 2, 128
    q, k, v = _gen(B, S, S, Hq, Hkv, D, seed=23)
    for dt in (torch.bfloat16, torch.float32):
        wide = torch.full((B, S, Hq + 3, D), 7.0, dtype=dt, device=cuda_device)
        o = wide[:, :, 1:1 + Hq]
        _check_views(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), cuda_device, o=o)
        assert torch.all(wide[:, :, 0] == 7.0) and torch.all(wide[:, :, 1 + Hq:] == 7.0)


def test_prefill_strided_no_visible_keys(cuda_device):
    """A strided call with no keys, and one whose first query tile sees none (key chunk after the
    queries): empty rows get O = 0 and LSE = -inf from the kernel itself."""
    B, S, Hq, Hkv, D = 1, 300, 4, 2, 128
    g = I.generator(24)
    qkv = I.randn_bf16((B, S, Hq + 2 * Hkv, D), g).to(cuda_device)
    q, k, v = qkv[:, :, :Hq], qkv[:, :, Hq:Hq + Hkv], qkv[:, :, Hq + Hkv:]
    o, lse = A.attn_prefill(q, k[:, :0], v[:, :0], causal=True)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
    o, lse = A.attn_prefill(q, k, v, causal=True, q_pos0=0, kv_pos0=200)
    torch.cuda.synchronize()
    ro, rl = O.attention(q.cpu().contiguous(), k.cpu().contiguous(), v.cpu().contiguous(), scale=1 / math.sqrt(D),
                         causal=True, q_pos0=0, kv_pos0=200)
    assert_o_close(o, ro)
    assert_lse_close(to_np(lse).transpose(0, 2, 1), rl)
    device_clean()


def test_prefill_many_work_items(cuda_device):
    """80000 one-token sequences make 80000 work items, 540 for each CTA of the persistent grid:
    every row is computed (one visible key: O = V, LSE = scale * q.k)."""
    B, D = 80000, 64
    q, k, v = _gen(B, 1, 1, 1, 1, D, seed=25)
    o, lse = A.attn_prefill(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), causal=True)
    torch.cuda.synchronize()
    ro, rl = O.attention(q, k, v, scale=1 / math.sqrt(D), causal=True)
    assert_o_close(o, ro)
    assert_lse_close(to_np(lse).transpose(0, 2, 1), rl)
    device_clean()


def test_prefill_concurrent_streams(cuda_device):
    """Three launches in flight at once on three streams (persistent grids sharing the SMs, each
    walking its own work items): all match the oracle."""
    cases = [_gen(1, 1024, 1024, 8, 2, 128, seed=31), _gen(2, 640, 640, 4, 4, 64, seed=32),
             _gen(1, 384, 384, 2, 1, 128, seed=33)]
    dev_cases = [tuple(x.to(cuda_device) for x in c) for c in cases]
    streams = [torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()]
    torch.cuda.synchronize()
    outs = []
    for (q, k, v), s in zip(dev_cases, streams):
        with torch.cuda.stream(s):
            outs.append(A.attn_prefill(q, k, v, causal=True, stream=s))
    torch.cuda.synchronize()
    for (q, k, v), (o, lse) in zip(cases, outs):
        ro, rl = O.attention(q, k, v, scale=1 / math.sqrt(q.shape[-1]), causal=True)
        assert_o_close(o, ro)
        assert_lse_close(to_np(lse).transpose(0, 2, 1), rl)
    device_clean()


def test_prefill_alternating_head_sizes(cuda_device):
    """Launches of the D = 64 and D = 128 kernels interleaved in one process: every row is computed
    each time (no state carries from one launch or instantiation to the next)."""
    cases = [_gen(1, 300, 300, 8, 2, 64, seed=41), _gen(1, 300, 300, 8, 2, 128, seed=42)]
    for _ in range(3):
        for q, k, v in cases:
            _check(q, k, v, cuda_device, causal=True)
