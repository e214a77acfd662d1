"""GPU parity of the chunk streamer (host-resident Q/K/V under a device budget) against the
oracle, plus its host-side failure paths (injected copy / allocation failures, budget)."""
import math

import numpy as np
import pytest
import torch

from exact_long_context_tmem_b200 import attn as A
from exact_long_context_tmem_b200 import inputs as I
from oracle import attention as O
from tests.parity import assert_lse_close, assert_o_close, device_clean, to_np

pytestmark = pytest.mark.gpu


def _host(B, S, Hq, Hkv, D, seed):
    g = I.generator(seed)
    q = I.randn_bf16((B, S, Hq, D), g).pin_memory()
    k = I.randn_bf16((B, S, Hkv, D), g).pin_memory()
    v = I.randn_bf16((B, S, Hkv, D), g).pin_memory()
    return q, k, v


@pytest.mark.parametrize("B,S,Hq,Hkv,D,chunk,budget,causal", [
    (1, 2000, 8, 2, 128, 512, 12 * 2**20, True),    # several query blocks and chunks, ragged ends
    (2, 1100, 4, 2, 64, 256, 4 * 2**20, True),      # batch 2: strided host copies
    (1, 900, 4, 4, 128, 256, 4 * 2**20, False),     # full (non-causal) attention
])
def test_stream_matches_oracle(cuda_device, B, S, Hq, Hkv, D, chunk, budget, causal):
    q, k, v = _host(B, S, Hq, Hkv, D, seed=S + chunk)
    plan = A.attn_stream_plan(B, Hq, Hkv, D, S, causal=causal, chunk_tokens=chunk, budget_bytes=budget)
    assert plan.q_block < S  # the budget forces more than one query block
    o, lse, stats = A.attn_chunked_stream(q, k, v, causal=causal, chunk_tokens=chunk, budget_bytes=budget)
    assert stats.plan.device_bytes <= budget
    assert stats.h2d_bytes > 0 and stats.d2h_bytes > 0
    # event timings: every copy direction and the compute steps were timed, within the device span
    assert stats.ms_h2d > 0 and stats.ms_d2h > 0 and stats.ms_compute_busy > 0
    assert 0 < stats.ms_compute_busy <= stats.ms_device * 1.001 and stats.ms_device <= stats.ms_total * 1.001
    ro, rl = O.attention(q, k, v, scale=1 / math.sqrt(D), causal=causal)
    assert_o_close(o, ro)
    assert_lse_close(to_np(lse).transpose(0, 2, 1), rl)
    device_clean()


def test_stream_device_memory_bounded_by_budget(cuda_device):
    """Device memory follows the plan, which the budget bounds whatever the sequence length: a
    sequence 16 times longer runs in the same budget, and every buffer is freed on return."""
    q, k, v = _host(1, 512, 4, 2, 128, seed=1)
    A.attn_chunked_stream(q, k, v, causal=True, chunk_tokens=256, budget_bytes=9 * 2**20)  # warm-up
    torch.cuda.synchronize()
    for S in (2048, 32768):
        q, k, v = _host(1, S, 4, 2, 128, seed=S)
        free0, _ = torch.cuda.mem_get_info()
        o, lse, stats = A.attn_chunked_stream(q, k, v, causal=True, chunk_tokens=512, budget_bytes=9 * 2**20)
        free1, _ = torch.cuda.mem_get_info()
        assert abs(free1 - free0) < 4 * 2**20  # everything freed
        assert 0 < stats.plan.device_bytes <= 9 * 2**20 and stats.plan.q_block < S
        rows = [0, S // 2, S - 1]
        ro, rl = O.attention(q, k, v, scale=1 / math.sqrt(128), causal=True, rows=rows)
        assert_o_close(o[:, rows], ro)
    device_clean()


@pytest.mark.parametrize("what,nth", [(1, 1), (1, 5), (2, 1), (2, 7)])
def test_stream_injected_failures(cuda_device, what, nth):
    q, k, v = _host(1, 1500, 4, 2, 128, seed=3)
    A.attn_chunked_stream(q, k, v, causal=True, chunk_tokens=256, budget_bytes=8 * 2**20)  # warm-up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    A.attn_debug_inject(what, nth)
    with pytest.raises(A.AttnError) as e:
        A.attn_chunked_stream(q, k, v, causal=True, chunk_tokens=256, budget_bytes=8 * 2**20)
    assert e.value.status == 6
    free1, _ = torch.cuda.mem_get_info()
    assert abs(free1 - free0) < 4 * 2**20  # no leak on the error path
    # the next call works
    o, lse, _ = A.attn_chunked_stream(q, k, v, causal=True, chunk_tokens=256, budget_bytes=8 * 2**20)
    ro, rl = O.attention(q, k, v, scale=1 / math.sqrt(128), causal=True, rows=[0, 700, 1499])
    assert_o_close(o[:, [0, 700, 1499]], ro)
    device_clean()


def test_stream_budget_too_small(cuda_device):
    q, k, v = _host(1, 1024, 4, 2, 128, seed=4)
    with pytest.raises(A.AttnError) as e:
        A.attn_chunked_stream(q, k, v, causal=True, chunk_tokens=512, budget_bytes=10**5)
    assert e.value.status == 4


@pytest.mark.slow
def test_stream_1m_tokens_sampled(cuda_device):
    """The streamed causal prefill over 2^20 tokens (32 query / 8 KV heads, head dim 128), with
    Q/K/V/O/LSE in pinned host memory, 64K-token key chunks and a 16e9-byte device budget,
    checked on 64 sampled query rows (all heads) against the float64 oracle."""
    w = I.WORKLOADS["stream_b1_h32g8_d128_s1m_chunk64k"]
    g = I.generator(w.seed)
    sq, skv = (w.B, w.S, w.Hq, w.D), (w.B, w.S, w.Hkv, w.D)
    q = I.randn_bf16(sq, g, out=torch.empty(sq, dtype=torch.bfloat16, pin_memory=True))
    k = I.randn_bf16(skv, g, out=torch.empty(skv, dtype=torch.bfloat16, pin_memory=True))
    v = I.randn_bf16(skv, g, out=torch.empty(skv, dtype=torch.bfloat16, pin_memory=True))
    o, lse, stats = A.attn_chunked_stream(q, k, v, causal=True, chunk_tokens=w.chunk_tokens,
                                          budget_bytes=w.budget_bytes)
    assert stats.plan.device_bytes <= w.budget_bytes and stats.plan.kv_chunk == w.chunk_tokens
    rows = I.sample_rows(w.S, 60, seed=w.seed, edges=(0, 65535, 65536, w.S - 1))
    ro, rl = O.attention(q, k, v, scale=w.scale, causal=True, rows=rows, row_chunk=64)
    assert_o_close(o[:, rows], ro)
    assert_lse_close(to_np(lse[:, rows]).transpose(0, 2, 1), rl)
    device_clean()
