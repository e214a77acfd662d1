"""C-ABI checks that need no GPU: the library loads, exports every entry point that
include/attn.h declares, rejects invalid arguments before any CUDA call, and the streamer's
planner (host code) covers the causal (query, key) plane exactly once."""
import ctypes
import os
import re

import numpy as np
import pytest

from exact_long_context_tmem_b200 import attn as A
from exact_long_context_tmem_b200 import build as Bld
from oracle import stream as OS

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "attn.h")


@pytest.fixture(scope="module")
def L():
    Bld.build()
    return A.lib()


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"ATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", txt)))


def test_header_declares_binding_exports():
    assert declared_symbols() == sorted(A.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_status_strings(L):
    for s in range(7):
        assert A.attn_status_string(s) and A.attn_status_string(s) != "unknown status"


def _dims(B=1, Hq=4, Hkv=2, D=64, scale=0.125):
    return A.Dims(B, Hq, Hkv, D, scale)


FAKE = ctypes.c_void_p(0x10000)  # 16-byte aligned, never dereferenced: validation fails first
MIS = ctypes.c_void_p(0x10008)


@pytest.mark.parametrize("case", [
    dict(dims=_dims(Hq=3, Hkv=2)),               # Hq % Hkv
    dict(dims=_dims(scale=0.0)),                  # scale <= 0
    dict(dims=_dims(scale=float("nan"))),
    dict(S=-1), dict(T=-1), dict(q_pos0=-5),
    dict(q=None), dict(o=None), dict(k=None),
    dict(q=MIS), dict(o=MIS),                    # alignment
    dict(o_dtype=1),                              # FP8 output not allowed
])
def test_prefill_invalid_args(L, case):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, o_dtype=0, lse=None, dims=_dims(), S=16, T=16, causal=1,
             q_pos0=0, kv_pos0=0)
    a.update(case)
    st = L.attn_prefill(a["q"], a["k"], a["v"], a["o"], a["o_dtype"], a["lse"], a["dims"], a["S"], a["T"],
                        a["causal"], a["q_pos0"], a["kv_pos0"], a.get("strides"), None)
    assert st == 1


def test_prefill_unsupported_head_dim(L):
    st = L.attn_prefill(FAKE, FAKE, FAKE, FAKE, 0, None, _dims(D=96), 16, 16, 1, 0, 0, None, None)
    assert st == 2


def test_prefill_empty_is_noop(L):
    assert L.attn_prefill(None, None, None, None, 0, None, _dims(B=0), 16, 16, 1, 0, 0, None, None) == 0
    assert L.attn_prefill(None, None, None, None, 0, None, _dims(), 0, 16, 1, 0, 0, None, None) == 0


def _strides(**bad):
    """Packed [B=1, S=16, H, D=64] strides for q/o (Hq=4) and k/v (Hkv=2), with overrides."""
    base = dict(q_b=16 * 4 * 64, q_s=4 * 64, q_h=64, k_b=16 * 2 * 64, k_s=2 * 64, k_h=64,
                v_b=16 * 2 * 64, v_s=2 * 64, v_h=64, o_b=16 * 4 * 64, o_s=4 * 64, o_h=64)
    base.update(bad)
    order = ["q_b", "q_s", "q_h", "k_b", "k_s", "k_h", "v_b", "v_s", "v_h", "o_b", "o_s", "o_h"]
    return (ctypes.c_longlong * 12)(*[base[n] for n in order])


@pytest.mark.parametrize("bad", [dict(q_h=0), dict(k_s=-128), dict(v_b=4), dict(o_h=68), dict(q_s=1 << 40),
                                 dict(k_h=63)])
def test_prefill_invalid_strides(L, bad):
    """Each stride must be positive, a whole number of 16-byte units and below TMA's limit; the
    check runs before any CUDA call (the pointers here are never dereferenced)."""
    st = L.attn_prefill(FAKE, FAKE, FAKE, FAKE, 0, None, _dims(), 16, 16, 1, 0, 0, _strides(**bad), None)
    assert st == 1


def test_prefill_float32_output_strides_in_4_element_units(L):
    """A float32 o needs its strides in 16-byte units = 4 elements; 68 is one, not for bf16."""
    st = L.attn_prefill(FAKE, FAKE, FAKE, FAKE, 2, None, _dims(D=96), 16, 16, 1, 0, 0, _strides(o_h=68), None)
    assert st == 2  # strides accepted; the head dim is what is unsupported
    st = L.attn_prefill(FAKE, FAKE, FAKE, FAKE, 0, None, _dims(D=96), 16, 16, 1, 0, 0, _strides(o_h=68), None)
    assert st == 1


@pytest.mark.parametrize("case", [
    dict(kv_dtype=1),                 # FP8 without scales
    dict(kv_dtype=3), dict(kv_dtype=4),  # INT8 / INT4 without scales
    dict(kv_dtype=2), dict(kv_dtype=5),  # not a cache element type
    dict(k_scale=FAKE),               # scales with bf16
    dict(kv_lens=None), dict(q=None), dict(Tmax=-1), dict(num_splits=-1), dict(num_splits=5000),
    dict(ws=None, num_splits=4),      # workspace required but missing
])
def test_decode_invalid_args(L, case):
    a = dict(q=FAKE, k=FAKE, v=FAKE, kv_dtype=0, k_scale=None, v_scale=None, kv_lens=FAKE, Tmax=4096,
             dims=_dims(D=128), num_splits=1, o=FAKE, lse=None, ws=FAKE, ws_bytes=1 << 30)
    a.update(case)
    st = L.attn_decode_splitkv(a["q"], a["k"], a["v"], a["kv_dtype"], a["k_scale"], a["v_scale"], a["kv_lens"],
                               a["Tmax"], a["dims"], a["num_splits"], a["o"], a["lse"], a["ws"], a["ws_bytes"], None)
    assert st == 1


def test_decode_unsupported(L):
    args = (FAKE, FAKE, FAKE, 0, None, None, FAKE, 4096)
    assert L.attn_decode_splitkv(*args, _dims(D=64), 1, FAKE, None, None, 0, None) == 2
    assert L.attn_decode_splitkv(*args, _dims(Hq=34, Hkv=2, D=128), 1, FAKE, None, None, 0, None) == 2


@pytest.mark.parametrize("case", [
    dict(page_size=100), dict(page_size=64), dict(max_pages=0), dict(num_pages=0), dict(page_table=None),
    dict(k_pool=None), dict(q=None), dict(kv_lens=None), dict(kv_dtype=7), dict(k_scale=FAKE),
    dict(kv_dtype=1), dict(kv_dtype=3), dict(kv_dtype=4), dict(ws=None), dict(num_splits=-1),
    dict(page_table=ctypes.c_void_p(0x10002)),
])
def test_decode_paged_invalid_args(L, case):
    a = dict(q=FAKE, k_pool=FAKE, v_pool=FAKE, kv_dtype=0, k_scale=None, v_scale=None, page_table=FAKE,
             max_pages=8, page_size=512, num_pages=64, kv_lens=FAKE, dims=_dims(D=128), num_splits=4, o=FAKE,
             lse=None, ws=FAKE, ws_bytes=1 << 30)
    a.update(case)
    st = L.attn_decode_paged(a["q"], a["k_pool"], a["v_pool"], a["kv_dtype"], a["k_scale"], a["v_scale"],
                             a["page_table"], a["max_pages"], a["page_size"], a["num_pages"], a["kv_lens"],
                             a["dims"], a["num_splits"], a["o"], a["lse"], a["ws"], a["ws_bytes"], None)
    assert st == 1


@pytest.mark.parametrize("case", [dict(n_q=0), dict(q=None), dict(k=None), dict(kv_dtype=1), dict(ws=None)])
def test_decode_multi_invalid_args(L, case):
    a = dict(q=FAKE, k=FAKE, v=FAKE, kv_dtype=0, k_scale=None, v_scale=None, kv_lens=FAKE, Tmax=4096, n_q=2,
             dims=_dims(D=128), num_splits=4, o=FAKE, lse=None, ws=FAKE, ws_bytes=1 << 30)
    a.update(case)
    st = L.attn_decode_multi(a["q"], a["k"], a["v"], a["kv_dtype"], a["k_scale"], a["v_scale"], a["kv_lens"],
                             a["Tmax"], a["n_q"], a["dims"], a["num_splits"], a["o"], a["lse"], a["ws"], a["ws_bytes"],
                             None)
    assert st == 1


@pytest.mark.parametrize("kv_dtype", [3, 4])
def test_decode_multi_integer_cache_unsupported(L, kv_dtype):
    st = L.attn_decode_multi(FAKE, FAKE, FAKE, kv_dtype, FAKE, FAKE, FAKE, 4096, 2, _dims(D=128), 4, FAKE, None, FAKE,
                             1 << 30, None)
    assert st == 2


def test_decode_multi_rows_beyond_the_mma(L):
    # 4 tokens x a group of 8 heads = 32 rows > 16
    st = L.attn_decode_multi(FAKE, FAKE, FAKE, 0, None, None, FAKE, 4096, 4, _dims(Hq=32, Hkv=4, D=128), 4, FAKE,
                             None, FAKE, 1 << 30, None)
    assert st == 2
    d = _dims(B=4, Hq=32, Hkv=8, D=128)
    assert L.attn_decode_multi_workspace_bytes(d, 8192, 3, 4) == 3 * L.attn_decode_workspace_bytes(d, 8192, 4) - 2 * 256


@pytest.mark.parametrize("case", [dict(total_q=-1), dict(max_s=-1), dict(cu_q=None), dict(cu_k=None), dict(q=None),
                                  dict(k=None), dict(o_dtype=1), dict(cu_q=ctypes.c_void_p(0x10002))])
def test_prefill_varlen_invalid_args(L, case):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, o_dtype=0, lse=None, dims=_dims(D=128), cu_q=FAKE, cu_k=FAKE,
             total_q=1000, total_k=1000, max_s=300, causal=1)
    a.update(case)
    st = L.attn_prefill_varlen(a["q"], a["k"], a["v"], a["o"], a["o_dtype"], a["lse"], a["dims"], a["cu_q"], a["cu_k"],
                               a["total_q"], a["total_k"], a["max_s"], a["causal"], None)
    assert st == 1


def test_decode_workspace_and_splits(L):
    d = _dims(B=4, Hq=32, Hkv=8, D=128)
    for P in (1, 2, 7, 19):
        n = L.attn_decode_num_splits(d, 131072, P)
        assert 1 <= n <= P
        ws = L.attn_decode_workspace_bytes(d, 131072, P)
        if n == 1:
            assert ws == 0
        else:
            assert ws >= n * 4 * 32 * (128 + 1) * 4
    assert L.attn_decode_num_splits(d, 300, 64) == 3  # at most one split per 128-token tile
    assert L.attn_decode_num_splits(d, 0, 0) == 1


@pytest.mark.parametrize("case", [
    dict(P=0, accumulate=0), dict(P=-1), dict(R=-1), dict(o_dtype=1),
    dict(accumulate=1, o_dtype=0),        # in-place merge needs a float32 accumulator
    dict(accumulate=1, lse_out=None),
    dict(o_out=None), dict(o_parts=None),
])
def test_merge_invalid_args(L, case):
    a = dict(o_parts=FAKE, lse_parts=FAKE, P=2, R=10, D=128, o_out=FAKE, o_dtype=2, lse_out=FAKE, accumulate=0)
    a.update(case)
    st = L.attn_merge_lse(a["o_parts"], a["lse_parts"], a["P"], a["R"], a["D"], a["o_out"], a["o_dtype"],
                          a["lse_out"], a["accumulate"], None)
    assert st == 1


def test_merge_empty_rows_noop(L):
    assert L.attn_merge_lse(FAKE, FAKE, 2, 0, 128, FAKE, 2, None, 0, None) == 0


def test_stream_plan_budget_error(L):
    plan = A.StreamPlan()
    d = _dims(B=1, Hq=32, Hkv=8, D=128)
    st = L.attn_stream_plan(d, 1 << 20, 1, 65536, 10**6, ctypes.byref(plan))
    assert st == 4
    st = L.attn_stream_plan(d, 1 << 20, 1, 100, 10**10, ctypes.byref(plan))  # chunk not a multiple of 128
    assert st == 1


def test_stream_plan_fits_budget_and_config(L):
    plan = A.attn_stream_plan(1, 32, 8, 128, 1 << 20, causal=True, chunk_tokens=65536, budget_bytes=16 * 10**9)
    assert plan.kv_chunk == 65536
    assert plan.device_bytes <= 16 * 10**9
    assert plan.q_block % 128 == 0 and plan.q_block >= 65536


@pytest.mark.parametrize("S,chunk,budget,causal", [
    (1000, 128, 10**12, True), (1000, 256, 10**12, False), (4096, 512, 3 * 10**6, True),
    (777, 0, 2 * 10**6, True), (5000, 1024, 8 * 10**6, True),
])
def test_stream_tasks_exact_cover(L, S, chunk, budget, causal):
    """Every visible (query, key) pair lies in exactly one task rectangle (the oracle's
    coverage counter decides)."""
    plan = A.attn_stream_plan(1, 4, 2, 64, S, causal=causal, chunk_tokens=chunk, budget_bytes=budget)
    assert plan.device_bytes <= budget
    tasks = [A.attn_stream_task(plan, S, causal, i) for i in range(plan.n_tasks)]
    counts, visible = OS.coverage(tasks, S, S, plan.q_block, plan.kv_chunk, causal)
    np.testing.assert_array_equal(counts, visible.astype(np.int64))
    # the planner's tasks are exactly the oracle's non-empty rectangles, in the same order
    assert tasks == OS.block_tasks(S, S, plan.q_block, plan.kv_chunk, causal)


def test_inject_validation(L):
    assert L.attn_debug_inject(3, 1) == 1
    assert L.attn_debug_inject(1, 0) == 1
    assert L.attn_debug_inject(0, 0) == 0
