"""Parity at the full benchmark sizes, in the launch configuration bench.py times: the paged
cache (512-token pages in seeded random pool order), multi-token decode (4 query tokens per
sequence) and the packed varlen prefill, on the same seeded inputs the benchmark draws."""
import pytest
import torch

from exact_long_context_tmem_b200 import attn as A
from exact_long_context_tmem_b200 import inputs as I
from oracle import attention as O
from oracle import fp8 as F
from tests.parity import assert_lse_close, assert_o_close, device_clean

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

PAGE_SIZE = 512
N_Q = 4
DECODE = {"bf16": "decode_b4_h32g8_d128_ragged64k_128k", "fp8": "decode_fp8_b16_h32g8_d128_t32768"}


@pytest.fixture(scope="module", params=["bf16", "fp8"])
def decode_case(request):
    w = I.WORKLOADS[DECODE[request.param]]
    return w, I.decode_inputs(w)


def _cache(d, dev):
    if "k_codes" in d:
        return (d["k_codes"].to(dev), d["v_codes"].to(dev)), {"k_scale": d["k_scale"].to(dev),
                                                              "v_scale": d["v_scale"].to(dev)}
    return (d["k"].to(dev), d["v"].to(dev)), {}


def test_paged_full_equals_contiguous(cuda_device, decode_case):
    """Paged decode at the benchmark's configuration is bit-identical to the contiguous decode
    (same splits, same arithmetic; only the addresses differ), whose full-size parity with the
    oracle is checked in test_gpu_decode."""
    w, d = decode_case
    dev = cuda_device
    (k, v), sc = _cache(d, dev)
    q, lens = d["q"].to(dev), d["kv_lens"].to(dev)
    pd = I.paged_inputs(d, PAGE_SIZE, seed=w.seed + 7)
    (kp, vp), scp = _cache(pd, dev)
    Tmax = pd["page_table"].shape[1] * PAGE_SIZE
    splits = A.attn_decode_num_splits(w.B, w.Hq, w.Hkv, w.D, Tmax)
    op, lp = A.attn_decode_paged(q, kp, vp, pd["page_table"].to(dev), lens, num_splits=splits, **scp)
    oc, lc = A.attn_decode_splitkv(q, k, v, lens, num_splits=splits, **sc)
    torch.cuda.synchronize()
    assert torch.equal(op, oc) and torch.equal(lp, lc)
    device_clean()


def test_multi_token_full(cuda_device, decode_case):
    w, d = decode_case
    dev = cuda_device
    (k, v), sc = _cache(d, dev)
    q = I.randn_bf16((w.B, N_Q, w.Hq, w.D), I.generator(w.seed + 11))
    o, lse = A.attn_decode_multi(q.to(dev), k, v, d["kv_lens"].to(dev), **sc)
    torch.cuda.synchronize()
    if "k_codes" in d:
        ro, rl = O.decode_multi(q, F.e4m3_decode(d["k_codes"]), F.e4m3_decode(d["v_codes"]), d["kv_lens"],
                                scale=w.scale, k_scale=d["k_scale"], v_scale=d["v_scale"])
    else:
        ro, rl = O.decode_multi(q, d["k"], d["v"], d["kv_lens"], scale=w.scale)
    assert_o_close(o, ro)
    assert_lse_close(lse, rl)
    device_clean()


def test_varlen_prefill_full(cuda_device):
    w = I.WORKLOADS["prefill_varlen_b16_h32g8_d128_ragged512_2048"]
    d = I.varlen_inputs(w)
    dev = cuda_device
    cu = d["cu"].to(dev)
    o, lse = A.attn_prefill_varlen(d["q"].to(dev), d["k"].to(dev), d["v"].to(dev), cu, cu, int(d["lens"].max()),
                                   causal=True)
    torch.cuda.synchronize()
    ro, rl = O.prefill_varlen(d["q"], d["k"], d["v"], d["cu"], d["cu"], scale=w.scale, causal=True)
    assert_o_close(o, ro)
    assert_lse_close(lse, rl)
    device_clean()
