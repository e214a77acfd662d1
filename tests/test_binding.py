"""Host-side logic of the Python binding and of the benchmark's byte counts (no GPU)."""
import re

import pytest
import torch

import bench
from exact_long_context_tmem_b200 import attn as A
from exact_long_context_tmem_b200 import inputs as I


def test_kv_kind_inference():
    D = 128

    def t(dtype, last=D):
        return torch.empty((1, 1, 1, last), dtype=dtype)

    assert A._kv_kind(t(torch.bfloat16), D, None) == A.ATTN_BF16
    assert A._kv_kind(t(torch.uint8), D, None) == A.ATTN_FP8_E4M3
    assert A._kv_kind(t(torch.float8_e4m3fn), D, None) == A.ATTN_FP8_E4M3
    assert A._kv_kind(t(torch.int8), D, None) == A.ATTN_INT8
    assert A._kv_kind(t(torch.uint8, D // 2), D, None) == A.ATTN_INT4  # packed rows of D/2 bytes
    assert A._kv_kind(t(torch.uint8), D, "int8") == A.ATTN_INT8       # explicit name wins
    with pytest.raises(ValueError):
        A._kv_kind(t(torch.uint8), D, "int2")


def test_binding_dtype_values_match_header():
    src = open(A.os.path.join(A._PKG, "..", "include", "attn.h")).read()
    enum = re.search(r"typedef enum \{([^}]*)\} attn_dtype_t;", src).group(1)
    vals = {k: int(v) for k, v in re.findall(r"(ATTN_\w+)\s*=\s*(\d+)", enum)}
    assert vals == {"ATTN_BF16": A.ATTN_BF16, "ATTN_FP8_E4M3": A.ATTN_FP8_E4M3, "ATTN_F32": A.ATTN_F32,
                    "ATTN_INT8": A.ATTN_INT8, "ATTN_INT4": A.ATTN_INT4}


@pytest.mark.parametrize("name,row", [("decode_b4_h32g8_d128_ragged64k_128k", 256),
                                      ("decode_fp8_b16_h32g8_d128_t32768", 128),
                                      ("decode_int8_b16_h32g8_d128_t32768", 128),
                                      ("decode_int4_b16_h32g8_d128_t32768", 64)])
def test_bench_decode_bytes(name, row):
    """Algorithmic bytes: every visible token's K and V rows of every KV head (plus its two fp32
    scales for a coded cache), Q and O in bf16 and the fp32 LSE."""
    w = I.WORKLOADS[name]
    lens = torch.tensor([1000, 0, 129] + [5] * (w.B - 3), dtype=torch.int32)
    coded = w.kv_fp8 or w.kv_bits
    per_tok = w.Hkv * (2 * row + (8 if coded else 0))
    qo = w.B * w.Hq * (w.D * 2 * 2 + 4)
    assert bench.decode_bytes(w, lens) == int(lens.sum()) * per_tok + qo


@pytest.mark.parametrize("kw,n_q", [({}, 1), ({"kv_fp8": True}, 1), ({"kv_bits": 8}, 1), ({"kv_bits": 4}, 1),
                                    ({}, 3), ({"kv_fp8": True}, 2)])
def test_bench_decode_oracle_sample(kw, n_q):
    """The per-decode-line CPU baseline runs the oracle on sequence 0 of the same inputs."""
    w = I.Workload("sample", "decode", B=3, Hq=8, Hkv=2, D=128, seed=3, **kw)
    d = I.decode_inputs(w, lens=torch.tensor([300, 0, 17], dtype=torch.int32), Tmax=384)
    cb = bench.decode_oracle_sample(w, d, n_q)
    assert cb["kind"] == "oracle" and cb["unit"] == "GB/s" and cb["value"] > 0 and cb["cores"] >= 1
    assert "300 tokens" in cb["sample"]


def test_bench_varlen_oracle_sample():
    w = I.Workload("sample_varlen", "prefill_varlen", B=3, Hq=4, Hkv=2, D=64, len_lo=40, len_hi=90, seed=9)
    d = I.varlen_inputs(w)
    cb = bench.varlen_oracle_sample(w, d)
    assert cb["kind"] == "oracle" and cb["unit"] == "TFLOP/s" and cb["value"] > 0
    assert f"{int(d['lens'][0])} tokens" in cb["sample"]


def test_oracle_rates():
    w = I.WORKLOADS["prefill_b2_h32g8_d128_s8192"]
    r = bench.oracle_rates(w, 10, 2.0, 0.02)
    assert r["rows_per_s"] == 5.0
    assert abs(r["extrapolated_full_config_s"] - bench.prefill_flops(w) / 0.02e12) < 0.1


def test_cache_row_size_is_checked():
    D = 128
    ok8 = torch.empty((1, 4, 2, D), dtype=torch.int8)
    A._check_kv_rows(ok8, ok8, D, A.ATTN_INT8)
    ok4 = torch.empty((1, 4, 2, D // 2), dtype=torch.uint8)
    A._check_kv_rows(ok4, ok4, D, A.ATTN_INT4)
    with pytest.raises(ValueError):
        A._check_kv_rows(ok8.view(torch.uint8), ok8.view(torch.uint8), D, A.ATTN_INT4)  # D bytes, not D/2
    with pytest.raises(ValueError):
        A._check_kv_rows(ok4, ok4, D, A.ATTN_FP8_E4M3)
    with pytest.raises(ValueError):
        A._check_kv_rows(ok8.transpose(1, 2), ok8, D, A.ATTN_INT8)  # not contiguous


def test_scale_shape_is_checked():
    D = 128
    k = torch.empty((2, 4, 3, D), dtype=torch.int8)
    ok = torch.empty((2, 4, 3), dtype=torch.float32)
    A._check_kv_rows(k, k, D, A.ATTN_INT8, ok, ok)
    with pytest.raises(ValueError):
        A._check_kv_rows(k, k, D, A.ATTN_INT8, ok.double(), ok)
    with pytest.raises(ValueError):
        A._check_kv_rows(k, k, D, A.ATTN_INT8, ok, torch.empty((2, 3, 4), dtype=torch.float32))


def test_bench_stream_oracle_sample():
    """The streamed workload's CPU baseline runs the oracle on rows near the end of the sequence for
    the query heads of KV head 0, from the same host tensors."""
    w = I.Workload("s", "stream", B=1, Hq=8, Hkv=2, D=64, S=700, T=700, chunk_tokens=128, seed=3)
    g = I.generator(w.seed)
    q = I.randn_bf16((1, w.S, w.Hq, w.D), g)
    k = I.randn_bf16((1, w.S, w.Hkv, w.D), g)
    v = I.randn_bf16((1, w.S, w.Hkv, w.D), g)
    cb = bench.stream_oracle_sample(w, q, k, v, n_rows=3)
    assert cb["kind"] == "oracle" and cb["unit"] == "TFLOP/s" and cb["value"] > 0
    assert "3 query rows" in cb["sample"] and "4 heads" in cb["sample"]
