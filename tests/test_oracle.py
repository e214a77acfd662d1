"""CPU pins of the float64 oracle (no GPU)."""
import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import fp8, stream
from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ATTENTION_PINS, ids=lambda f: f.__name__)
def test_attention_pin(pin):
    pin(A)


def test_e4m3_golden_codes():
    ex = P.golden()["e4m3_codes"]
    got = fp8.e4m3_decode(np.array(ex["codes"], dtype=np.uint8))
    want = np.array([float(x) for x in ex["values"]])
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    np.testing.assert_array_equal(got[ok], want[ok])
    np.testing.assert_array_equal(np.signbit(got[ok]), np.signbit(want[ok]))


def test_e4m3_all_codes_match_torch():
    """All 256 codes against torch's float8_e4m3fn (a library special case)."""
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = fp8.e4m3_decode(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    assert np.isnan(got).sum() == 2
    assert np.nanmax(got) == 448.0 and np.nanmin(got) == -448.0


def test_e4m3_values_exact_in_bf16():
    """Every finite E4M3 value is exactly representable in bf16, so decoding a code to
    bf16 before the score product loses nothing."""
    vals = fp8.E4M3_TABLE[~np.isnan(fp8.E4M3_TABLE)]
    t = torch.tensor(vals, dtype=torch.float64)
    assert torch.equal(t.to(torch.bfloat16).to(torch.float64), t)


@pytest.mark.parametrize("S,Bq,Ck", [(37, 8, 8), (64, 16, 32), (50, 50, 7), (9, 4, 16)])
@pytest.mark.parametrize("causal", [True, False])
def test_stream_tasks_exact_cover(S, Bq, Ck, causal):
    tasks = stream.block_tasks(S, S, Bq, Ck, causal)
    counts, visible = stream.coverage(tasks, S, S, Bq, Ck, causal)
    np.testing.assert_array_equal(counts, visible.astype(np.int64))


def test_stream_chunked_equals_unsplit():
    r = np.random.default_rng(11)
    B, S, Hq, Hkv, D = 1, 45, 4, 2, 8
    q = r.standard_normal((B, S, Hq, D))
    k = r.standard_normal((B, S, Hkv, D))
    v = r.standard_normal((B, S, Hkv, D))
    o, l = A.attention(q, k, v, scale=0.3, causal=True)
    for Bq, Ck in [(16, 16), (8, 20), (45, 9)]:
        o2, l2 = stream.chunked_attention(q, k, v, scale=0.3, causal=True, Bq=Bq, Ck=Ck)
        np.testing.assert_allclose(o2, o, atol=1e-12)
        np.testing.assert_allclose(l2, l, atol=1e-12)
