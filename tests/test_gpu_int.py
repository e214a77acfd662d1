"""GPU parity of the split-KV decode over INT8 / INT4 KV caches (ORT CPU GQA analysis: integer
KV caches with V dequantised inside the SV accumulation) against the float64 oracle, contiguous
and paged."""
import pytest
import torch

from exact_long_context_tmem_b200 import attn as A
from exact_long_context_tmem_b200 import inputs as I
from oracle import attention as O
from oracle import intq as IQ
from oracle import paged as PG
from tests.parity import assert_lse_close, assert_o_close, device_clean

pytestmark = pytest.mark.gpu


def _case(lens, Tmax, bits, Hq=32, Hkv=8, seed=61):
    w = I.Workload("int_gpu", "decode", B=len(lens), Hq=Hq, Hkv=Hkv, D=128, kv_bits=bits, seed=seed)
    return w, I.decode_inputs(w, lens=torch.tensor(lens, dtype=torch.int32), Tmax=Tmax)


def _run(d, dev, splits=0):
    o, lse = A.attn_decode_splitkv(d["q"].to(dev), d["k_codes"].to(dev), d["v_codes"].to(dev), d["kv_lens"].to(dev),
                                   k_scale=d["k_scale"].to(dev), v_scale=d["v_scale"].to(dev), num_splits=splits)
    torch.cuda.synchronize()
    device_clean()  # a wait that ran out leaves stale partials: report it as such, not as a mismatch
    return o, lse


def _ref(d, scale):
    bits = d["kv_bits"]
    return O.decode(d["q"], IQ.int_values(d["k_codes"], bits), IQ.int_values(d["v_codes"], bits), d["kv_lens"],
                    scale=scale, k_scale=d["k_scale"], v_scale=d["v_scale"])


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("splits", [1, 4, 0])
def test_int_small_ragged(cuda_device, bits, splits):
    w, d = _case([513, 1024, 0, 1, 130], 1024, bits)
    o, lse = _run(d, cuda_device, splits)
    ro, rl = _ref(d, w.scale)
    assert_o_close(o, ro)
    assert_lse_close(lse, rl)
    assert torch.all(o[2] == 0) and torch.all(torch.isneginf(lse[2]))
    device_clean()


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (16, 16), (12, 1), (6, 3), (64, 8), (32, 2)])
def test_int_groups(cuda_device, bits, Hq, Hkv):
    w, d = _case([1, 2049], 2100, bits, Hq=Hq, Hkv=Hkv, seed=Hq * 10 + Hkv + 700)
    for splits in (1, 5):
        o, lse = _run(d, cuda_device, splits)
        ro, rl = _ref(d, w.scale)
        assert_o_close(o, ro)
        assert_lse_close(lse, rl)
    device_clean()


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (64, 8), (48, 4)])
def test_int_many_items_per_cta(cuda_device, bits, Hq, Hkv):
    """More (split, KV head, sequence) work items than SMs, so each persistent CTA walks several,
    with empty splits, single tokens and odd tile counts between them."""
    g = torch.Generator().manual_seed(bits * 100 + Hq + Hkv)
    lens = torch.randint(0, 1537, (48,), generator=g)
    lens[::7] = 0
    lens[3::11] = 1
    lens[5::13] = 1536
    w, d = _case(lens.tolist(), 1536, bits, Hq=Hq, Hkv=Hkv, seed=900 + bits + Hq)
    ro, rl = _ref(d, w.scale)
    for splits in (3, 0):
        o, lse = _run(d, cuda_device, splits)
        assert_o_close(o, ro)
        assert_lse_close(lse, rl)
        empty = (d["kv_lens"] == 0).nonzero().flatten().tolist()
        assert all(torch.all(o[b] == 0) and torch.all(torch.isneginf(lse[b])) for b in empty)
    device_clean()


@pytest.mark.parametrize("bits", [8, 4])
def test_int_scale_extremes(cuda_device, bits):
    """Per-token V scales over six decades, a K-scale ramp (the running maximum moves past the lazy
    threshold tile after tile) and query heads of very different magnitude (each row carries its
    own power-of-two exponent)."""
    Tmax = 2000
    w, d = _case([2000, 1700], Tmax, bits, seed=93)
    g = torch.Generator().manual_seed(5)
    vexp = torch.randint(-3, 4, (2, Tmax, 8), generator=g).float()
    d["v_scale"] = d["v_scale"] * torch.pow(10.0, vexp)
    d["k_scale"] = d["k_scale"] * (1.0 + torch.arange(Tmax, dtype=torch.float32) / 40.0)[None, :, None]
    qs = torch.tensor([1e-6, 1e-2, 1.0, 30.0] * 8, dtype=torch.float32)
    d["q"] = (d["q"].float() * qs[None, :, None]).to(torch.bfloat16)
    for splits in (1, 3):
        o, lse = _run(d, cuda_device, splits)
        ro, rl = _ref(d, w.scale)
        assert_o_close(o, ro)
        assert_lse_close(lse, rl)
    device_clean()


@pytest.mark.parametrize("bits", [8, 4])
def test_int_query_dynamic_range(cuda_device, bits):
    """Query rows whose elements span 2^-30 .. 2^2 of one large element, a row with a single
    nonzero element, and an all-zero row: the INT8 scores take Q as integers of 22 bits (elements
    below 2^-14 of the row maximum are rounded), the INT4 scores as scaled f16 rows."""
    w, d = _case([1500, 900], 1500, bits, Hq=16, Hkv=4, seed=121)
    g = torch.Generator().manual_seed(7)
    q = d["q"].float()
    span = torch.pow(2.0, torch.randint(-30, 3, q.shape, generator=g).float())
    q = q * span
    q[0, 1] = 0.0
    q[0, 1, 17] = 3.0
    q[1, 2] = 0.0
    d["q"] = q.to(torch.bfloat16)
    for splits in (1, 2):
        o, lse = _run(d, cuda_device, splits)
        ro, rl = _ref(d, w.scale)
        assert_o_close(o, ro)
        assert_lse_close(lse, rl)
    device_clean()


@pytest.mark.parametrize("bits", [8, 4])
def test_int_all_code_values(cuda_device, bits):
    """Every code value (-128..127 / -8..7) appears in K and V, at both ends of a row."""
    w, d = _case([640], 640, bits, Hq=8, Hkv=1, seed=97)
    n = d["k_codes"].shape[-1]
    allb = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    dt = torch.int8 if bits == 8 else torch.uint8
    for t in range(0, 640, 3):
        d["k_codes"][0, t, 0] = torch.roll(allb, t)[:n].view(dt)
        d["v_codes"][0, t, 0] = torch.roll(allb, 2 * t)[:n].view(dt)
    o, lse = _run(d, cuda_device, 2)
    ro, rl = _ref(d, w.scale)
    assert_o_close(o, ro)
    assert_lse_close(lse, rl)
    device_clean()


def _ref_paged(pd, scale):
    bits = pd["kv_bits"]
    return PG.decode_paged(pd["q"], torch.from_numpy(IQ.int_values(pd["k_codes"], bits)),
                           torch.from_numpy(IQ.int_values(pd["v_codes"], bits)), pd["page_table"], pd["kv_lens"],
                           pd["page_size"], scale=scale, k_scale_pool=pd["k_scale"], v_scale_pool=pd["v_scale"])


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("page_size", [128, 512])
def test_int_paged_matches_oracle_and_contiguous(cuda_device, bits, page_size):
    lens = [3000, 0, 1, 512, 1024, 2049]
    w, d = _case(lens, 3072, bits, seed=67)
    pd = I.paged_inputs(d, page_size, seed=page_size + bits)
    ro, rl = _ref_paged(pd, w.scale)
    dev = cuda_device
    for splits in (1, 3, 0):
        o, lse = A.attn_decode_paged(pd["q"].to(dev), pd["k_codes"].to(dev), pd["v_codes"].to(dev),
                                     pd["page_table"].to(dev), pd["kv_lens"].to(dev), k_scale=pd["k_scale"].to(dev),
                                     v_scale=pd["v_scale"].to(dev), num_splits=splits)
        torch.cuda.synchronize()
        assert_o_close(o, ro)
        assert_lse_close(lse, rl)
        oc, lc = _run(d, dev, splits)
        assert torch.equal(o, oc) and torch.equal(lse, lc)  # only the addresses differ
    device_clean()


@pytest.mark.parametrize("bits", [8, 4])
def test_int_bad_page_entry_reads_zeros_and_is_reported(cuda_device, bits):
    """A table entry outside the pool is never dereferenced (its codes land as zeros through the
    TMA's out-of-bounds fill, its scales are not read) and is reported by the status word."""
    w, d = _case([1000], 1024, bits, seed=71)
    pd = I.paged_inputs(d, 128, seed=4)
    pd["page_table"][0, 2] = pd["num_pages"] + 5
    dev = cuda_device
    o, lse = A.attn_decode_paged(pd["q"].to(dev), pd["k_codes"].to(dev), pd["v_codes"].to(dev),
                                 pd["page_table"].to(dev), pd["kv_lens"].to(dev), k_scale=pd["k_scale"].to(dev),
                                 v_scale=pd["v_scale"].to(dev), num_splits=1)
    torch.cuda.synchronize()
    st, site = A.attn_device_status(reset=True)
    assert st == A.ATTN_ERR_INVALID_ARG and site == 44
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()


def test_int_multi_token_unsupported(cuda_device):
    w, d = _case([300], 384, 8)
    q = d["q"][:, None].repeat(1, 2, 1, 1).contiguous().to(cuda_device)
    with pytest.raises(A.AttnError) as e:
        A.attn_decode_multi(q, d["k_codes"].to(cuda_device), d["v_codes"].to(cuda_device),
                            d["kv_lens"].to(cuda_device), k_scale=d["k_scale"].to(cuda_device),
                            v_scale=d["v_scale"].to(cuda_device))
    assert e.value.status == A.ATTN_ERR_UNSUPPORTED


@pytest.mark.slow
@pytest.mark.parametrize("name", ["decode_int8_b16_h32g8_d128_t32768", "decode_int4_b16_h32g8_d128_t32768"])
def test_int_full_workload(cuda_device, name):
    w = I.WORKLOADS[name]
    d = I.decode_inputs(w)
    o, lse = _run(d, cuda_device, 0)
    ro, rl = _ref(d, w.scale)
    assert_o_close(o, ro)
    assert_lse_close(lse, rl)
    device_clean()
