"""The no-allocation decode entry point (attn_decode_splitkv_noalloc).

Some callers cannot allocate device memory: a serving engine that has already reserved
nearly all of the GPU's memory for its own pool, or a latency-critical decode loop in which
a cudaMalloc (which may synchronise the device) is not allowed.  For them the library keeps
the split-KV partials in one static device array instead of a caller-provided workspace.
These tests call that entry point through the C ABI and check that it gives the same result
as attn_decode_splitkv with a workspace and as the float64 oracle, on two calls in a row (the
array keeps the previous call's contents, which must not leak into the next result), and that
it allocates nothing; one more call goes through the Python wrapper with preallocated outputs.
This file is collected last on purpose.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from exact_long_context_tmem_b200 import attn as A
from exact_long_context_tmem_b200 import inputs as I
from oracle import attention as OR
from oracle import fp8 as F8
from tests.parity import LSE_ATOL, O_ATOL, O_RTOL, assert_lse_close, assert_o_close

LIMIT = 4 << 20  # ATTN_NOALLOC_SCRATCH_BYTES in include/attn.h


def _case(B, Hq, Hkv, lens, Tmax, seed, fp8):
    w = I.Workload("noalloc", "decode", B=B, Hq=Hq, Hkv=Hkv, D=128, kv_fp8=fp8, seed=seed)
    return w, I.decode_inputs(w, lens=torch.tensor(lens, dtype=torch.int32), Tmax=Tmax)


def _dev(d, dev):
    out = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    if "k_codes" in out:
        out["k"], out["v"] = out["k_codes"], out["v_codes"]
    else:
        out["k_scale"] = out["v_scale"] = None
    return out


def _noalloc_c_abi(d, w, splits, o, lse):
    L = A.lib()
    dims = A.Dims(w.B, w.Hq, w.Hkv, w.D, 1.0 / math.sqrt(w.D))
    kvt = A.ATTN_FP8_E4M3 if d["k"].dtype == torch.uint8 else A.ATTN_BF16
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return L.attn_decode_splitkv_noalloc(p(d["q"]), p(d["k"]), p(d["v"]), kvt, p(d["k_scale"]), p(d["v_scale"]),
                                         p(d["kv_lens"]), int(d["Tmax"]), dims, int(splits), p(o), p(lse),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.gpu
def test_noalloc_matches_workspace_decode_two_calls(cuda_device):
    cases = [
        (_case(3, 8, 2, [1000, 0, 777], 1024, seed=61, fp8=False), 3),
        (_case(2, 32, 8, [513, 1024], 1024, seed=62, fp8=True), 4),
    ]
    for (w, d), splits in cases:
        assert 0 < A.attn_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.D, d["Tmax"], splits) <= LIMIT
    outs = []
    for (w, d), splits in cases:
        dd = _dev(d, cuda_device)
        ref_o, ref_l = A.attn_decode_splitkv(dd["q"], dd["k"], dd["v"], dd["kv_lens"], k_scale=dd["k_scale"],
                                             v_scale=dd["v_scale"], num_splits=splits)
        o = torch.empty_like(ref_o)
        lse = torch.empty_like(ref_l)
        outs.append((w, dd, splits, ref_o, ref_l, o, lse))
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for w, dd, splits, ref_o, ref_l, o, lse in outs:  # two calls in a row on the shared scratch array
        assert _noalloc_c_abi(dd, w, splits, o, lse) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, "the no-allocation entry point changed device memory use"
    for ((w, d), _), (w2, dd, splits, ref_o, ref_l, o, lse) in zip(cases, outs):
        ro, go = ref_o.float().cpu().numpy(), o.float().cpu().numpy()
        assert np.all(np.abs(go - ro) <= O_ATOL + O_RTOL * np.abs(ro))
        rl, gl = ref_l.cpu().numpy(), lse.cpu().numpy()
        np.testing.assert_array_equal(np.isneginf(gl), np.isneginf(rl))
        fin = np.isfinite(rl)
        assert np.all(np.abs(gl[fin] - rl[fin]) <= LSE_ATOL)
        # and against the float64 oracle on the same seeded inputs
        if "k_codes" in d:
            kv, vv = F8.e4m3_decode(d["k_codes"]), F8.e4m3_decode(d["v_codes"])
            oo, ol = OR.decode(d["q"], kv, vv, d["kv_lens"], scale=w.scale, k_scale=d["k_scale"],
                               v_scale=d["v_scale"])
        else:
            oo, ol = OR.decode(d["q"], d["k"], d["v"], d["kv_lens"], scale=w.scale)
        assert_o_close(o, oo, "no-alloc O vs oracle")
        assert_lse_close(lse, ol, "no-alloc LSE vs oracle")
    # one more call through the Python wrapper, into preallocated outputs
    w, dd, splits, ref_o, ref_l, o, lse = outs[0]
    o.fill_(float("nan"))
    lse.fill_(float("nan"))
    A.attn_decode_splitkv_noalloc(dd["q"], dd["k"], dd["v"], dd["kv_lens"], num_splits=splits, o=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.equal(o, ref_o) or np.all(np.abs(o.float().cpu().numpy() - ref_o.float().cpu().numpy())
                                          <= O_ATOL + O_RTOL * np.abs(ref_o.float().cpu().numpy()))
    st, site = A.attn_device_status(reset=True)
    assert st == 0, f"device status {st} at wait site {site}"


def test_noalloc_rejects_requests_beyond_the_scratch_limit():
    """A split count whose partials need more than the static array is refused before any
    CUDA call (no GPU needed)."""
    L = A.lib()
    dims = A.Dims(64, 32, 8, 128, 0.088)
    need = L.attn_decode_workspace_bytes(dims, 131072, 1024)
    assert need > LIMIT
    fake = ctypes.c_void_p(0x10000)
    st = L.attn_decode_splitkv_noalloc(fake, fake, fake, A.ATTN_BF16, None, None, fake, 131072, dims, 1024, fake,
                                       None, None)
    assert st == 4  # ATTN_ERR_BUDGET


@pytest.mark.parametrize("bad,status", [("q", 1), ("head_dim", 2)])
def test_noalloc_argument_errors_come_before_the_limit(bad, status):
    """A request beyond the scratch limit that is also malformed (a null query) or unsupported
    (head dim 96) reports that, not the limit: the checks run in attn_decode_splitkv's order
    first (no GPU needed: nothing is launched)."""
    L = A.lib()
    dims = A.Dims(64, 32, 8, 96 if bad == "head_dim" else 128, 0.088)
    fake = ctypes.c_void_p(0x10000)
    q = None if bad == "q" else fake
    st = L.attn_decode_splitkv_noalloc(q, fake, fake, A.ATTN_BF16, None, None, fake, 131072, dims, 1024, fake,
                                       None, None)
    assert st == status
