"""Comparison helpers for GPU-vs-oracle parity (tolerances of the float path)."""
import numpy as np
import torch

O_ATOL = 2e-2
O_RTOL = 2e-2
LSE_ATOL = 1e-3


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_o_close(got, ref, what="O"):
    got = to_np(got) if isinstance(got, torch.Tensor) else np.asarray(got, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err = np.abs(got - ref)
    bad = err > O_ATOL + O_RTOL * np.abs(ref)
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; "
                           f"max abs err {err.max():.3e}")
    return float(err.max())


def assert_lse_close(got, ref, what="LSE"):
    got = to_np(got) if isinstance(got, torch.Tensor) else np.asarray(got, dtype=np.float64)
    np.testing.assert_array_equal(np.isneginf(got), np.isneginf(ref), err_msg=f"{what}: empty-row pattern")
    fin = np.isfinite(ref)
    err = np.abs(got[fin] - ref[fin])
    assert (err <= LSE_ATOL).all(), f"{what}: max abs err {err.max():.3e}"
    return float(err.max()) if err.size else 0.0


def device_clean():
    from exact_long_context_tmem_b200 import attn as A
    st, site = A.attn_device_status(reset=True)
    assert st == 0, f"device status {st} at wait site {site}"
