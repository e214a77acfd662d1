"""GPU parity of the log-sum-exp merge kernel against the oracle's merge."""
import numpy as np
import pytest
import torch

from exact_long_context_tmem_b200 import attn as A
from oracle import attention as O
from tests.parity import device_clean, to_np

pytestmark = pytest.mark.gpu


def _parts(P, R, D, seed, empty_frac=0.2):
    g = torch.Generator().manual_seed(seed)
    o = torch.randn(P, R, D, generator=g)
    lse = torch.randn(P, R, generator=g) * 4
    lse[torch.rand(P, R, generator=g) < empty_frac] = float("-inf")
    lse[:, 0] = float("-inf")  # one row with every part empty
    return o, lse


@pytest.mark.parametrize("P,R,D", [(1, 37, 128), (3, 1000, 128), (19, 513, 128), (40, 77, 64), (2, 8, 64)])
def test_merge_matches_oracle(cuda_device, P, R, D):
    o, lse = _parts(P, R, D, seed=P * 100 + R)
    ref_o, ref_l = O.merge_lse(o.numpy(), lse.numpy())
    go, gl = A.attn_merge_lse(o.to(cuda_device), lse.to(cuda_device))
    torch.cuda.synchronize()
    np.testing.assert_allclose(to_np(go), ref_o, atol=1e-5, rtol=1e-5)
    gl = to_np(gl)
    np.testing.assert_array_equal(np.isneginf(gl), np.isneginf(ref_l))
    fin = np.isfinite(ref_l)
    np.testing.assert_allclose(gl[fin], ref_l[fin], atol=1e-5)
    assert np.all(to_np(go)[0] == 0)
    device_clean()


def test_merge_bf16_out(cuda_device):
    o, lse = _parts(5, 300, 128, seed=9)
    ref_o, _ = O.merge_lse(o.numpy(), lse.numpy())
    go, _ = A.attn_merge_lse(o.to(cuda_device), lse.to(cuda_device), out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    np.testing.assert_allclose(to_np(go), ref_o, atol=1e-2, rtol=1e-2)
    device_clean()


def test_merge_accumulate_in_place(cuda_device):
    o, lse = _parts(4, 256, 128, seed=11)
    ref_o, ref_l = O.merge_lse(o.numpy(), lse.numpy())
    acc_o = o[0].clone().to(cuda_device)
    acc_l = lse[0].clone().to(cuda_device)
    A.attn_merge_lse(o[1:].to(cuda_device), lse[1:].to(cuda_device), o_out=acc_o, lse_out=acc_l, accumulate=True)
    torch.cuda.synchronize()
    np.testing.assert_allclose(to_np(acc_o), ref_o, atol=1e-5, rtol=1e-5)
    fin = np.isfinite(ref_l)
    np.testing.assert_allclose(to_np(acc_l)[fin], ref_l[fin], atol=1e-5)
    device_clean()
