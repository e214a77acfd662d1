"""Bounded-wait timeout path: a kernel waits on an mbarrier nothing arrives at, gives up after
its limit, records the timeout in the device status word and returns; the context stays usable."""
import pytest
import torch

from exact_long_context_tmem_b200 import attn as A

pytestmark = pytest.mark.gpu


def test_wait_probe_times_out_and_context_survives(cuda_device):
    A.attn_device_status(reset=True)
    st = A.attn_debug_wait_probe(50_000_000)  # 50 ms
    assert st == 5
    st2, site = A.attn_device_status(reset=True)
    assert st2 == 5 and site == 1
    assert A.attn_device_status()[0] == 0
    # the GPU still runs ordinary work
    x = torch.randn(1000, device=cuda_device)
    assert torch.isfinite((x * 2).sum()).item()


def test_polynomial_exp2_matches_float64(cuda_device):
    """The FMA-pipe exp2 the prefill softmax uses for one exponential pair in eight: relative error
    within its fitted bound (1.02e-4, checked at 1.1e-4) of float64 exp2 on the softmax's input
    range (x <= 8, the lazy-rescale headroom), exactly 1 at x = 0 and at the integers, and exact 0 at
    and below -127 (masked scores).  The bound is far inside what a weight rounded to bf16 (2^-9)
    and a row sum needed to 1e-3 in log space can tell apart."""
    import numpy as np
    g = torch.Generator().manual_seed(3)
    x = torch.cat([torch.linspace(-126.0, 8.0, 2_000_001), torch.rand(1_000_000, generator=g) * 28 - 20,
                   torch.tensor([0.0, 0.5, -0.5, 8.0, -1e-30, 1e-30])]).float()
    ref = np.exp2(x.double().numpy())
    y_poly = A.attn_debug_exp2(x.to(cuda_device), mode=0).cpu().double().numpy()
    rel_poly = np.abs(y_poly / ref - 1)
    assert rel_poly.max() <= 1.1e-4, rel_poly.max()
    ints = torch.arange(-126, 9, dtype=torch.float32)
    assert torch.equal(A.attn_debug_exp2(ints.to(cuda_device), mode=0).cpu(), torch.exp2(ints))
    z = torch.tensor([-float("inf"), -1000.0, -200.0, -127.0], device=cuda_device)
    assert torch.all(A.attn_debug_exp2(z, mode=0) == 0)
