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
