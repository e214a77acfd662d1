"""GPU parity of the packed variable-length prefill against the oracle."""
import numpy as np
import pytest
import torch

from exact_long_context_tmem_b200 import attn as A
from exact_long_context_tmem_b200 import inputs as I
from oracle import attention as O
from tests.parity import assert_lse_close, assert_o_close, device_clean

pytestmark = pytest.mark.gpu


def _packed(pairs, Hq, Hkv, D, seed):
    g = I.generator(seed)
    tq, tk = sum(p[0] for p in pairs), sum(p[1] for p in pairs)
    q = I.randn_bf16((tq, Hq, D), g)
    k = I.randn_bf16((tk, Hkv, D), g)
    v = I.randn_bf16((tk, Hkv, D), g)
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum([p[0] for p in pairs])]), dtype=torch.int32)
    cu_k = torch.tensor(np.concatenate([[0], np.cumsum([p[1] for p in pairs])]), dtype=torch.int32)
    return q, k, v, cu_q, cu_k


@pytest.mark.parametrize("D,Hq,Hkv", [(128, 32, 8), (64, 6, 2), (128, 9, 3)])
@pytest.mark.parametrize("causal", [True, False])
def test_varlen_prefill(cuda_device, D, Hq, Hkv, causal):
    # past + new (Sk > Sq), plain prefill (Sk = Sq), ragged tails, an empty sequence, a sequence
    # with queries but no keys, and one longer than two query tiles
    pairs = [(300, 700), (128, 128), (0, 50), (77, 77), (5, 0), (1, 1), (513, 600), (200, 1000)]
    q, k, v, cu_q, cu_k = _packed(pairs, Hq, Hkv, D, seed=D + Hq + int(causal))
    scale = 1.0 / D ** 0.5
    o, lse = A.attn_prefill_varlen(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), cu_q.to(cuda_device),
                                   cu_k.to(cuda_device), max(p[0] for p in pairs), causal=causal)
    torch.cuda.synchronize()
    ro, rl = O.prefill_varlen(q, k, v, cu_q, cu_k, scale=scale, causal=causal)
    assert_o_close(o, ro)
    assert_lse_close(lse, rl)
    device_clean()


def test_varlen_matches_dense_prefill(cuda_device):
    """Equal lengths packed = the dense batch (same tiles, same arithmetic)."""
    B, S, Hq, Hkv, D = 3, 384, 16, 4, 128
    g = I.generator(77)
    q = I.randn_bf16((B, S, Hq, D), g).to(cuda_device)
    k = I.randn_bf16((B, S, Hkv, D), g).to(cuda_device)
    v = I.randn_bf16((B, S, Hkv, D), g).to(cuda_device)
    od, ld = A.attn_prefill(q, k, v, causal=True)
    cu = torch.arange(0, (B + 1) * S, S, dtype=torch.int32, device=cuda_device)
    ov, lv = A.attn_prefill_varlen(q.reshape(B * S, Hq, D), k.reshape(B * S, Hkv, D), v.reshape(B * S, Hkv, D),
                                   cu, cu, S, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(ov.reshape(B, S, Hq, D), od)
    assert torch.equal(lv.reshape(B, S, Hq), ld)
    device_clean()
