"""Pins for the INT8 / INT4 KV-code oracle (oracle/intq.py) against facts outside it: the
hand-derived golden bytes, library two's complement conversions (torch int8, numpy's arithmetic
shift), the synthetic quantiser's round-trip bound, and closed forms of decode over integer
caches.  A mutation test plants plausible mistakes in copies of the oracle and checks that the
pins catch each one."""
import math
import os
import types

import numpy as np
import pytest
import torch

from exact_long_context_tmem_b200 import inputs as I
from oracle import attention as A
from oracle import intq
from tests import oracle_pins as P

SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "intq.py")


def pin_golden(m):
    ex = P.golden()["int_kv_codes"]
    np.testing.assert_array_equal(m.int8_values(np.array(ex["int8_bytes"], dtype=np.uint8)),
                                  np.array(ex["int8_values"], dtype=np.float64))
    np.testing.assert_array_equal(m.int4_values(np.array(ex["int4_bytes"], dtype=np.uint8)),
                                  np.array(ex["int4_values"], dtype=np.float64))


def pin_int8_all_bytes_match_torch(m):
    b = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = b.view(torch.int8).to(torch.float64).numpy()
    np.testing.assert_array_equal(m.int8_values(b), ref)
    np.testing.assert_array_equal(m.int8_values(b.view(torch.int8)), ref)


def pin_int4_all_bytes_match_arithmetic_shift(m):
    b = np.arange(256, dtype=np.uint8)
    lo = ((b << 4).astype(np.uint8).view(np.int8) >> 4).astype(np.float64)  # sign-extending shifts
    hi = (b.view(np.int8) >> 4).astype(np.float64)
    got = m.int4_values(b.reshape(256, 1))
    np.testing.assert_array_equal(got[:, 0], lo)
    np.testing.assert_array_equal(got[:, 1], hi)


def pin_quantiser_layout_and_round_trip(m):
    # A row of integers with absmax 7 quantises to itself with scale 1 (INT4) / 7/127 (INT8).
    row = torch.tensor([[1.0, -2.0, 7.0, -7.0, 0.0, 3.0, -1.0, 5.0]])
    c4, s4 = I.quantize_int_per_token(row, 4)
    assert float(s4[0]) == 1.0
    # byte i = element 2i (low nibble) | element 2i+1 (high nibble), 4-bit two's complement
    assert c4[0].tolist() == [0x01 | 0xE0, 0x07 | 0x90, 0x00 | 0x30, 0x0F | 0x50]
    np.testing.assert_array_equal(m.int4_values(c4)[0], row[0].numpy())
    g = torch.Generator().manual_seed(5)
    x = torch.randn(4, 9, 128, generator=g) * 3.0
    for bits, qmax in ((8, 127), (4, 7)):
        c, s = I.quantize_int_per_token(x, bits)
        vals = m.int_values(c, bits)
        assert np.abs(vals).max() <= qmax
        deq = vals * s.double().numpy()[..., None]
        err = np.abs(deq - x.double().numpy())
        assert np.all(err <= s.double().numpy()[..., None] * (0.5 + 1e-6))


def pin_decode_closed_forms(m):
    """One visible token: O = its dequantised V row, LSE = its scaled score.  Two visible tokens
    with the same K codes and scale: O = the mean of their V rows, LSE = score + ln 2."""
    g = np.random.default_rng(11)
    D, scale = 128, 1.0 / math.sqrt(128)
    for bits in (8, 4):
        nbytes = D if bits == 8 else D // 2
        kc = g.integers(0, 256, size=(1, 3, 1, nbytes), dtype=np.uint8)
        vc = g.integers(0, 256, size=(1, 3, 1, nbytes), dtype=np.uint8)
        kc[0, 1] = kc[0, 0]
        ks = np.array([[[0.03], [0.03], [0.5]]])
        vs = np.array([[[0.02], [0.07], [0.1]]])
        q = g.standard_normal((1, 1, D))
        kv = m.int_values(kc, bits)
        vv = m.int_values(vc, bits)
        s0 = scale * float(q[0, 0] @ (kv[0, 0, 0] * 0.03))
        o1, l1 = A.decode(q, kv, vv, [1], scale=scale, k_scale=ks, v_scale=vs)
        np.testing.assert_allclose(o1[0, 0], vv[0, 0, 0] * 0.02, rtol=1e-12, atol=1e-12)
        assert abs(l1[0, 0] - s0) < 1e-10
        o2, l2 = A.decode(q, kv, vv, [2], scale=scale, k_scale=ks, v_scale=vs)
        np.testing.assert_allclose(o2[0, 0], 0.5 * (vv[0, 0, 0] * 0.02 + vv[0, 1, 0] * 0.07), rtol=1e-12,
                                   atol=1e-12)
        assert abs(l2[0, 0] - (s0 + math.log(2.0))) < 1e-10


PINS = [pin_golden, pin_int8_all_bytes_match_torch, pin_int4_all_bytes_match_arithmetic_shift,
        pin_quantiser_layout_and_round_trip, pin_decode_closed_forms]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(intq)


MUTANTS = {
    "nibbles_swapped": ("out[..., 0::2] = np.where(lo >= 8, lo - 16, lo)\n    out[..., 1::2] = np.where(hi >= 8, hi - 16, hi)",
                        "out[..., 0::2] = np.where(hi >= 8, hi - 16, hi)\n    out[..., 1::2] = np.where(lo >= 8, lo - 16, lo)"),
    "int4_unsigned": ("np.where(lo >= 8, lo - 16, lo)", "lo"),
    "int4_offset_binary": ("np.where(hi >= 8, hi - 16, hi)", "hi - 8"),
    "int8_unsigned": ("np.where(u >= 128, u - 256, u)", "u"),
    "int8_sign_magnitude": ("np.where(u >= 128, u - 256, u)", "np.where(u >= 128, 128 - u, u)"),
}


def _mutant(old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("intq_mutant")
    exec(compile(src.replace(old, new), "intq_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    mod = _mutant(*MUTANTS[name])
    caught = []
    for pin in PINS:
        try:
            pin(mod)
        except Exception:  # noqa: BLE001 - any failure counts as caught
            caught.append(pin.__name__)
    assert caught, f"no pin caught mutant {name}"
