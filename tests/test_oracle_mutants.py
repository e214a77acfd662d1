"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that the pins
catch every one: a dropped term, a wrong sign or index, a transposed operand, an
off-by-one mask, an ignored offset or length."""
import os
import types

import pytest

from tests import oracle_pins as P

SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "attention.py")

MUTANTS = {
    "interleaved_gqa_mapping": ("for h in range(kvh * G, (kvh + 1) * G):", "for h in range(kvh, Hq, Hkv):"),
    "causal_off_by_one": ("key_pos[None, :] <= (q_pos0 + rr)[:, None]", "key_pos[None, :] < (q_pos0 + rr)[:, None]"),
    "dropped_scale": ("s = scale * (Qr @ K.T)", "s = (Qr @ K.T)"),
    "k_for_v": ("o[b, r0:r0 + len(rr), h, :] = w @ V", "o[b, r0:r0 + len(rr), h, :] = w @ K"),
    "sign_flip_exp": ("e = np.exp(s - mx_safe[:, None])", "e = np.exp(mx_safe[:, None] - s)"),
    "lse_without_max": ("row_lse = np.where(has, mx_safe + np.log(tot), -np.inf)",
                        "row_lse = np.where(has, np.log(tot), -np.inf)"),
    "merge_unnormalised": ("wn = np.where(has[None], w / np.where(has, tot, 1.0)[None], 0.0)",
                           "wn = np.where(has[None], w, 0.0)"),
    "merge_lse_without_max": ("lse = np.where(has, mx_safe + np.log(np.where(has, tot, 1.0)), -np.inf)",
                              "lse = np.where(has, np.log(np.where(has, tot, 1.0)), -np.inf)"),
    "k_scale_on_v": ("K = K * as_f64(k_scale[b, :L, kvh])[:, None]", "V = V * as_f64(k_scale[b, :L, kvh])[:, None]"),
    "q_offset_ignored": ("(q_pos0 + rr)[:, None]", "(rr)[:, None]"),
    "kv_offset_ignored": ("key_pos = kv_pos0 + np.arange(L)", "key_pos = np.arange(L)"),
    "kv_lens_ignored": ("L = int(min(lens[b], T))", "L = T"),
    "transposed_scores": ("Qr @ K.T", "(K @ Qr.T).T[:, ::-1]"),
}


def _mutant(old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, old
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    m = _mutant(*MUTANTS[name])
    caught = []
    for pin in P.ATTENTION_PINS:
        try:
            pin(m)
        except Exception as e:  # noqa: BLE001 - any failure counts as caught
            caught.append(pin.__name__)
    assert caught, f"no pin caught mutant {name}"
