"""Plant plausible mistakes in copies of the multi-token decode, packed varlen prefill, paged
gather and streamed-decomposition oracles (on the CPU) and check that their pins catch every
one: a query position off by one, a lost causal mask, reversed tokens, top-left instead of
bottom-right alignment, key ranges taken from the query offsets, a page index off by one, an
ignored page table, a dropped partial page, a shifted slot offset, a causal chunk test off by one
or taken at the block's first row, and task offsets dropped."""
import os
import types

import pytest

from tests import test_oracle as TO
from tests import test_oracle_multi as TM
from tests import test_oracle_paged as TP
from tests import test_oracle_varlen as TV

ORACLE = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle")

MUTANTS = {
    # oracle/attention.py: decode_multi
    "multi_position_off_by_one": ("attention.py", "causal=True, q_pos0=lens[b] - n_q,",
                                  "causal=True, q_pos0=lens[b] - n_q + 1,"),
    "multi_not_causal": ("attention.py", "causal=True, q_pos0=lens[b] - n_q,", "causal=False, q_pos0=lens[b] - n_q,"),
    "multi_tokens_reversed": ("attention.py", "        o[b] = ob[0]\n", "        o[b] = ob[0][::-1]\n"),
    # oracle/attention.py: prefill_varlen
    "varlen_top_left_alignment": ("attention.py", "q_pos0=(ke - ks) - (qe - qs), kv_pos0=0)", "q_pos0=0, kv_pos0=0)"),
    "varlen_keys_from_query_offsets": ("attention.py", "qs, qe, ks, ke = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]",
                                       "qs, qe, ks, ke = cu_q[b], cu_q[b + 1], cu_q[b], cu_q[b + 1]"),
    # oracle/paged.py: gather
    "page_index_off_by_one": ("paged.py", "pg = int(table[b, i])", "pg = int(table[b, max(i - 1, 0)])"),
    "page_table_ignored": ("paged.py", "pg = int(table[b, i])", "pg = b * max_pages + i"),
    "partial_page_dropped": ("paged.py", "for i in range((n + page_size - 1) // page_size):",
                             "for i in range(n // page_size):"),
    "slot_offset_shifted": ("paged.py", "out[b, lo:hi] = pool[pg, : hi - lo]",
                            "out[b, lo:hi] = pool[pg, page_size - (hi - lo):]"),
    # oracle/stream.py: the (query block, key chunk) decomposition
    "chunk_test_off_by_one": ("stream.py", "if causal and kv_pos0 + kc > q_last:",
                              "if causal and kv_pos0 + kc >= q_last:"),
    "chunk_test_at_block_start": ("stream.py", "q_last = q_pos0 + min(S, qb + Bq) - 1", "q_last = q_pos0 + qb"),
    "task_query_offset_dropped": ("stream.py", "q_pos0=qb, kv_pos0=kc)", "q_pos0=0, kv_pos0=kc)"),
    "task_key_offset_dropped": ("stream.py", "q_pos0=qb, kv_pos0=kc)", "q_pos0=qb, kv_pos0=0)"),
}


def _mutant(fname, old, new):
    src = open(os.path.join(ORACLE, fname)).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("oracle_mutant_" + fname[:-3])
    mod.__package__ = "oracle"  # the paged oracle imports the attention oracle relatively
    exec(compile(src.replace(old, new), mod.__name__, "exec"), mod.__dict__)
    return mod


def _pins(fname):
    """(test module, attribute the pins call the oracle through, pin callables)."""
    if fname == "stream.py":
        shapes = [(37, 8, 8), (64, 16, 32), (50, 50, 7), (9, 4, 16)]
        return TO, "stream", [(lambda a=a, c=c: TO.test_stream_tasks_exact_cover(*a, c))
                              for a in shapes for c in (True, False)] + [TO.test_stream_chunked_equals_unsplit]
    if fname == "paged.py":
        return TP, "PG", [TP.test_gather_by_hand, TP.test_swapped_entries_change_the_result,
                          TP.test_unmapped_page_below_length_is_an_error,
                          lambda: TP.test_identity_table_equals_contiguous(128),
                          lambda: TP.test_permuted_pool_equals_contiguous(False),
                          lambda: TP.test_permuted_pool_equals_contiguous(True)]
    return None, "O", [TM.test_one_token_is_decode, TM.test_each_token_is_a_decode_over_its_prefix,
                       TM.test_fp8_scales_follow_the_tokens, TM.test_token_without_keys_is_empty,
                       TV.test_brute_force_scalar_loops, TV.test_order_of_sequences_does_not_matter,
                       TV.test_single_sequence_is_dense_prefill_with_past]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, monkeypatch):
    fname, old, new = MUTANTS[name]
    mod = _mutant(fname, old, new)
    target, attr, pins = _pins(fname)
    for m in ((target,) if target else (TM, TV)):
        monkeypatch.setattr(m, attr, mod)
    caught = 0
    for pin in pins:
        try:
            pin()
        except (Exception, pytest.fail.Exception):  # noqa: BLE001 - any failure counts as caught
            caught += 1
    assert caught, f"no pin caught mutant {name}"


def test_unmutated_oracles_pass_the_same_pins():
    for fname in ("attention.py", "paged.py", "stream.py"):
        _, _, pins = _pins(fname)
        for pin in pins:
            pin()
