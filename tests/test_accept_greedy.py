"""Greedy acceptance of a verified block (dec_accept_greedy, host-only).

The contract ("Can CTC make Qwen3-ASR faster?", §03 Speculative decoding and
§08): draft token t_{i+1} is accepted only while it equals the target's
greedy prediction at the position before it, out_ids[i]; at the first
mismatch the target's token is emitted instead and the rest is dropped;
after a full match the prediction after the last draft is the bonus token.
The expected outputs below are written out from that rule by hand."""
import pytest

from decoder_greedy_decode_b200 import capi


def test_full_match_emits_all_drafts_and_the_bonus():
    # t0 = 7, drafts 11 12 13; the target predicts 11 after 7, 12 after 11, ...
    assert capi.dec_accept_greedy([7, 11, 12, 13], [11, 12, 13, 99]) == [11, 12, 13, 99]


def test_first_draft_rejected():
    assert capi.dec_accept_greedy([7, 5, 12, 13], [11, 12, 13, 99]) == [11]


def test_mismatch_in_the_middle():
    # 11 accepted, 40 rejected (target says 12): emit 11 then the correction 12
    assert capi.dec_accept_greedy([7, 11, 40, 13, 14], [11, 12, 50, 60, 70]) == [11, 12]


def test_a_later_match_after_a_mismatch_is_not_accepted():
    # draft 13 would match out_ids[2], but the run already ended at index 1
    assert capi.dec_accept_greedy([7, 11, 40, 13], [11, 12, 13, 99]) == [11, 12]


def test_block_of_one_is_a_plain_step():
    assert capi.dec_accept_greedy([7], [11]) == [11]


def test_invalid_verify_step_is_rejected():
    with pytest.raises(RuntimeError):
        capi.dec_accept_greedy([7, 11], [-1, -1])
