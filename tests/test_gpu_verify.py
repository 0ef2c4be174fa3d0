"""Block verification (dec_verify) and greedy speculative decoding on the GPU
against the CPU oracle.

"Can CTC make Qwen3-ASR faster?", §11 Phase A: one target forward over a
draft block returns the target's greedy ids for every position (the id at
position i checks draft token i + 1); with the baseline transcript itself as
the draft, and with mismatches injected at chosen positions, the committed
tokens must equal ordinary greedy decoding, and the cache crop is the host's
position."""
import numpy as np
import pytest
import torch

import oracle
from conftest import oracle_cache, oracle_shape, oracle_weights
from decoder_greedy_decode_b200 import capi, synth
from decoder_greedy_decode_b200.decoder import Decoder, to_device
from gpu_util import NEAR_TIE, assert_close, assert_id, i32
from test_gpu_step import _check_kv_row

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    capi.lib()


def _setup(s, seed, kv_batch, max_ctx, lengths, kind="bf16", max_batch=16):
    w = synth.model_weights(s, seed=seed)
    kv_host, sc_host = synth.kv_prefill(s, kv_batch, max_ctx, lengths, seed=seed + 1, kind=kind)
    m = oracle.Model(oracle_shape(s), oracle_weights(w))
    dec = Decoder(s, to_device(w), max_batch=max_batch)
    kv = dec.kv_cache(kv_batch, max_ctx, kind)
    if kind == "bf16":
        kv.values.copy_(kv_host.cuda())
    else:
        kv.codes.copy_(kv_host.cuda())
        kv.scales.copy_(sc_host.cuda())
    return m, dec, kv, kv_host, sc_host


def _verify(dec, kv, toks, p0, seq):
    k = len(toks)
    out = torch.full((k,), -7, dtype=torch.int32, device="cuda")
    logits = torch.empty((k, dec.shape.vocab), dtype=torch.float32, device="cuda")
    dec.verify(kv, i32(toks), i32(range(p0, p0 + k)), seq, out, logits)
    st = dec.check()
    assert st == 0, capi.error_string(st)
    return out.cpu().tolist(), logits.cpu().numpy()


@pytest.mark.parametrize("kind", ["bf16", "fp8"])
@pytest.mark.parametrize("k,max_batch", [(1, 16), (2, 16), (3, 16), (4, 16), (9, 16),
                                         (2, 4), (3, 4), (4, 4)])
def test_verify_block_equals_single_steps(kind, k, max_batch):
    """A block of k tokens of sequence 1 (of 3 in the cache) equals k
    teacher-forced single steps of the oracle: logits, ids, appended rows;
    the other sequences' rows are untouched.  One-token blocks run on the
    persistent kernel, and so do blocks of 2 to 4 on a handle without a
    batched step (max_batch 4; the prefix read once for the whole block);
    the others run on the batched step."""
    s = synth.TINY
    n0, seq = 40, 1
    m, dec, kv, kv_host, sc_host = _setup(s, 80, 3, 64, [30, n0, 50], kind, max_batch=max_batch)
    cache = oracle_cache(kv_host, sc_host, seq)
    toks = [int(t) for t in synth.tokens(s.vocab, k, seed=81)]
    before = kv.buf.clone()
    ids, logits = _verify(dec, kv, toks, n0, seq)
    for i in range(k):
        r = m.step(cache, toks[i], n0 + i)
        assert_close(logits[i], r.logits, f"row {i} logits")
        assert_id(ids[i], r, f"row {i}")
        _check_kv_row(kv, cache, seq, n0 + i, f"row {i}")
    # sequences 0 and 2 unchanged
    if kind == "bf16":
        a = before.view(torch.bfloat16).view(kv.values.shape)
        for b in (0, 2):
            assert torch.equal(a[:, :, b].view(torch.int16), kv.values[:, :, b].view(torch.int16))
    dec.close()


def test_speculative_decode_commits_the_greedy_sequence():
    """Oracle-draft speculation with injected mismatches: blocks of 8, the
    draft is the oracle's greedy continuation with some tokens replaced;
    after verify + greedy acceptance the committed tokens equal the greedy
    sequence (up to a permitted near-tie, where the test stops)."""
    s = synth.TINY
    n0, total, blk = 24, 40, 8
    m, dec, kv, kv_host, _ = _setup(s, 90, 1, 96, [n0])
    # reference: the oracle's own greedy decode from the same cache
    ref_cache = oracle_cache(kv_host, None, 0)
    t0 = int(synth.tokens(s.vocab, 1, seed=91)[0])
    ref, margins, tok = [], [], t0
    for i in range(total + blk):
        r = m.step(ref_cache, tok, n0 + i)
        ref.append(r.token)
        margins.append(r.margin)
        tok = r.token
    rng = np.random.default_rng(92)
    committed, cur, p = [], t0, n0
    while len(committed) < total:
        c = len(committed)
        draft = list(ref[c:c + blk - 1])
        if rng.random() < 0.6:  # inject a mismatch at a random draft position
            j = int(rng.integers(0, len(draft)))
            draft[j] = (draft[j] + 1 + int(rng.integers(0, s.vocab - 1))) % s.vocab
        ids, _ = _verify(dec, kv, [cur] + draft, p, 0)
        emitted = capi.dec_accept_greedy([cur] + draft, ids)
        for e in emitted:
            i = len(committed)
            if i >= total:
                break
            if e != ref[i]:
                assert margins[i] < NEAR_TIE, f"token {i}: {e} != {ref[i]}"
                dec.close()
                return  # a permitted near-tie: the sequences may part here
            committed.append(e)
        p += len(emitted)  # the cache crop is the host's position
        cur = emitted[-1]
    assert committed == ref[:total]
    dec.close()


def test_verify_block_limits():
    """A handle of max_batch 4 verifies blocks of up to 4 (persistent kernel),
    not 5; a block whose positions are not consecutive is reported on the
    device and leaves the cache unchanged."""
    s = synth.TINY
    w = to_device(synth.model_weights(s, seed=93))
    dec = Decoder(s, w, max_batch=4)
    kv = dec.kv_cache(1, 32)
    out = torch.zeros(5, dtype=torch.int32, device="cuda")
    with pytest.raises(RuntimeError):
        dec.verify(kv, i32([1, 2, 3, 4, 5]), i32([3, 4, 5, 6, 7]), 0, out)
    before = kv.buf.clone()
    dec.verify(kv, i32([1, 2]), i32([3, 5]), 0, out[:2])
    assert dec.check() == capi.DEC_DEV_BAD_POSITION
    assert out[:2].cpu().tolist() == [-1, -1]
    assert torch.equal(before, kv.buf)
    dec.verify(kv, i32([1, 2]), i32([3, 4]), 0, out[:2])
    assert dec.check() == 0
    dec.close()


@pytest.mark.parametrize("blk", [2, 4])
def test_speculative_small_blocks_commit_the_greedy_sequence(blk):
    """Speculation with blocks of 2 and 4 (the persistent kernel verifies
    them): the committed tokens equal the oracle's greedy sequence."""
    s = synth.TINY
    n0, total = 24, 24
    m, dec, kv, kv_host, _ = _setup(s, 96, 1, 96, [n0], max_batch=4)
    ref_cache = oracle_cache(kv_host, None, 0)
    t0 = int(synth.tokens(s.vocab, 1, seed=97)[0])
    ref, margins, tok = [], [], t0
    for i in range(total + blk):
        r = m.step(ref_cache, tok, n0 + i)
        ref.append(r.token)
        margins.append(r.margin)
        tok = r.token
    rng = np.random.default_rng(98)
    committed, cur, p = [], t0, n0
    while len(committed) < total:
        c = len(committed)
        draft = list(ref[c:c + blk - 1])
        if rng.random() < 0.5:
            j = int(rng.integers(0, len(draft)))
            draft[j] = (draft[j] + 1 + int(rng.integers(0, s.vocab - 1))) % s.vocab
        ids, _ = _verify(dec, kv, [cur] + draft, p, 0)
        emitted = capi.dec_accept_greedy([cur] + draft, ids)
        for e in emitted:
            i = len(committed)
            if i >= total:
                break
            if e != ref[i]:
                assert margins[i] < NEAR_TIE, f"token {i}: {e} != {ref[i]}"
                dec.close()
                return
            committed.append(e)
        p += len(emitted)
        cur = emitted[-1]
    assert committed == ref[:total]
    dec.close()


@pytest.fixture(scope="module")
def big06():
    s = synth.QWEN3_0_6B
    w = synth.model_weights(s, seed=2)
    return s, w, to_device(w)


@pytest.mark.parametrize("k,max_batch", [(4, 4), (4, 64), (16, 64)])
def test_0p6b_verify_block(big06, k, max_batch):
    """0.6B shape, context 795, blocks of 4 (persistent kernel on a handle of
    max_batch 4, batched step otherwise) and 16 (batched step): sampled rows
    vs the oracle."""
    s, w, wd = big06
    n0 = 795
    kv_host, _ = synth.kv_prefill(s, 1, 816, [n0], seed=94)
    dec = Decoder(s, wd, max_batch=max_batch)
    kv = dec.kv_cache(1, 816)
    kv.values.copy_(kv_host.cuda())
    m = oracle.Model(oracle_shape(s), oracle_weights(w))
    cache = oracle_cache(kv_host, None, 0)
    toks = [int(t) for t in synth.tokens(s.vocab, k, seed=95)]
    ids, logits = _verify(dec, kv, toks, n0, 0)
    for i in range(k):
        r = m.step(cache, toks[i], n0 + i)
        if i in (0, k // 2, k - 1):
            assert_close(logits[i], r.logits, f"row {i} logits")
            _check_kv_row(kv, cache, 0, n0 + i, f"row {i}")
        assert_id(ids[i], r, f"row {i}")
    dec.close()
