"""The on-device decode loop (dec_generate) against step-by-step decoding and
the CPU oracle.

faster-qwen-asr GB10 record (notes.configuration): the emitted token is fed
back on the device; Baseten article ("Minimizing host-to-device syncs"): no
host read-back inside the loop.  dec_generate must equal n dec_step calls
that feed their ids back and advance the positions, and retire a sequence at
its end-of-sequence token."""
import numpy as np
import pytest
import torch

import oracle
from conftest import oracle_cache, oracle_shape, oracle_weights
from decoder_greedy_decode_b200 import capi, synth
from decoder_greedy_decode_b200.decoder import Decoder, to_device
from gpu_util import NEAR_TIE, i32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    capi.lib()


def _fixture(batch, seed, n0s, max_ctx=96, max_batch=None):
    s = synth.TINY
    w = synth.model_weights(s, seed=seed)
    kv_host, _ = synth.kv_prefill(s, batch, max_ctx, n0s, seed=seed + 1)
    dec = Decoder(s, to_device(w), max_batch=max_batch or batch)
    toks = [int(t) for t in synth.tokens(s.vocab, batch, seed=seed + 2)]
    return s, w, kv_host, dec, toks


def _cache(dec, batch, max_ctx, kv_host):
    kv = dec.kv_cache(batch, max_ctx)
    kv.values.copy_(kv_host.cuda())
    return kv


def _step_loop(dec, kv, toks, n0s, n, eos=-1):
    """dec_step n times, feeding the ids back; positions advance by one, and
    stop for a sequence after it emits eos (whose later outputs are eos)."""
    B = len(toks)
    tok, pos, done = i32(toks), i32(n0s), [False] * B
    out_all = []
    for _ in range(n):
        out = torch.empty(B, dtype=torch.int32, device="cuda")
        dec.step(kv, tok, pos, out)
        ids = out.cpu().tolist()
        p = pos.cpu().tolist()
        for b in range(B):
            if done[b]:
                ids[b] = eos
            elif eos >= 0 and ids[b] == eos:
                done[b] = True
            else:
                p[b] += 1
        out_all.append(ids)
        tok, pos = i32(ids), i32(p)
    return out_all, pos.cpu().tolist()


@pytest.mark.parametrize("batch,max_batch", [(2, 2), (6, 8)])
def test_generate_equals_step_loop(batch, max_batch):
    n0s = [20 + 7 * b for b in range(batch)]
    s, w, kv_host, dec, toks = _fixture(batch, 100 + batch, n0s, max_batch=max_batch)
    n = 12
    kv_a = _cache(dec, batch, 96, kv_host)
    out = torch.empty((n, batch), dtype=torch.int32, device="cuda")
    pos = i32(n0s)
    dec.generate(kv_a, i32(toks), pos, out)
    assert dec.check() == 0
    kv_b = _cache(dec, batch, 96, kv_host)
    ref, ref_pos = _step_loop(dec, kv_b, toks, n0s, n)
    assert out.cpu().tolist() == ref          # the same kernels: identical ids
    assert pos.cpu().tolist() == ref_pos == [p + n for p in n0s]
    assert torch.equal(kv_a.buf, kv_b.buf)
    # and the oracle's greedy sequence, up to a permitted near-tie
    m = oracle.Model(oracle_shape(s), oracle_weights(w))
    got = np.array(ref)
    for b in range(batch):
        cache = oracle_cache(kv_host, None, b)
        tok = toks[b]
        for i in range(n):
            r = m.step(cache, tok, n0s[b] + i)
            if got[i, b] != r.token:
                assert r.margin < NEAR_TIE, f"seq {b} step {i}"
                break
            tok = r.token
    dec.close()


def _seq_rows(kv, b, lo, hi):
    """Cache rows [lo, hi) of sequence b (all layers, K and V) as raw bits."""
    return kv.values[:, :, b, :, lo:hi].contiguous().view(torch.int16)


@pytest.mark.parametrize("batch,max_batch", [(2, 2), (6, 8)])
def test_generate_retires_a_sequence_at_eos(batch, max_batch):
    """A sequence that emits the end token stops: its later ids are the end
    token, its position stays at the row of that step, and its cache holds
    exactly what a loop that stops stepping it there leaves (no later write
    into its rows)."""
    n = 10
    n0s = [30 + 10 * b for b in range(batch)]
    s, w, kv_host, dec, toks = _fixture(batch, 120, n0s, max_batch=max_batch)
    # the token sequence 0 emits at step 4 becomes the end token
    kv_r = _cache(dec, batch, 96, kv_host)
    free, _ = _step_loop(dec, kv_r, toks, n0s, n)
    eos = free[4][0]
    first = {b: next((i for i in range(n) if free[i][b] == eos), None) for b in range(batch)}
    kv_a = _cache(dec, batch, 96, kv_host)
    out = torch.empty((n, batch), dtype=torch.int32, device="cuda")
    pos = i32(n0s)
    dec.generate(kv_a, i32(toks), pos, out, eos=eos)
    assert dec.check() == 0
    got = out.cpu().tolist()
    kv_b = _cache(dec, batch, 96, kv_host)
    ref, ref_pos = _step_loop(dec, kv_b, toks, n0s, n, eos=eos)
    assert got == ref and pos.cpu().tolist() == ref_pos
    f0 = first[0]
    assert f0 is not None and f0 <= 4
    assert all(got[i][0] == eos for i in range(f0, n))
    assert ref_pos[0] == n0s[0] + f0          # the position stopped at the eos step
    if first[1] is None:
        assert ref_pos[1] == n0s[1] + n
    # sequence 0's cache: rows 0 .. n0 + f0 equal those of a loop that ran
    # only the steps up to and including the eos step; every later row still
    # holds the prefill
    kv_c = _cache(dec, batch, 96, kv_host)
    _step_loop(dec, kv_c, toks, n0s, f0 + 1)
    last = n0s[0] + f0 + 1
    assert torch.equal(_seq_rows(kv_a, 0, 0, last), _seq_rows(kv_c, 0, 0, last))
    init = _cache(dec, batch, 96, kv_host)
    assert torch.equal(_seq_rows(kv_a, 0, last, 96), _seq_rows(init, 0, last, 96))
    dec.close()


def test_generate_stops_when_every_sequence_retired():
    """When every sequence has emitted the end token the remaining steps are
    not run: their ids are the end token and the positions stay."""
    n = 12
    n0s = [25]
    s, w, kv_host, dec, toks = _fixture(1, 140, n0s)
    kv_r = _cache(dec, 1, 96, kv_host)
    free, _ = _step_loop(dec, kv_r, toks, n0s, n)
    eos = free[2][0]
    f0 = next(i for i in range(n) if free[i][0] == eos)
    kv_a = _cache(dec, 1, 96, kv_host)
    out = torch.full((n, 1), -7, dtype=torch.int32, device="cuda")
    pos = i32(n0s)
    dec.generate(kv_a, i32(toks), pos, out, eos=eos)
    assert dec.check() == 0
    got = [r[0] for r in out.cpu().tolist()]
    assert got[:f0 + 1] == [free[i][0] for i in range(f0 + 1)]
    assert all(g == eos for g in got[f0:])
    assert pos.cpu().tolist() == [n0s[0] + f0]
    dec.close()


def test_generate_position_past_the_cache_is_reported():
    """A sequence that would step past max_ctx stops the loop: DEC_DEV_BAD_POSITION,
    and the steps that could not run report -1."""
    s, w, kv_host, dec, toks = _fixture(1, 150, [90])
    kv = _cache(dec, 1, 96, kv_host)
    out = torch.full((8, 1), -7, dtype=torch.int32, device="cuda")
    pos = i32([90])
    dec.generate(kv, i32(toks), pos, out)
    assert dec.check() == capi.DEC_DEV_BAD_POSITION
    got = [r[0] for r in out.cpu().tolist()]
    assert all(0 <= g < s.vocab for g in got[:6]) and got[6:] == [-1, -1]
    dec.close()


def test_generate_rejects_bad_arguments():
    s, w, kv_host, dec, toks = _fixture(1, 130, [10])
    kv = _cache(dec, 1, 96, kv_host)
    out = torch.empty((2, 1), dtype=torch.int32, device="cuda")
    with pytest.raises(RuntimeError):
        capi.dec_generate(dec.h, 1, 0, i32(toks), i32([10]), kv.kv, out)
    with pytest.raises(RuntimeError):
        capi.dec_generate(dec.h, 2, 2, i32(toks), i32([10]), kv.kv, out)
    dec.close()


def _follows_oracle(m, caches, toks, n0s, got, n):
    """The ids of each sequence are the oracle's greedy ids for the first n
    steps, up to the first permitted near-tie."""
    for b, cache in enumerate(caches):
        tok = toks[b]
        for i in range(n):
            r = m.step(cache, tok, n0s[b] + i)
            if got[i][b] != r.token:
                assert r.margin < NEAR_TIE, f"seq {b} step {i}"
                break
            tok = r.token


@pytest.mark.parametrize("batch,max_batch", [(3, 4), (6, 8)])
def test_generate_fp8_cache_equals_step_loop(batch, max_batch):
    """An E4M3 cache (one fp32 scale per row): batch 3 runs on the persistent
    kernel, batch 6 on the batched step.  The loop equals dec_step calls bit
    for bit and follows the oracle's E4M3-cache model."""
    s = synth.TINY
    n0s = [15 + 9 * b for b in range(batch)]
    w = synth.model_weights(s, seed=160 + batch)
    codes, scales = synth.kv_prefill(s, batch, 96, n0s, seed=161 + batch, kind="fp8")
    dec = Decoder(s, to_device(w), max_batch=max_batch)
    toks = [int(t) for t in synth.tokens(s.vocab, batch, seed=162 + batch)]

    def cache():
        kv = dec.kv_cache(batch, 96, "fp8")
        kv.codes.copy_(codes.cuda())
        kv.scales.copy_(scales.cuda())
        return kv

    n = 10
    kv_a = cache()
    out = torch.empty((n, batch), dtype=torch.int32, device="cuda")
    pos = i32(n0s)
    dec.generate(kv_a, i32(toks), pos, out)
    assert dec.check() == 0
    kv_b = cache()
    ref, ref_pos = _step_loop(dec, kv_b, toks, n0s, n)
    assert out.cpu().tolist() == ref
    assert pos.cpu().tolist() == ref_pos == [p + n for p in n0s]
    assert torch.equal(kv_a.buf, kv_b.buf)
    m = oracle.Model(oracle_shape(s), oracle_weights(w))
    _follows_oracle(m, [oracle_cache(codes, scales, b) for b in range(batch)], toks, n0s, ref, n)
    dec.close()


def test_0p6b_bs1_generate_130_steps_in_one_launch():
    """The one-launch loop as the benchmark runs it: 0.6B shape, batch 1, 795
    prefilled rows, the 130-token window ("Qwen3-ASR -- Latency & Bottleneck
    Analysis", 01 Method & setup) in one dec_generate call.  It equals 130
    dec_step calls bit for bit (ids, final position, every cache row), and its
    first 8 ids are the oracle's greedy ids (up to a permitted near-tie)."""
    s = synth.QWEN3_0_6B
    w = synth.model_weights(s, seed=2)
    dec = Decoder(s, to_device(w), 1)
    kv_host, _ = synth.kv_prefill(s, 1, 928, [795], seed=3)
    tok0 = int(synth.tokens(s.vocab, 1, seed=4)[0])
    n = 130
    kv_a = _cache(dec, 1, 928, kv_host)
    out = torch.full((n, 1), -7, dtype=torch.int32, device="cuda")
    pos = i32([795])
    dec.generate(kv_a, i32([tok0]), pos, out)
    assert dec.check() == 0
    got = out.cpu().tolist()
    kv_b = _cache(dec, 1, 928, kv_host)
    ref, ref_pos = _step_loop(dec, kv_b, [tok0], [795], n)
    assert got == ref
    assert pos.cpu().tolist() == ref_pos == [795 + n]
    assert torch.equal(kv_a.buf, kv_b.buf)
    del kv_a, kv_b
    m = oracle.Model(oracle_shape(s), oracle_weights(w))
    _follows_oracle(m, [oracle_cache(kv_host, None, 0)], [tok0], [795], got, 8)
    dec.close()
