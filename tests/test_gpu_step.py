"""Parity of the CUDA decode step (through the C ABI) against the CPU oracle.

Teacher forcing: every step both sides get the oracle's token, each keeps
its own KV cache, and logits, residual stream, emitted id and the appended
cache rows are compared ("Can CTC make Qwen3-ASR faster?", 11 Phase A:
switchable paths compared token for token; faster-qwen-asr GB10 record,
notes.correctness: transcripts byte-identical across paths)."""
import numpy as np
import pytest
import torch

import oracle
from conftest import oracle_cache, oracle_shape, oracle_weights
from decoder_greedy_decode_b200 import capi, synth
from decoder_greedy_decode_b200.decoder import Decoder, to_device
from gpu_util import assert_close, assert_id, bf16_values, close_report, i32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    capi.lib()


def _setup(s, seed, batch, max_ctx, lengths, kind="bf16", gain_std=0.0):
    w = synth.model_weights(s, seed=seed, gain_std=gain_std)
    kv_host, sc_host = synth.kv_prefill(s, batch, max_ctx, lengths, seed=seed + 100, kind=kind)
    m = oracle.Model(oracle_shape(s), oracle_weights(w))
    caches = [oracle_cache(kv_host, sc_host, b) for b in range(batch)]
    dec = Decoder(s, to_device(w), max_batch=max(batch, 1))
    kv = dec.kv_cache(batch, max_ctx, kind)
    if kind == "bf16":
        kv.values.copy_(kv_host.cuda())
    else:
        kv.codes.copy_(kv_host.cuda())
        kv.scales.copy_(sc_host.cuda())
    return w, m, caches, dec, kv


def _gpu_step(dec, kv, toks, poss, want_hidden=True):
    s = dec.shape
    B = len(toks)
    out = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    logits = torch.empty((B, s.vocab), dtype=torch.float32, device="cuda")
    if want_hidden:
        hid = torch.empty((s.n_layers + 1, B, s.hidden), dtype=torch.float32, device="cuda")
        dec.step_debug(kv, i32(toks), i32(poss), out, logits, hid)
    else:
        hid = None
        dec.step(kv, i32(toks), i32(poss), out, logits)
    st = dec.check()
    assert st == 0, capi.error_string(st)
    return out.cpu().numpy(), logits.cpu().numpy(), (hid.cpu().numpy() if want_hidden else None)


def _check_kv_row(kv, cache, b, p, what):
    """The row the step appended at position p of sequence b vs the oracle's."""
    if kv.dtype == "bf16":
        got = bf16_values(kv.values[:, :, b, :, p, :])           # [L, 2, Hkv, D]
        ref = oracle.bf16_to_double(cache.kv[:, :, :, p, :])
        assert_close(got, ref, what + " appended KV row")
    else:
        codes = kv.codes[:, :, b, :, p, :].cpu().numpy()
        scales = kv.scales[:, :, b, :, p].cpu().numpy()
        got = oracle.e4m3_decode(codes) * scales[..., None]
        ref = oracle.e4m3_decode(cache.kv[:, :, :, p, :]) * cache.scales[:, :, :, p][..., None]
        # Each side quantises its own k (scale = amax / 448, RNE to E4M3).  An
        # element near a rounding boundary may land one code apart: at most one
        # top-binade step, 32 x scale.  When the two amax differ (within the k
        # tolerance) the same code also decodes to values 448 x |scale gap|
        # apart.
        ref_sc = cache.scales[:, :, :, p][..., None]
        bound = 32.0 * scales[..., None] + 448.0 * np.abs(scales[..., None] - ref_sc)
        assert np.all(np.abs(got - ref) <= bound * (1 + 1e-6) + 1e-12), what
        assert close_report(got, ref)[1] <= 0.05, what


def _run_teacher_forced(s, seed, batch, max_ctx, lengths, steps, kind="bf16", gain_std=0.0,
                        check_unchanged=True):
    w, m, caches, dec, kv = _setup(s, seed, batch, max_ctx, lengths, kind, gain_std)
    toks = [int(t) for t in synth.tokens(s.vocab, batch, seed=seed + 200)]
    for t in range(steps):
        poss = [lengths[b] + t for b in range(batch)]
        refs = [m.step(caches[b], toks[b], poss[b], want_hidden=True) for b in range(batch)]
        before = kv.buf.clone() if check_unchanged else None
        ids, logits, hid = _gpu_step(dec, kv, toks, poss)
        for b in range(batch):
            tag = f"step {t} seq {b} p={poss[b]}"
            assert_close(logits[b], refs[b].logits, tag + " logits")
            for l in range(s.n_layers + 1):
                assert_close(hid[l, b], refs[b].hidden[l], tag + f" hidden {l}")
            assert_id(int(ids[b]), refs[b], tag)
            _check_kv_row(kv, caches[b], b, poss[b], tag)
        if check_unchanged:
            _check_only_rows_changed(before, kv, poss)
        toks = [r.token for r in refs]
    dec.close()


def _check_only_rows_changed(before, kv, poss):
    """Every cache byte outside rows poss[b] of sequence b is unchanged."""
    if kv.dtype == "bf16":
        a = before.view(torch.bfloat16).view(kv.values.shape)
        bnow = kv.values
        mask = torch.ones(kv.values.shape[:-1], dtype=torch.bool, device="cuda")
        for b, p in enumerate(poss):
            mask[:, :, b, :, p] = False
        assert torch.equal(a.view(torch.int16)[mask], bnow.view(torch.int16)[mask])
    else:
        codes_b = before[:kv.codes.numel()].view(kv.codes.shape)
        mask = torch.ones(kv.codes.shape[:-1], dtype=torch.bool, device="cuda")
        for b, p in enumerate(poss):
            mask[:, :, b, :, p] = False
        assert torch.equal(codes_b[mask], kv.codes[mask])


# ------------------------------------------------------------------ tiny
def test_tiny_bs1_teacher_forced_16_steps():
    """The small decoder: 2 layers, hidden 256, 4/2 heads of 64, FFN 768,
    vocab 4096; cache prefilled with 128 rows; 16 greedy steps."""
    _run_teacher_forced(synth.TINY, seed=1, batch=1, max_ctx=256, lengths=[128], steps=16)


def test_tiny_gains_not_one():
    _run_teacher_forced(synth.TINY, seed=2, batch=1, max_ctx=64, lengths=[20], steps=3,
                        gain_std=0.1)


def test_tiny_ragged_batch_with_empty_cache():
    # p = 0 attends only to itself; ragged contexts across the batch
    _run_teacher_forced(synth.TINY, seed=3, batch=4, max_ctx=320, lengths=[0, 1, 150, 300],
                        steps=3)


def test_tiny_fp8_cache():
    _run_teacher_forced(synth.TINY, seed=4, batch=2, max_ctx=256, lengths=[128, 77], steps=6,
                        kind="fp8")


def test_tiny_last_position():
    _run_teacher_forced(synth.TINY, seed=5, batch=1, max_ctx=64, lengths=[63], steps=1)


def test_gqa_three_query_heads_per_kv_head():
    s = synth.ModelShape(2, 256, 12, 4, 64, 512, 1000)
    _run_teacher_forced(s, seed=6, batch=2, max_ctx=128, lengths=[40, 90], steps=2)


def test_one_query_head_per_kv_head_d128():
    s = synth.ModelShape(1, 512, 4, 4, 128, 1024, 2000)
    _run_teacher_forced(s, seed=7, batch=1, max_ctx=96, lengths=[50], steps=2)


# ---------------------------------------------------- invalid inputs / API
def test_invalid_position_and_token_raise_status_and_leave_cache():
    s = synth.TINY
    w, m, caches, dec, kv = _setup(s, 8, 1, 64, [10])
    before = kv.buf.clone()
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    dec.step(kv, i32([5]), i32([64]), out)                 # position == max_ctx
    assert dec.check() == capi.DEC_DEV_BAD_POSITION
    assert int(out[0]) == -1
    dec.step(kv, i32([s.vocab]), i32([10]), out)           # token == vocab
    assert dec.check() == capi.DEC_DEV_BAD_TOKEN
    dec.step(kv, i32([-1]), i32([-3]), out)
    assert dec.check() == capi.DEC_DEV_BAD_POSITION | capi.DEC_DEV_BAD_TOKEN
    assert torch.equal(before, kv.buf)
    # the context stays usable: a valid step still matches the oracle
    r = m.step(caches[0], 5, 10)
    ids, logits, _ = _gpu_step(dec, kv, [5], [10], want_hidden=False)
    assert_close(logits[0], r.logits, "after invalid steps")
    dec.close()


def test_host_arguments_rejected():
    s = synth.TINY
    w, m, caches, dec, kv = _setup(s, 9, 1, 64, [10])
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(capi.DecError):
        capi.dec_step(dec.h, 2, i32([1, 2]), i32([1, 2]), kv.kv, out)   # batch > max_batch
    with pytest.raises(capi.DecError):
        capi.dec_step(dec.h, 1, None, i32([1]), kv.kv, out)
    bad = torch.zeros(100, dtype=torch.uint8, device="cuda")
    with pytest.raises(capi.DecError):
        capi.dec_kv_alloc(dec.h, 1, 64, capi.DEC_KV_BF16, bad, 100)
    with pytest.raises(capi.DecError):
        capi.dec_kv_alloc(dec.h, 1, 60, capi.DEC_KV_BF16, kv.buf, kv.buf.numel())
    dec.close()


def test_logits_optional_and_out_ids_alias_token_ids():
    """out_ids may alias token_ids (device-side token feedback): a free-running
    self-feeding loop gives the same ids as the oracle's own greedy loop up to
    the first near-tie of the oracle."""
    s = synth.TINY
    w, m, caches, dec, kv = _setup(s, 10, 1, 128, [64])
    tok = int(synth.tokens(s.vocab, 1, seed=11)[0])
    buf = i32([tok])
    ref_tok = tok
    for t in range(12):
        p = 64 + t
        r = m.step(caches[0], ref_tok, p)
        dec.step(kv, buf, i32([p]), buf)            # no logits, aliasing ids
        assert dec.check() == 0
        got = int(buf[0])
        if r.margin < 1e-2:
            break
        assert got == r.token, f"step {t}"
        ref_tok = r.token
    dec.close()


def test_step_host_matches_device_step():
    s = synth.TINY
    w, m, caches, dec, kv = _setup(s, 12, 2, 128, [30, 60])
    kv2 = dec.kv_cache(2, 128)
    kv2.buf.copy_(kv.buf)
    toks, poss = [3, 4000], [30, 60]
    out_h = torch.zeros(2, dtype=torch.int32).pin_memory()
    log_h = torch.zeros((2, s.vocab), dtype=torch.float32).pin_memory()
    dec.step_host(kv, torch.tensor(toks, dtype=torch.int32), torch.tensor(poss, dtype=torch.int32),
                  out_h, log_h)
    ids, logits, _ = _gpu_step(dec, kv2, toks, poss, want_hidden=False)
    assert np.array_equal(out_h.numpy(), ids)
    assert np.array_equal(log_h.numpy(), logits)
    assert torch.equal(kv.buf, kv2.buf)
    for b in range(2):
        assert_close(logits[b], m.step(caches[b], toks[b], poss[b]).logits, "step_host")
    dec.close()


# ------------------------------------------------------------ 0.6B shape
@pytest.fixture(scope="module")
def big06():
    s = synth.QWEN3_0_6B
    w = synth.model_weights(s, seed=2)
    return s, w, oracle.Model(oracle_shape(s), oracle_weights(w)), to_device(w)


def test_0p6b_bs1_ctx795_teacher_forced(big06):
    """0.6B shape, batch 1, 795 prefilled rows: the first decode steps, and the
    step at the end of the 130-token window (p = 924) on a 924-row prefill."""
    s, w, m, wd = big06
    dec = Decoder(s, wd, 1)
    for n0, steps in ((795, 3), (924, 1)):
        kv_host, _ = synth.kv_prefill(s, 1, 928, [n0], seed=3)
        cache = oracle_cache(kv_host, None, 0)
        kv = dec.kv_cache(1, 928)
        kv.values.copy_(kv_host.cuda())
        tok = int(synth.tokens(s.vocab, 1, seed=4)[0])
        for t in range(steps):
            p = n0 + t
            r = m.step(cache, tok, p, want_hidden=True)
            ids, logits, hid = _gpu_step(dec, kv, [tok], [p])
            tag = f"0.6B p={p}"
            assert_close(logits[0], r.logits, tag + " logits")
            for l in (0, 1, 14, 27, 28):
                assert_close(hid[l, 0], r.hidden[l], tag + f" hidden {l}")
            assert_id(int(ids[0]), r, tag)
            _check_kv_row(kv, cache, 0, p, tag)
            tok = r.token
        del kv
    dec.close()


def test_0p6b_bs1_window_130_teacher_forced(big06):
    """The whole 130-token window of the 0.6B workload ("Qwen3-ASR -- Latency &
    Bottleneck Analysis", 01 Method & setup: 795 prompt tokens, then 130
    generated), positions 795 .. 924, teacher-forced: every step's logits,
    every layer's residual stream, the emitted id and the appended cache row
    against the oracle."""
    s, w, m, wd = big06
    dec = Decoder(s, wd, 1)
    kv_host, _ = synth.kv_prefill(s, 1, 928, [795], seed=3)
    cache = oracle_cache(kv_host, None, 0)
    kv = dec.kv_cache(1, 928)
    kv.values.copy_(kv_host.cuda())
    tok = int(synth.tokens(s.vocab, 1, seed=4)[0])
    worst = (0.0, 0.0)
    for t in range(130):
        p = 795 + t
        r = m.step(cache, tok, p, want_hidden=True)
        ids, logits, hid = _gpu_step(dec, kv, [tok], [p])
        tag = f"0.6B window p={p}"
        ma, rl = assert_close(logits[0], r.logits, tag + " logits")
        worst = (max(worst[0], ma), max(worst[1], rl))
        for l in range(s.n_layers + 1):
            assert_close(hid[l, 0], r.hidden[l], tag + f" hidden {l}")
        assert_id(int(ids[0]), r, tag)
        _check_kv_row(kv, cache, 0, p, tag)
        tok = r.token
    print(f"130-step window: worst logits max-abs {worst[0]:.3g}, rel-L2 {worst[1]:.3g}")
    del kv
    dec.close()


def test_0p6b_bs1_free_running_follows_oracle_greedy(big06):
    """The device feeds its own ids back (out_ids aliases token_ids) from
    position 795; the ids equal the oracle's own greedy sequence up to the
    oracle's first near-tie (top-2 margin below 1e-2), after which the two
    may legitimately part."""
    s, w, m, wd = big06
    dec = Decoder(s, wd, 1)
    kv_host, _ = synth.kv_prefill(s, 1, 928, [795], seed=3)
    cache = oracle_cache(kv_host, None, 0)
    kv = dec.kv_cache(1, 928)
    kv.values.copy_(kv_host.cuda())
    tok = int(synth.tokens(s.vocab, 1, seed=4)[0])
    buf = i32([tok])
    n = 0
    for t in range(130):
        p = 795 + t
        r = m.step(cache, tok, p)
        dec.step(kv, buf, i32([p]), buf)
        assert dec.check() == 0
        if r.margin < 1e-2:
            break
        assert int(buf[0]) == r.token, f"free-running step {t} (p={p})"
        tok = r.token
        n += 1
    assert n >= 1
    print(f"free-running: {n} steps equal to the oracle's greedy ids before its first near-tie")
    del kv
    dec.close()


def test_0p6b_batch4_ragged(big06):
    s, w, m, wd = big06
    dec = Decoder(s, wd, 4)
    lengths = [200, 420, 1, 333]
    kv_host, _ = synth.kv_prefill(s, 4, 432, lengths, seed=5)
    caches = [oracle_cache(kv_host, None, b) for b in range(4)]
    kv = dec.kv_cache(4, 432)
    kv.values.copy_(kv_host.cuda())
    toks = [int(t) for t in synth.tokens(s.vocab, 4, seed=6)]
    refs = [m.step(caches[b], toks[b], lengths[b]) for b in range(4)]
    ids, logits, _ = _gpu_step(dec, kv, toks, lengths, want_hidden=False)
    for b in range(4):
        assert_close(logits[b], refs[b].logits, f"bs4 seq {b}")
        assert_id(int(ids[b]), refs[b], f"bs4 seq {b}")
        _check_kv_row(kv, caches[b], b, lengths[b], f"bs4 seq {b}")
    dec.close()


# ------------------------------------------------------------ 1.7B shape
@pytest.fixture(scope="module")
def big17():
    s = synth.QWEN3_1_7B
    w = synth.model_weights(s, seed=17)
    return s, w, oracle.Model(oracle_shape(s), oracle_weights(w)), to_device(w)


@pytest.mark.parametrize("kind,n0", [("bf16", 4095), ("fp8", 2500)])
def test_1p7b_bs1_long_context(big17, kind, n0):
    """1.7B shape (hidden 2048, FFN 6144), batch 1, contexts up to 4096, bf16
    cache and the E4M3 cache read back from the same stored bytes."""
    s, w, m, wd = big17
    dec = Decoder(s, wd, 1)
    kv_host, sc_host = synth.kv_prefill(s, 1, 4096, [n0], seed=18, kind=kind)
    cache = oracle_cache(kv_host, sc_host, 0)
    kv = dec.kv_cache(1, 4096, kind)
    if kind == "bf16":
        kv.values.copy_(kv_host.cuda())
    else:
        kv.codes.copy_(kv_host.cuda())
        kv.scales.copy_(sc_host.cuda())
    tok = int(synth.tokens(s.vocab, 1, seed=19)[0])
    r = m.step(cache, tok, n0, want_hidden=True)
    ids, logits, hid = _gpu_step(dec, kv, [tok], [n0])
    assert_close(logits[0], r.logits, f"1.7B {kind} logits")
    for l in (1, 28):
        assert_close(hid[l, 0], r.hidden[l], f"1.7B {kind} hidden {l}")
    assert_id(int(ids[0]), r, f"1.7B {kind}")
    _check_kv_row(kv, cache, 0, n0, f"1.7B {kind}")
    del kv
    dec.close()
