"""Parity of the batched decode step (batch 5..64: tensor-core projections)
against the CPU oracle, through the C ABI.

The Baseten Qwen3-ASR article ("KV cache quantization") serves many
sequences at once; the step for a batch must give every sequence what the
single-sequence definition gives it.  Teacher forcing as in the other step
tests: both sides get the oracle's token every step and keep their own
caches; logits, residual stream, emitted id and appended cache rows are
compared per sequence."""
import numpy as np
import pytest
import torch

import oracle
from conftest import oracle_cache, oracle_shape, oracle_weights
from decoder_greedy_decode_b200 import capi, synth
from decoder_greedy_decode_b200.decoder import Decoder, quantize_int8, to_device
from gpu_util import assert_close, assert_id, i32
from test_gpu_step import _check_kv_row, _check_only_rows_changed, _gpu_step, _run_teacher_forced

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    capi.lib()


# ------------------------------------------------------------------ tiny
@pytest.mark.parametrize("batch", [5, 16, 64])
def test_tiny_batched_ragged_teacher_forced(batch):
    """Ragged contexts including an empty cache (p = 0) and the last row."""
    lengths = synth.ragged_lengths(0, 250, batch, seed=30 + batch)
    lengths[0], lengths[-1] = 0, 253
    _run_teacher_forced(synth.TINY, seed=31, batch=batch, max_ctx=256, lengths=lengths, steps=3)


def test_tiny_batched_fp8_cache():
    lengths = synth.ragged_lengths(1, 200, 24, seed=40)
    _run_teacher_forced(synth.TINY, seed=41, batch=24, max_ctx=224, lengths=lengths, steps=3,
                        kind="fp8")


def test_tiny_batched_gains_not_one():
    lengths = synth.ragged_lengths(10, 60, 8, seed=42)
    _run_teacher_forced(synth.TINY, seed=43, batch=8, max_ctx=80, lengths=lengths, steps=2,
                        gain_std=0.1)


def test_batched_gqa_and_d128_shapes():
    # 3 query heads per KV head (head_dim 64), then MHA with head_dim 128
    s = synth.ModelShape(2, 256, 12, 4, 64, 512, 1000)
    _run_teacher_forced(s, seed=44, batch=6, max_ctx=128, lengths=[40, 90, 0, 7, 126, 64],
                        steps=2)
    s = synth.ModelShape(1, 512, 4, 4, 128, 1024, 2000)
    _run_teacher_forced(s, seed=45, batch=9, max_ctx=96,
                        lengths=synth.ragged_lengths(0, 90, 9, seed=46), steps=2)


def test_vocab_not_a_multiple_of_the_tile():
    # 1000 = 7 full 128-row lm_head tiles + a ragged one (zero-filled by TMA)
    s = synth.ModelShape(1, 256, 4, 2, 64, 256, 1000)
    _run_teacher_forced(s, seed=47, batch=12, max_ctx=64,
                        lengths=synth.ragged_lengths(0, 60, 12, seed=48), steps=2)


def test_sequences_are_independent_of_the_batch():
    """Sequence b's results do not depend on which other sequences share the
    step: batch 64 and batch 7 over the same first 7 caches agree.  The
    projections agree bit for bit (the tensor-core tile always spans 64
    sequences and the split-K plan depends only on the shape); the attention
    chunking follows the batch, so the float results agree to rounding."""
    s = synth.TINY
    w = synth.model_weights(s, seed=50)
    wd = to_device(w)
    lengths = synth.ragged_lengths(0, 120, 64, seed=51)
    kv_host, _ = synth.kv_prefill(s, 64, 128, lengths, seed=52)
    toks = [int(t) for t in synth.tokens(s.vocab, 64, seed=53)]
    dec = Decoder(s, wd, 64)
    res = []
    for B in (64, 7):
        kv = dec.kv_cache(64, 128)
        kv.values.copy_(kv_host.cuda())
        ids, logits, hid = _gpu_step(dec, kv, toks[:B], lengths[:B])
        res.append((ids[:7], logits[:7], hid[:, :7],
                    kv.values[:, :, :7].float().cpu().numpy()))
    assert np.array_equal(res[0][0], res[1][0])
    for a, b in zip(res[0][1:3], res[1][1:3]):        # logits, residual stream
        assert np.max(np.abs(a - b)) <= 1e-4
    # cache rows of layers >= 1 come from attention outputs that differ by
    # fp32 rounding: their bf16 storage may differ by one unit in the last place
    ka, kb = res[0][3], res[1][3]
    assert np.all(np.abs(ka - kb) <= 2.0 ** -7 * np.maximum(np.abs(ka), np.abs(kb)))
    dec.close()


def test_batched_invalid_inputs_raise_status_and_leave_cache():
    s = synth.TINY
    w = synth.model_weights(s, seed=55)
    lengths = [10] * 8
    kv_host, _ = synth.kv_prefill(s, 8, 64, lengths, seed=56)
    m = oracle.Model(oracle_shape(s), oracle_weights(w))
    dec = Decoder(s, to_device(w), 8)
    kv = dec.kv_cache(8, 64)
    kv.values.copy_(kv_host.cuda())
    before = kv.buf.clone()
    out = torch.zeros(8, dtype=torch.int32, device="cuda")
    dec.step(kv, i32([5] * 8), i32([10] * 7 + [64]), out)          # one position == max_ctx
    assert dec.check() == capi.DEC_DEV_BAD_POSITION
    assert torch.all(out == -1)
    dec.step(kv, i32([5] * 7 + [s.vocab]), i32([10] * 8), out)     # one token == vocab
    assert dec.check() == capi.DEC_DEV_BAD_TOKEN
    assert torch.all(out == -1)
    assert torch.equal(before, kv.buf)
    # the context stays usable: a valid step matches the oracle
    cache = oracle_cache(kv_host, None, 3)
    r = m.step(cache, 5, 10)
    ids, logits, _ = _gpu_step(dec, kv, [5] * 8, [10] * 8, want_hidden=False)
    assert_close(logits[3], r.logits, "after invalid steps")
    assert_id(int(ids[3]), r, "after invalid steps")
    dec.close()


def test_batched_self_feeding_and_no_logits():
    """out_ids may alias token_ids; out_logits may be NULL."""
    s = synth.TINY
    w = synth.model_weights(s, seed=57)
    lengths = synth.ragged_lengths(5, 50, 10, seed=58)
    kv_host, _ = synth.kv_prefill(s, 10, 64, lengths, seed=59)
    m = oracle.Model(oracle_shape(s), oracle_weights(w))
    caches = [oracle_cache(kv_host, None, b) for b in range(10)]
    dec = Decoder(s, to_device(w), 10)
    kv = dec.kv_cache(10, 64)
    kv.values.copy_(kv_host.cuda())
    toks = [int(t) for t in synth.tokens(s.vocab, 10, seed=60)]
    buf = i32(toks)
    for t in range(3):
        poss = [n + t for n in lengths]
        refs = [m.step(caches[b], toks[b], poss[b]) for b in range(10)]
        dec.step(kv, buf, i32(poss), buf)
        assert dec.check() == 0
        got = buf.cpu().tolist()
        for b in range(10):
            assert_id(got[b], refs[b], f"self-feeding step {t} seq {b}")
        # keep teacher forcing so that a permitted near-tie cannot diverge the caches
        toks = [r.token for r in refs]
        buf.copy_(i32(toks))
    dec.close()


def test_batched_step_host():
    s = synth.TINY
    w = synth.model_weights(s, seed=61)
    lengths = synth.ragged_lengths(1, 40, 6, seed=62)
    kv_host, _ = synth.kv_prefill(s, 6, 48, lengths, seed=63)
    m = oracle.Model(oracle_shape(s), oracle_weights(w))
    dec = Decoder(s, to_device(w), 6)
    kv = dec.kv_cache(6, 48)
    kv.values.copy_(kv_host.cuda())
    toks = [int(t) for t in synth.tokens(s.vocab, 6, seed=64)]
    out_h = torch.zeros(6, dtype=torch.int32).pin_memory()
    log_h = torch.zeros((6, s.vocab), dtype=torch.float32).pin_memory()
    dec.step_host(kv, torch.tensor(toks, dtype=torch.int32),
                  torch.tensor(lengths, dtype=torch.int32), out_h, log_h)
    for b in range(6):
        r = m.step(oracle_cache(kv_host, None, b), toks[b], lengths[b])
        assert_close(log_h[b].numpy(), r.logits, f"step_host seq {b}")
        assert_id(int(out_h[b]), r, f"step_host seq {b}")
    dec.close()


# ------------------------------------------------------- full-size shapes
def _fill_batch(s, kv, lengths, seed, kind, sampled):
    """Fill the device cache: sampled sequences from their own CPU generator
    (host copies kept for the oracle), the others on the device."""
    host = {}
    g = torch.Generator(device="cuda").manual_seed(seed)
    for b, n in enumerate(lengths):
        if b in sampled:
            vals, sc = synth.kv_prefill_seq(s, kv.max_ctx, n, seed=seed * 1000 + b, kind=kind)
            if kind == "bf16":
                kv.values[:, :, b].copy_(vals.cuda())
            else:
                kv.codes[:, :, b].copy_(vals.cuda())
                kv.scales[:, :, b].copy_(sc.cuda())
            host[b] = (vals, sc)
        else:
            shp = (s.n_layers, 2, s.n_kv_heads, n, s.head_dim)
            z = torch.randn(shp, generator=g, device="cuda")
            if kind == "bf16":
                kv.values[:, :, b, :, :n].copy_(z.to(torch.bfloat16))
            else:
                kv.codes[:, :, b, :, :n].copy_((z * 32.0).to(torch.float8_e4m3fn).view(torch.uint8))
                kv.scales[:, :, b, :, :n].copy_(
                    0.02 + 0.02 * torch.rand(shp[:-1], generator=g, device="cuda"))
    return host


def _seq_cache(vals, sc):
    if sc is None:
        return oracle.Cache("bf16", np.ascontiguousarray(synth.bits16(vals)))
    return oracle.Cache("fp8", np.ascontiguousarray(vals.numpy()), np.ascontiguousarray(sc.numpy()))


def _full_size(s, w, wd, batch, lengths, max_ctx, kind, sampled, steps, seed, w8=False):
    """w8: an 8-bit handle (True or "int8": dec_quantize_int8 of wd; "fp8":
    dec_quantize_fp8w) against the oracle's model of the same codes."""
    ow = oracle_weights(w)
    wk = "int8" if w8 is True else w8
    if wk:
        m = oracle.Model(oracle_shape(s), oracle.quantize_weights_int8(ow) if wk == "int8"
                         else oracle.quantize_weights_fp8(ow))
        dec = Decoder(s, quantize_int8(wd, kind=wk), batch)
    else:
        m = oracle.Model(oracle_shape(s), ow)
        dec = Decoder(s, wd, batch)
    kv = dec.kv_cache(batch, max_ctx, kind)
    host = _fill_batch(s, kv, lengths, seed, kind, sampled)
    caches = {b: _seq_cache(*host[b]) for b in sampled}
    toks = [int(t) for t in synth.tokens(s.vocab, batch, seed=seed + 1)]
    for t in range(steps):
        poss = [n + t for n in lengths]
        ids, logits, hid = _gpu_step(dec, kv, toks, poss)
        for b in sampled:
            r = m.step(caches[b], toks[b], poss[b], want_hidden=True)
            tag = f"{kind} step {t} seq {b} p={poss[b]}"
            assert_close(logits[b], r.logits, tag + " logits")
            for l in (0, 1, s.n_layers // 2, s.n_layers - 1, s.n_layers):
                assert_close(hid[l, b], r.hidden[l], tag + f" hidden {l}")
            assert_id(int(ids[b]), r, tag)
            _check_kv_row(kv, caches[b], b, poss[b], tag)
            toks[b] = r.token
        # unsampled sequences feed themselves
        for b in range(batch):
            if b not in sampled:
                toks[b] = int(ids[b])
    del kv
    dec.close()


@pytest.fixture(scope="module")
def big06():
    s = synth.QWEN3_0_6B
    w = synth.model_weights(s, seed=2)
    return s, w, to_device(w)


def test_0p6b_bs64_ragged(big06):
    """0.6B shape, 64 sequences, contexts U[200, 420]: sampled sequences vs
    the oracle over two teacher-forced steps."""
    s, w, wd = big06
    lengths = synth.ragged_lengths(200, 420, 64, seed=70)
    sampled = sorted({0, 21, 42, 63, int(np.argmax(lengths)), int(np.argmin(lengths))})
    _full_size(s, w, wd, 64, lengths, 432, "bf16", sampled, steps=2, seed=71)


def test_0p6b_bs64_every_sequence_one_step(big06):
    """0.6B shape, 64 sequences, contexts U[200, 420]: every sequence of the
    batch against the oracle for one step."""
    s, w, wd = big06
    lengths = synth.ragged_lengths(200, 420, 64, seed=74)
    _full_size(s, w, wd, 64, lengths, 432, "bf16", list(range(64)), steps=1, seed=75)


@pytest.fixture(scope="module")
def big17():
    s = synth.QWEN3_1_7B
    w = synth.model_weights(s, seed=17)
    return s, w, to_device(w)


@pytest.mark.parametrize("kind", ["bf16", "fp8"])
def test_1p7b_bs64_long_context(big17, kind):
    """1.7B shape, 64 sequences with contexts U[2048, 4096], bf16 and E4M3
    caches; sampled sequences vs the oracle."""
    s, w, wd = big17
    lengths = synth.ragged_lengths(2048, 4080, 64, seed=72)
    sampled = sorted({5, int(np.argmax(lengths))})
    _full_size(s, w, wd, 64, lengths, 4096, kind, sampled, steps=1, seed=73)
