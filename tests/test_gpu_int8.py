"""Weight-only int8 decoding on the GPU (dec_quantize_int8, dec_init_int8)
against the CPU oracle.

faster-qwen-asr GB10 benchmark record, "cuda_graph_int8" entries: int8
weight-only quantisation of the text decoder and lm_head.  The oracle
quantises the same bf16 weights with its own routine; dec_quantize_int8's
codes and scales must equal them bit for bit (the rounding decision is taken
in fp32 on both sides), and a step of an int8 handle must match the oracle's
int8 model within the step tolerances."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from conftest import oracle_cache, oracle_shape, oracle_weights
from decoder_greedy_decode_b200 import capi, synth
from decoder_greedy_decode_b200.decoder import Decoder, quantize_int8, to_device
from gpu_util import assert_close, assert_id, i32
from test_gpu_step import _check_kv_row, _check_only_rows_changed

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "int8_rows.json")


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    capi.lib()


def _quantize_gpu(bits):
    """bf16 bits (numpy uint16 [rows, cols]) -> dec_quantize_int8 codes, scales."""
    w = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).cuda()
    rows, cols = bits.shape
    codes = torch.full((rows, cols), 99, dtype=torch.int8, device="cuda")
    scales = torch.full((rows,), -1.0, dtype=torch.float32, device="cuda")
    capi.dec_quantize_int8(w, rows, cols, codes, scales)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


def _bf16_bits(f32):
    u = np.asarray(f32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def test_quantizer_golden_rows():
    g = json.load(open(GOLDEN))
    W = np.stack([_bf16_bits(r["w"]) for r in g["rows"]])
    codes, scales = _quantize_gpu(W)
    for i, r in enumerate(g["rows"]):
        assert codes[i].tolist() == r["codes"], r["note"]
        assert float(scales[i]) == r["scale"], r["note"]


def test_quantizer_bit_exact_vs_oracle():
    """1003 rows (a ragged last block of warps) of 264 columns (not a multiple
    of 256): normal rows, a zero row, rows of tiny values (subnormal fp32
    scales), huge values and ties."""
    rng = np.random.default_rng(7)
    f = (rng.standard_normal((1003, 264)) * 0.02).astype(np.float32)
    f[0] = 0.0
    f[1] *= 2.0 ** -110          # scale = amax / 127 below 2^-126
    f[2] *= 2.0 ** 100
    f[3, :] = ((np.arange(264) % 200) - 100 + 0.5) * 0.5  # w / scale = k + 1/2: ties
    f[3, 0] = 63.5                                          # scale 0.5 exactly
    W = _bf16_bits(f)
    codes, scales = _quantize_gpu(W)
    ref_c, ref_s = oracle.int8_quantize_rows(W)
    assert np.array_equal(scales.view(np.uint32), ref_s.view(np.uint32))
    bad = np.argwhere(codes != ref_c)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[0].tolist()}"


def test_quantizer_rejects_bad_arguments():
    w = torch.zeros((4, 20), dtype=torch.bfloat16, device="cuda")
    codes = torch.zeros((4, 20), dtype=torch.int8, device="cuda")
    scales = torch.zeros(4, dtype=torch.float32, device="cuda")
    with pytest.raises(capi.DecError):
        capi.dec_quantize_int8(w, 4, 20, codes, scales)            # cols % 8
    w2 = torch.zeros(4 * 16 + 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(capi.DecError):
        capi.dec_quantize_int8(w2.data_ptr() + 2, 4, 16, codes, scales)  # misaligned


def _setup_int8(s, seed, batch, max_ctx, lengths, kind="bf16", gain_std=0.0, max_batch=None):
    w = synth.model_weights(s, seed=seed, gain_std=gain_std)
    kv_host, sc_host = synth.kv_prefill(s, batch, max_ctx, lengths, seed=seed + 100, kind=kind)
    m = oracle.Model(oracle_shape(s), oracle.quantize_weights_int8(oracle_weights(w)))
    caches = [oracle_cache(kv_host, sc_host, b) for b in range(batch)]
    dec = Decoder(s, quantize_int8(to_device(w)), max_batch=max_batch or batch)
    kv = dec.kv_cache(batch, max_ctx, kind)
    if kind == "bf16":
        kv.values.copy_(kv_host.cuda())
    else:
        kv.codes.copy_(kv_host.cuda())
        kv.scales.copy_(sc_host.cuda())
    return m, caches, dec, kv


def _step(dec, kv, toks, poss):
    s = dec.shape
    B = len(toks)
    out = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    logits = torch.empty((B, s.vocab), dtype=torch.float32, device="cuda")
    hid = torch.empty((s.n_layers + 1, B, s.hidden), dtype=torch.float32, device="cuda")
    dec.step_debug(kv, i32(toks), i32(poss), out, logits, hid)
    st = dec.check()
    assert st == 0, capi.error_string(st)
    return out.cpu().numpy(), logits.cpu().numpy(), hid.cpu().numpy()


@pytest.mark.parametrize("batch,kind,gain_std", [(1, "bf16", 0.0), (2, "fp8", 0.1),
                                                 (3, "bf16", 0.1), (4, "bf16", 0.0),
                                                 (5, "bf16", 0.1), (16, "fp8", 0.0),
                                                 (64, "bf16", 0.0)])
def test_tiny_int8_teacher_forced(batch, kind, gain_std):
    """Batches of 1-4 run on the persistent kernel, 5-64 on the batched
    step (int8 codes widened to bf16 operand tiles, row scales in the
    epilogue)."""
    s = synth.TINY
    lengths = [17, 1, 40, 63][:batch] if batch <= 4 else \
        [(13 * b + 5) % 76 for b in range(batch)]
    m, caches, dec, kv = _setup_int8(s, 300 + batch, batch, 80, lengths, kind, gain_std)
    toks = [int(t) for t in synth.tokens(s.vocab, batch, seed=400 + batch)]
    for t in range(4):
        poss = [lengths[b] + t for b in range(batch)]
        refs = [m.step(caches[b], toks[b], poss[b], want_hidden=True) for b in range(batch)]
        before = kv.buf.clone()
        ids, logits, hid = _step(dec, kv, toks, poss)
        for b in range(batch):
            tag = f"int8 step {t} seq {b} p={poss[b]}"
            assert_close(logits[b], refs[b].logits, tag + " logits")
            for l in range(s.n_layers + 1):
                assert_close(hid[l, b], refs[b].hidden[l], tag + f" hidden {l}")
            assert_id(int(ids[b]), refs[b], tag)
            _check_kv_row(kv, caches[b], b, poss[b], tag)
        _check_only_rows_changed(before, kv, poss)
        toks = [r.token for r in refs]
    dec.close()


def test_int8_handle_limits():
    s = synth.TINY
    w8 = quantize_int8(to_device(synth.model_weights(s, seed=310)))
    with pytest.raises(capi.DecError):
        Decoder(s, w8, max_batch=65)         # the batched step takes up to 64
    dec = Decoder(s, w8, max_batch=4)
    kv = dec.kv_cache(1, 32)
    out = torch.zeros(5, dtype=torch.int32, device="cuda")
    with pytest.raises(RuntimeError):       # blocks of 5 and more need the batched step
        dec.verify(kv, i32([1, 2, 3, 4, 5]), i32([3, 4, 5, 6, 7]), 0, out)
    dec.close()


def test_int8_verify_block_equals_single_steps():
    """A block of 4 tokens verified on an int8 handle (persistent kernel)
    equals 4 teacher-forced single steps of the oracle's int8 model."""
    s = synth.TINY
    n0, k = 30, 4
    m, caches, dec, kv = _setup_int8(s, 320, 1, 64, [n0], "bf16", 0.0, max_batch=4)
    toks = [int(t) for t in synth.tokens(s.vocab, k, seed=321)]
    out = torch.full((k,), -7, dtype=torch.int32, device="cuda")
    logits = torch.empty((k, s.vocab), dtype=torch.float32, device="cuda")
    dec.verify(kv, i32(toks), i32(range(n0, n0 + k)), 0, out, logits)
    assert dec.check() == 0
    ids, lg = out.cpu().tolist(), logits.cpu().numpy()
    for i in range(k):
        r = m.step(caches[0], toks[i], n0 + i)
        assert_close(lg[i], r.logits, f"int8 verify row {i} logits")
        assert_id(ids[i], r, f"int8 verify row {i}")
        _check_kv_row(kv, caches[0], 0, n0 + i, f"int8 verify row {i}")
    dec.close()


def test_int8_verify_block_on_the_batched_step():
    """A block of 9 tokens on an int8 handle of max_batch 16 (the batched
    step) equals 9 teacher-forced single steps of the oracle's int8 model."""
    s = synth.TINY
    n0, k = 30, 9
    m, caches, dec, kv = _setup_int8(s, 322, 1, 64, [n0], "bf16", 0.0, max_batch=16)
    toks = [int(t) for t in synth.tokens(s.vocab, k, seed=323)]
    out = torch.full((k,), -7, dtype=torch.int32, device="cuda")
    logits = torch.empty((k, s.vocab), dtype=torch.float32, device="cuda")
    dec.verify(kv, i32(toks), i32(range(n0, n0 + k)), 0, out, logits)
    assert dec.check() == 0
    ids, lg = out.cpu().tolist(), logits.cpu().numpy()
    for i in range(k):
        r = m.step(caches[0], toks[i], n0 + i)
        assert_close(lg[i], r.logits, f"int8 batched verify row {i} logits")
        assert_id(ids[i], r, f"int8 batched verify row {i}")
        _check_kv_row(kv, caches[0], 0, n0 + i, f"int8 batched verify row {i}")
    dec.close()


def test_int8_generate_equals_steps():
    """dec_generate on an int8 handle equals step-by-step decoding."""
    s = synth.TINY
    m, caches, dec, kv = _setup_int8(s, 320, 2, 64, [10, 30])
    kv2 = dec.kv_cache(2, 64)
    kv2.buf.copy_(kv.buf)
    toks = [int(t) for t in synth.tokens(s.vocab, 2, seed=321)]
    n = 6
    out = torch.empty((n, 2), dtype=torch.int32, device="cuda")
    pos = i32([10, 30])
    dec.generate(kv, i32(toks), pos, out)
    assert dec.check() == 0
    ref, tok, p = [], i32(toks), [10, 30]
    for _ in range(n):
        o = torch.empty(2, dtype=torch.int32, device="cuda")
        dec.step(kv2, tok, i32(p), o)
        ref.append(o.cpu().tolist())
        tok, p = o, [x + 1 for x in p]
    assert out.cpu().tolist() == ref and pos.cpu().tolist() == p
    assert torch.equal(kv.buf, kv2.buf)
    dec.close()


@pytest.fixture(scope="module")
def big06_int8():
    s = synth.QWEN3_0_6B
    w = synth.model_weights(s, seed=2)
    m = oracle.Model(oracle_shape(s), oracle.quantize_weights_int8(oracle_weights(w)))
    return s, w, m


def test_0p6b_int8_bs1_ctx795(big06_int8):
    """The 0.6B shape with int8 weights, batch 1, 795 prefilled rows: the
    codes of every projection equal the oracle's, and the 130 teacher-forced
    steps of the window match the oracle's int8 model."""
    s, w, m = big06_int8
    wd = to_device(w)
    w8 = quantize_int8(wd)
    torch.cuda.synchronize()
    for l in (0, 27):
        for key in ("q", "down"):
            c = w8["layers"][l][key].cpu().numpy()
            assert np.array_equal(c, m.w.layers[l][key]), (l, key)
            assert np.array_equal(w8["scales"][l][key].cpu().numpy(), m.w.scales[l][key])
    assert np.array_equal(w8["lm_head"].cpu().numpy(), m.w.lm_head)
    del wd
    dec = Decoder(s, w8, 1)
    n0 = 795
    kv_host, _ = synth.kv_prefill(s, 1, 928, [n0], seed=3)
    cache = oracle_cache(kv_host, None, 0)
    kv = dec.kv_cache(1, 928)
    kv.values.copy_(kv_host.cuda())
    tok = int(synth.tokens(s.vocab, 1, seed=4)[0])
    # the whole 130-token window (positions 795 .. 924), teacher-forced
    for t in range(130):
        p = n0 + t
        r = m.step(cache, tok, p, want_hidden=True)
        ids, logits, hid = _step(dec, kv, [tok], [p])
        tag = f"0.6B int8 p={p}"
        assert_close(logits[0], r.logits, tag + " logits")
        for l in range(s.n_layers + 1):
            assert_close(hid[l, 0], r.hidden[l], tag + f" hidden {l}")
        assert_id(int(ids[0]), r, tag)
        _check_kv_row(kv, cache, 0, p, tag)
        tok = r.token
    dec.close()


def test_0p6b_int8_bs64_every_sequence_one_step():
    """The 0.6B shape with int8 weights, 64 sequences, contexts U[200, 420]
    (the batched step): every sequence of the batch against the oracle's
    int8 model for one step."""
    from test_gpu_batched import _full_size
    s = synth.QWEN3_0_6B
    w = synth.model_weights(s, seed=2)
    wd = to_device(w)
    lengths = synth.ragged_lengths(200, 420, 64, seed=76)
    _full_size(s, w, wd, 64, lengths, 432, "bf16", list(range(64)), steps=1, seed=77, w8=True)
