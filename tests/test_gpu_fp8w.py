"""Weight-only E4M3 decoding on the GPU (dec_quantize_fp8w, dec_init_fp8w)
against the CPU oracle.

"Qwen3-ASR -- Latency & Bottleneck Analysis", 08 Optimization roadmap: an
fp8 lm_head (and the same weight-only scheme for the projections).  The
oracle quantises the same bf16 weights with its own routine;
dec_quantize_fp8w's codes and scales must equal them bit for bit (both take
the rounding decision in fp32), and steps of an E4M3 handle must match the
oracle's E4M3 model within the step tolerances: on the persistent kernel
(batch 1-4) and on the batched step (batch 5-64)."""
import numpy as np
import pytest
import torch

import oracle
from conftest import oracle_cache, oracle_shape, oracle_weights
from decoder_greedy_decode_b200 import capi, synth
from decoder_greedy_decode_b200.decoder import Decoder, quantize_fp8w, to_device
from gpu_util import NEAR_TIE, assert_close, assert_id, i32
from test_gpu_step import _check_kv_row, _check_only_rows_changed

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    capi.lib()


def _bf16_bits(f32):
    u = np.asarray(f32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def test_quantizer_bit_exact_vs_oracle():
    """1003 rows of 264 columns: normal rows, a zero row, rows of tiny values
    (subnormal fp32 scales), huge values, and rows whose quotients land on
    E4M3 rounding ties."""
    rng = np.random.default_rng(8)
    f = (rng.standard_normal((1003, 264)) * 0.02).astype(np.float32)
    f[0] = 0.0
    f[1] *= 2.0 ** -110
    f[2] *= 2.0 ** 100
    f[3, :] = 448.0
    f[3, 1:] = ((np.arange(263) % 32) + 0.5) * 2.0 ** -6  # w / scale on ties of the grid
    W = _bf16_bits(f)
    wt = torch.from_numpy(W.astype(np.int16)).view(torch.bfloat16).cuda()
    codes = torch.full((1003, 264), 0x55, dtype=torch.uint8, device="cuda")
    scales = torch.full((1003,), -1.0, dtype=torch.float32, device="cuda")
    capi.dec_quantize_fp8w(wt, 1003, 264, codes, scales)
    torch.cuda.synchronize()
    ref_c, ref_s = oracle.fp8w_quantize_rows(W)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
    got = codes.cpu().numpy()
    bad = np.argwhere(got != ref_c)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[0].tolist()}"


def _setup(s, seed, batch, max_ctx, lengths, kind="bf16", gain_std=0.0, max_batch=None):
    w = synth.model_weights(s, seed=seed, gain_std=gain_std)
    kv_host, sc_host = synth.kv_prefill(s, batch, max_ctx, lengths, seed=seed + 100, kind=kind)
    m = oracle.Model(oracle_shape(s), oracle.quantize_weights_fp8(oracle_weights(w)))
    caches = [oracle_cache(kv_host, sc_host, b) for b in range(batch)]
    dec = Decoder(s, quantize_fp8w(to_device(w)), max_batch=max_batch or batch)
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


@pytest.mark.parametrize("batch,kind,gain_std", [(1, "bf16", 0.0), (3, "fp8", 0.1),
                                                 (8, "bf16", 0.1), (64, "fp8", 0.0)])
def test_tiny_fp8w_teacher_forced(batch, kind, gain_std):
    """Batches of 1 and 3 run on the persistent kernel, 8 and 64 on the
    batched step (E4M3 codes widened to bf16 operand tiles)."""
    s = synth.TINY
    lengths = [17, 1, 40][:batch] if batch <= 3 else [(11 * b + 3) % 76 for b in range(batch)]
    m, caches, dec, kv = _setup(s, 500 + batch, batch, 80, lengths, kind, gain_std)
    toks = [int(t) for t in synth.tokens(s.vocab, batch, seed=600 + batch)]
    for t in range(3):
        poss = [lengths[b] + t for b in range(batch)]
        refs = [m.step(caches[b], toks[b], poss[b], want_hidden=True) for b in range(batch)]
        before = kv.buf.clone()
        ids, logits, hid = _step(dec, kv, toks, poss)
        for b in range(batch):
            tag = f"fp8w step {t} seq {b} p={poss[b]}"
            assert_close(logits[b], refs[b].logits, tag + " logits")
            for l in range(s.n_layers + 1):
                assert_close(hid[l, b], refs[b].hidden[l], tag + f" hidden {l}")
            assert_id(int(ids[b]), refs[b], tag)
            _check_kv_row(kv, caches[b], b, poss[b], tag)
        _check_only_rows_changed(before, kv, poss)
        toks = [r.token for r in refs]
    dec.close()


def test_fp8w_verify_block_on_the_persistent_kernel():
    """A block of 4 tokens on an E4M3 handle of max_batch 4 equals 4
    teacher-forced single steps of the oracle's E4M3 model."""
    s = synth.TINY
    n0, k = 30, 4
    m, caches, dec, kv = _setup(s, 520, 1, 64, [n0], max_batch=4)
    toks = [int(t) for t in synth.tokens(s.vocab, k, seed=521)]
    out = torch.full((k,), -7, dtype=torch.int32, device="cuda")
    logits = torch.empty((k, s.vocab), dtype=torch.float32, device="cuda")
    dec.verify(kv, i32(toks), i32(range(n0, n0 + k)), 0, out, logits)
    assert dec.check() == 0
    ids, lg = out.cpu().tolist(), logits.cpu().numpy()
    for i in range(k):
        r = m.step(caches[0], toks[i], n0 + i)
        assert_close(lg[i], r.logits, f"fp8w verify row {i} logits")
        assert_id(ids[i], r, f"fp8w verify row {i}")
        _check_kv_row(kv, caches[0], 0, n0 + i, f"fp8w verify row {i}")
    dec.close()


def test_0p6b_fp8w_bs1_ctx795():
    """The 0.6B shape with E4M3 weights, batch 1, 795 prefilled rows: the
    codes of sampled projections equal the oracle's, and 16 teacher-forced
    steps from position 795 match the oracle's E4M3 model."""
    s = synth.QWEN3_0_6B
    w = synth.model_weights(s, seed=2)
    m = oracle.Model(oracle_shape(s), oracle.quantize_weights_fp8(oracle_weights(w)))
    wd = to_device(w)
    w8 = quantize_fp8w(wd)
    torch.cuda.synchronize()
    for l in (0, 27):
        for key in ("k", "gate"):
            assert np.array_equal(w8["layers"][l][key].cpu().numpy(), m.w.layers[l][key]), (l, key)
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
    for t in range(16):
        p = n0 + t
        r = m.step(cache, tok, p, want_hidden=True)
        ids, logits, hid = _step(dec, kv, [tok], [p])
        tag = f"0.6B fp8w p={p}"
        assert_close(logits[0], r.logits, tag + " logits")
        for l in range(s.n_layers + 1):
            assert_close(hid[l, 0], r.hidden[l], tag + f" hidden {l}")
        assert_id(int(ids[0]), r, tag)
        _check_kv_row(kv, cache, 0, p, tag)
        tok = r.token
    dec.close()


def test_0p6b_fp8w_bs64_every_sequence_one_step():
    """The 0.6B shape with E4M3 weights, 64 sequences, contexts U[200, 420]
    (the batched step): every sequence against the oracle's E4M3 model."""
    from test_gpu_batched import _full_size
    s = synth.QWEN3_0_6B
    w = synth.model_weights(s, seed=2)
    wd = to_device(w)
    lengths = synth.ragged_lengths(200, 420, 64, seed=78)
    _full_size(s, w, wd, 64, lengths, 432, "bf16", list(range(64)), steps=1, seed=79, w8="fp8")


@pytest.mark.parametrize("batch,max_batch", [(2, 2), (6, 8)])
def test_fp8w_generate_equals_steps(batch, max_batch):
    """dec_generate on an E4M3-weight handle (batch 2 on the persistent
    kernel, batch 6 on the batched step) equals step-by-step decoding bit for
    bit, and its ids are the oracle's E4M3 model's greedy ids (up to a
    permitted near-tie)."""
    s = synth.TINY
    n0s = [12 + 8 * b for b in range(batch)]
    m, caches, dec, kv = _setup(s, 540 + batch, batch, 64, n0s, max_batch=max_batch)
    kv2 = dec.kv_cache(batch, 64)
    kv2.buf.copy_(kv.buf)
    toks = [int(t) for t in synth.tokens(s.vocab, batch, seed=541 + batch)]
    n = 6
    out = torch.empty((n, batch), dtype=torch.int32, device="cuda")
    pos = i32(n0s)
    dec.generate(kv, i32(toks), pos, out)
    assert dec.check() == 0
    ref, tok, p = [], i32(toks), list(n0s)
    for _ in range(n):
        o = torch.empty(batch, dtype=torch.int32, device="cuda")
        dec.step(kv2, tok, i32(p), o)
        ref.append(o.cpu().tolist())
        tok, p = o, [x + 1 for x in p]
    assert out.cpu().tolist() == ref and pos.cpu().tolist() == p
    assert torch.equal(kv.buf, kv2.buf)
    for b in range(batch):
        t = toks[b]
        for i in range(n):
            r = m.step(caches[b], t, n0s[b] + i)
            if ref[i][b] != r.token:
                assert r.margin < NEAR_TIE, f"seq {b} step {i}"
                break
            t = r.token
    dec.close()
