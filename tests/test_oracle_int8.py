"""Pins of the oracle's int8 weight-only path (CPU, no GPU).

faster-qwen-asr GB10 benchmark record, "cuda_graph_int8" entries: int8
weight-only quantisation of the text decoder's projections and lm_head.  The
oracle's reading (per output row, scale = amax/127, round half to even in
fp32) is pinned by hand-derived rows (tests/golden/int8_rows.json), by the
round-to-nearest error bound, by brute force over all codes, and by the
special case of power-of-two scales, where the int8 model must equal the bf16
model whose weights are the dequantised values, bit for bit."""
import json
import os

import numpy as np
import pytest

import oracle
from conftest import oracle_shape, oracle_weights
from decoder_greedy_decode_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "int8_rows.json")


def _bf16_bits(v):
    """bf16 bits of values that are exact in bf16 (asserted)."""
    f = np.asarray(v, dtype=np.float32)
    u = f.view(np.uint32)
    assert ((u & 0xFFFF) == 0).all()
    return (u >> 16).astype(np.uint16)


def _bf16_value(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def test_golden_rows():
    g = json.load(open(GOLDEN))
    W = np.stack([_bf16_bits(r["w"]) for r in g["rows"]])
    codes, scales = oracle.int8_quantize_rows(W)
    assert codes.dtype == np.int8 and scales.dtype == np.float32
    for i, r in enumerate(g["rows"]):
        assert codes[i].tolist() == r["codes"], r["note"]
        assert float(scales[i]) == r["scale"], r["note"]
    # rows are quantised independently: the same rows one at a time
    for i in range(W.shape[0]):
        c1, s1 = oracle.int8_quantize_rows(W[i:i + 1])
        assert np.array_equal(c1[0], codes[i]) and s1[0] == scales[i]


def _random_bf16(rows, cols, seed, std=0.02):
    rng = np.random.default_rng(seed)
    f = (rng.standard_normal((rows, cols)) * std).astype(np.float32)
    # round to nearest even bf16
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def test_properties_on_random_rows():
    W = _random_bf16(37, 512, seed=5)
    W[3] = 0                      # a zero row
    W[7, :] = _bf16_bits(np.full(512, -0.5, np.float32))  # constant negative row
    codes, scales = oracle.int8_quantize_rows(W)
    w = _bf16_value(W).astype(np.float64)
    assert codes.min() >= -127 and codes.max() <= 127
    for r in range(W.shape[0]):
        a = np.abs(w[r])
        if a.max() == 0:
            assert scales[r] == 0 and not codes[r].any()
            continue
        j = int(np.argmax(a))
        assert abs(int(codes[r, j])) == 127 and np.sign(codes[r, j]) == np.sign(w[r, j])
        # round to nearest: within half a step (plus the fp32 division's rounding)
        err = np.abs(w[r] / float(scales[r]) - codes[r].astype(np.float64))
        assert err.max() <= 0.5 + 1e-5
        # the scale times 127 is the row's amax (one fp32 rounding)
        assert abs(float(scales[r]) * 127.0 - a.max()) <= a.max() * 2.0 ** -23
    assert np.all(codes[7] == -127)


def test_brute_force_nearest_code():
    """Each code is the integer in [-127, 127] nearest to fp32(w)/scale, ties
    to the even one, found by trying all 255 codes."""
    W = _random_bf16(6, 64, seed=9, std=1.0)
    codes, scales = oracle.int8_quantize_rows(W)
    w = _bf16_value(W)
    cand = np.arange(-127, 128, dtype=np.float64)
    for r in range(W.shape[0]):
        for j in range(W.shape[1]):
            q = float(np.float32(w[r, j]) / np.float32(scales[r]))   # the fp32 decision
            d = np.abs(q - cand)
            best = cand[d == d.min()]
            want = best[0] if best.size == 1 else best[best % 2 == 0][0]
            assert codes[r, j] == int(want), (r, j, q)


def test_gemv_i8_with_power_of_two_scales_is_the_bf16_gemv():
    """With scales 2^k every dequantised weight c * 2^k is exact in bf16, so
    the int8 product must equal the (pinned) bf16 product bit for bit; a
    wrong row / column index or a transposed operand breaks it (19 x 48)."""
    rng = np.random.default_rng(11)
    C = rng.integers(-127, 128, size=(19, 48)).astype(np.int8)
    k = rng.integers(-12, -4, size=19)
    s = np.ldexp(1.0, k).astype(np.float32)
    x = rng.standard_normal(48)
    Wb = _bf16_bits(C.astype(np.float32) * s[:, None])
    got = oracle.gemv_i8(C, s, x)
    assert np.array_equal(got, oracle.gemv(Wb, x))
    # doubling one row's scale doubles only that row
    s2 = s.copy()
    s2[4] *= 2
    got2 = oracle.gemv_i8(C, s2, x)
    assert got2[4] == 2 * got[4] and np.array_equal(np.delete(got2, 4), np.delete(got, 4))


def _pow2_int8_model(s, seed):
    """An int8 model with random codes and power-of-two row scales (each
    matrix and row its own exponent) and the bf16 model of its dequantised
    weights."""
    rng = np.random.default_rng(seed)
    wb = oracle_weights(synth.model_weights(s, seed=seed))
    layers8, scales8, layersb = [], [], []

    def q(shape):
        C = rng.integers(-127, 128, size=shape).astype(np.int8)
        sc = np.ldexp(1.0, rng.integers(-13, -8, size=shape[0])).astype(np.float32)
        return C, sc, _bf16_bits(C.astype(np.float32) * sc[:, None])

    for lw in wb.layers:
        l8, s8, lb = dict(lw), {}, dict(lw)
        for key in oracle.PROJ_KEYS:
            l8[key], s8[key], lb[key] = q(lw[key].shape)
        layers8.append(l8)
        scales8.append(s8)
        layersb.append(lb)
    lm8, lms, lmb = q(wb.lm_head.shape)
    w8 = oracle.Weights(embed=wb.embed, lm_head=lm8, final_norm=wb.final_norm, layers=layers8,
                        kind="int8", lm_scale=lms, scales=scales8)
    wbf = oracle.Weights(embed=wb.embed, lm_head=lmb, final_norm=wb.final_norm, layers=layersb)
    return w8, wbf


@pytest.mark.parametrize("kind", ["bf16", "fp8"])
def test_int8_model_equals_bf16_model_of_its_dequantised_weights(kind):
    s = synth.TINY
    w8, wbf = _pow2_int8_model(s, seed=21)
    m8 = oracle.Model(oracle_shape(s), w8)
    mb = oracle.Model(oracle_shape(s), wbf)
    kv, sc = synth.kv_prefill(s, 1, 64, [20], seed=22, kind=kind)
    from conftest import oracle_cache
    c8 = oracle_cache(kv, sc if kind == "fp8" else None, 0)
    cb = oracle_cache(kv, sc if kind == "fp8" else None, 0)
    for i, tok in enumerate([5, 77, 4000]):
        r8 = m8.step(c8, tok, 20 + i, want_hidden=True, want_new_kv=True)
        rb = mb.step(cb, tok, 20 + i, want_hidden=True, want_new_kv=True)
        assert np.array_equal(r8.logits, rb.logits)
        assert np.array_equal(r8.hidden, rb.hidden)
        assert np.array_equal(r8.new_k, rb.new_k) and np.array_equal(r8.new_v, rb.new_v)
        assert r8.token == rb.token
    assert np.array_equal(c8.kv, cb.kv)


def test_quantize_weights_int8_touches_only_the_projections():
    s = synth.TINY
    wb = oracle_weights(synth.model_weights(s, seed=31, gain_std=0.1))
    w8 = oracle.quantize_weights_int8(wb)
    assert w8.kind == "int8" and w8.lm_head.dtype == np.int8
    assert np.array_equal(w8.embed, wb.embed) and np.array_equal(w8.final_norm, wb.final_norm)
    for l8, lb, sc in zip(w8.layers, wb.layers, w8.scales):
        for key in oracle.LAYER_KEYS:
            if key in oracle.PROJ_KEYS:
                c, sref = oracle.int8_quantize_rows(lb[key])
                assert l8[key].dtype == np.int8 and np.array_equal(l8[key], c)
                assert np.array_equal(sc[key], sref)
            else:
                assert np.array_equal(l8[key], lb[key])
