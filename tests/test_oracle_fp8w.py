"""Pins of the oracle's E4M3 weight-only path (CPU, no GPU).

"Qwen3-ASR -- Latency & Bottleneck Analysis", 08 Optimization roadmap: an
fp8 lm_head; the same weight-only scheme for the projections.  The oracle's
reading quantises each weight row with the per-row E4M3 quantiser of the KV
rows (scale = max(amax, 2^-126)/448 in fp32, codes round to nearest even,
saturating).  Pinned by rows derived by hand from the OCP E4M3 definition,
by the round-to-nearest error bound, and by the special case of power-of-two
scales, where the E4M3 model must equal the bf16 model whose weights are the
dequantised values, bit for bit."""
import numpy as np
import pytest

import oracle
from conftest import oracle_cache, oracle_shape, oracle_weights
from decoder_greedy_decode_b200 import synth


def _bf16_bits(v):
    """bf16 bits of values that are exact in bf16 (asserted)."""
    f = np.asarray(v, dtype=np.float32)
    u = f.view(np.uint32)
    assert ((u & 0xFFFF) == 0).all()
    return (u >> 16).astype(np.uint16)


def _random_bf16(rows, cols, seed, std=0.02):
    rng = np.random.default_rng(seed)
    f = (rng.standard_normal((rows, cols)) * std).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _e4m3_values():
    """The 254 finite E4M3 values (every code but the two NaNs), from the
    format's definition: 1 sign, 4 exponent bits (bias 7), 3 fraction bits,
    subnormals M/8 * 2^-6."""
    vals = []
    for c in range(256):
        s, E, M = c >> 7, (c >> 3) & 15, c & 7
        if E == 15 and M == 7:
            continue
        v = (M / 8.0) * 2.0 ** -6 if E == 0 else (1 + M / 8.0) * 2.0 ** (E - 7)
        vals.append((c, -v if s else v))
    return vals


def test_hand_derived_rows():
    """Row [1, 2, -1, 0]: amax 2, scale fp32(2/448); 1/scale = 224 =
    1.75 * 2^7 -> E = 14, M = 6 -> 0x76; 2/scale = 448 = 1.75 * 2^8 -> 0x7E;
    -1 -> 0xF6; 0 -> 0.  Row [448, 0.5, 0.3125, 0.875 * 2^-6, 2^-10,
    3 * 2^-10]: scale 1; 448 -> 0x7E; 0.5 = 2^-1 -> E = 6, M = 0 -> 0x30;
    0.3125 = 1.25 * 2^-2 -> E = 5, M = 2 -> 0x2A; 0.875 * 2^-6 (subnormal,
    M = 7) -> 0x07; 2^-10 is half the subnormal quantum 2^-9 and rounds to
    even (0); 3 * 2^-10 is halfway between 1 and 2 quanta and rounds to even
    (code 2)."""
    W = np.stack([_bf16_bits([1.0, 2.0, -1.0, 0.0, 0.0, 0.0]),
                  _bf16_bits([448.0, 0.5, 0.3125, 0.875 * 2.0 ** -6, 2.0 ** -10,
                              3 * 2.0 ** -10])])
    codes, scales = oracle.fp8w_quantize_rows(W)
    assert codes.dtype == np.uint8 and scales.dtype == np.float32
    assert codes[0].tolist() == [0x76, 0x7E, 0xF6, 0, 0, 0]
    assert scales[0] == np.float32(2.0) / np.float32(448.0)
    assert codes[1].tolist() == [0x7E, 0x30, 0x2A, 0x07, 0x00, 0x02]
    assert scales[1] == 1.0


def test_properties_on_random_rows():
    """Every dequantised weight e4m3(code) * scale is within the
    round-to-nearest bound of the weight: half a unit in the last place of
    E4M3 (2^-4 relative) for normal codes, half the subnormal quantum
    (2^-10 * scale) below 2^-6 * scale; the row's largest magnitude maps to
    +-448 exactly; a zero row gives zero codes."""
    W = _random_bf16(29, 384, seed=6)
    W[2] = 0
    codes, scales = oracle.fp8w_quantize_rows(W)
    dec = oracle.e4m3_decode(codes) * scales[:, None].astype(np.float64)
    w = (W.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    bound = np.maximum(np.abs(w) * 2.0 ** -4, 2.0 ** -10 * scales[:, None]) * (1 + 1e-6)
    assert np.all(np.abs(dec - w) <= bound)
    amax_codes = codes[np.arange(29), np.argmax(np.abs(w), axis=1)]
    assert np.all((amax_codes[np.arange(29) != 2] & 0x7F) == 0x7E)
    assert np.all(codes[2] == 0)


def test_gemv_f8_with_power_of_two_scales_is_the_bf16_gemv():
    """With scales 2^k every dequantised weight e4m3(c) * 2^k is exact in
    bf16, so the E4M3 product must equal the (pinned) bf16 product bit for
    bit; a wrong row / column index, a transposed operand or a wrong code
    decode breaks it (17 x 40)."""
    rng = np.random.default_rng(12)
    vals = _e4m3_values()
    pick = rng.integers(0, len(vals), size=(17, 40))
    C = np.array([[vals[i][0] for i in row] for row in pick], dtype=np.uint8)
    V = np.array([[vals[i][1] for i in row] for row in pick], dtype=np.float64)
    k = rng.integers(-14, -6, size=17)
    s = np.ldexp(1.0, k).astype(np.float32)
    x = rng.standard_normal(40)
    Wb = _bf16_bits((V * s[:, None].astype(np.float64)).astype(np.float32))
    got = oracle.gemv_f8(C, s, x)
    assert np.array_equal(got, oracle.gemv(Wb, x))


def _pow2_fp8_model(s, seed):
    """An E4M3 model with random codes and power-of-two row scales, and the
    bf16 model of its dequantised weights."""
    rng = np.random.default_rng(seed)
    vals = _e4m3_values()
    codes_of = np.array([c for c, _ in vals], dtype=np.uint8)
    value_of = np.array([v for _, v in vals], dtype=np.float64)
    wb = oracle_weights(synth.model_weights(s, seed=seed))
    layers8, scales8, layersb = [], [], []

    def q(shape):
        pick = rng.integers(0, len(vals), size=shape)
        sc = np.ldexp(1.0, rng.integers(-14, -9, size=shape[0])).astype(np.float32)
        dq = (value_of[pick] * sc[:, None].astype(np.float64)).astype(np.float32)
        return codes_of[pick], sc, _bf16_bits(dq)

    for lw in wb.layers:
        l8, s8, lb = dict(lw), {}, dict(lw)
        for key in oracle.PROJ_KEYS:
            l8[key], s8[key], lb[key] = q(lw[key].shape)
        layers8.append(l8)
        scales8.append(s8)
        layersb.append(lb)
    lm8, lms, lmb = q(wb.lm_head.shape)
    w8 = oracle.Weights(embed=wb.embed, lm_head=lm8, final_norm=wb.final_norm, layers=layers8,
                        kind="fp8", lm_scale=lms, scales=scales8)
    wbf = oracle.Weights(embed=wb.embed, lm_head=lmb, final_norm=wb.final_norm, layers=layersb)
    return w8, wbf


def test_fp8_model_equals_bf16_model_of_its_dequantised_weights():
    s = synth.TINY
    w8, wbf = _pow2_fp8_model(s, seed=23)
    m8 = oracle.Model(oracle_shape(s), w8)
    mb = oracle.Model(oracle_shape(s), wbf)
    kv, _ = synth.kv_prefill(s, 1, 64, [20], seed=24)
    c8 = oracle_cache(kv, None, 0)
    cb = oracle_cache(kv, None, 0)
    for i, tok in enumerate([5, 77, 4000]):
        r8 = m8.step(c8, tok, 20 + i, want_hidden=True, want_new_kv=True)
        rb = mb.step(cb, tok, 20 + i, want_hidden=True, want_new_kv=True)
        assert np.array_equal(r8.logits, rb.logits)
        assert np.array_equal(r8.hidden, rb.hidden)
        assert r8.token == rb.token
    assert np.array_equal(c8.kv, cb.kv)


def test_quantize_weights_fp8_touches_only_the_projections():
    s = synth.TINY
    wb = oracle_weights(synth.model_weights(s, seed=32, gain_std=0.1))
    w8 = oracle.quantize_weights_fp8(wb)
    assert w8.kind == "fp8" and w8.lm_head.dtype == np.uint8
    assert np.array_equal(w8.embed, wb.embed) and np.array_equal(w8.final_norm, wb.final_norm)
    for l8, lb, sc in zip(w8.layers, wb.layers, w8.scales):
        for key in oracle.LAYER_KEYS:
            if key in oracle.PROJ_KEYS:
                c, sref = oracle.fp8w_quantize_rows(lb[key])
                assert l8[key].dtype == np.uint8 and np.array_equal(l8[key], c)
                assert np.array_equal(sc[key], sref)
            else:
                assert np.array_equal(l8[key], lb[key])
