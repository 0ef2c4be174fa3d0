"""Pins of the oracle's number formats (bf16 rounding, OCP FP8 E4M3).

The stored-cache formats decide what attention reads back ("the attention
math runs at full precision", Baseten Qwen3-ASR article, KV cache
quantization), so the oracle's encoders are checked against library routines
(torch's bf16 and float8_e4m3fn casts), the format's defining values and
exhaustive enumeration."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_bf16_decode_is_upper_half_of_binary32():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 16, 4000, dtype=np.uint32).astype(np.uint16)
    got = oracle.bf16_to_double(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))


def test_bf16_round_matches_torch_rne_on_float32_inputs():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(3000).astype(np.float32),
        (rng.standard_normal(1000) * 1e-38).astype(np.float32),   # subnormal range
        (rng.standard_normal(500) * 1e30).astype(np.float32),
    ])
    # exact ties: low 16 bits 0x8000 (tie) with even and odd kept bit
    tie = (rng.integers(0, 1 << 15, 200, dtype=np.uint32) << 16 | 0x8000).astype(np.uint32)
    x = np.concatenate([x, tie.view(np.float32)])
    got = oracle.bf16_round(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_round_overflow_and_specials():
    assert oracle.bf16_round([3.5e38])[0] == 0x7F80            # above bf16 max -> +inf
    assert oracle.bf16_round([-3.5e38])[0] == 0xFF80
    assert oracle.bf16_round([0.0])[0] == 0x0000
    assert oracle.bf16_round([1.0])[0] == 0x3F80
    # 1 + 2^-8 is the exact midpoint of 1 and 1 + 2^-7: ties to even -> 1.0
    assert oracle.bf16_round([1.0 + 2.0 ** -8])[0] == 0x3F80
    assert oracle.bf16_round([1.0 + 3 * 2.0 ** -8])[0] == 0x3F82


def test_e4m3_defining_values():
    g = json.load(open(os.path.join(GOLDEN, "e4m3_defining_values.json")))
    for code, val in g["codes"].items():
        got = oracle.e4m3_decode([int(code, 16)])[0]
        assert got == val and math.copysign(1, got) == math.copysign(1, val), code
    for code in g["nan_codes"]:
        assert np.isnan(oracle.e4m3_decode([int(code, 16)])[0])


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def test_e4m3_round_trip_of_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    back = oracle.e4m3_encode(vals)
    assert np.array_equal(back, codes)


def test_e4m3_encode_rne_matches_torch_in_range():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.standard_normal(4000) * 50, rng.standard_normal(1000) * 0.01])
    x = x[np.abs(x) < 448].astype(np.float32)
    # the midpoints between neighbouring codes: ties go to the even code
    codes = np.arange(0, 0x7E, dtype=np.uint8)
    v = oracle.e4m3_decode(codes)
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids])
    got = oracle.e4m3_encode(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_e4m3_encode_saturates():
    assert oracle.e4m3_encode([449.0])[0] == 0x7E
    assert oracle.e4m3_encode([1e9])[0] == 0x7E
    assert oracle.e4m3_encode([-1e9])[0] == 0xFE
    assert oracle.e4m3_encode([464.0])[0] == 0x7E   # midpoint 448/480 -> still 448
    assert oracle.e4m3_encode([2.0 ** -10])[0] == 0x00  # half the smallest subnormal: tie to even 0
    assert oracle.e4m3_encode([3 * 2.0 ** -10])[0] == 0x02


def test_e4m3_quantize_row_scale_and_bound():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(128).astype(np.float32)
    codes, scale = oracle.e4m3_quantize_row(x)
    amax = np.abs(x).max()
    assert scale == np.float32(amax) / np.float32(448.0)
    deq = oracle.e4m3_decode(codes) * scale
    # |x| <= 448*scale, and RNE error at most half a code step: <= 2^-4 relative for normals
    assert np.all(np.abs(deq - x) <= np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * scale) + 1e-12)
    # the largest element maps to the largest code
    i = int(np.argmax(np.abs(x)))
    assert codes[i] & 0x7F == 0x7E


def test_e4m3_quantize_row_all_zero_uses_floor_scale():
    codes, scale = oracle.e4m3_quantize_row(np.zeros(64, dtype=np.float32))
    assert scale == np.float32(2.0 ** -126) / np.float32(448.0)
    assert not codes.any()
