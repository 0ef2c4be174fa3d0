"""Pins of the oracle's building blocks against closed forms, invariants and
library routines (no test retypes the oracle's formula)."""
import math

import numpy as np
import pytest
import torch

import oracle


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def _val(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()


# ----------------------------------------------------------------- RMSNorm
def test_rmsnorm_constant_vector_closed_form():
    # x = c * 1: mean square c^2 -> y_i = c / sqrt(c^2 + eps) * g_i
    n, c, eps = 64, -3.0, 1e-6
    g = _bf16(np.linspace(0.5, 2.0, n))
    y = oracle.rmsnorm(np.full(n, c), g, eps)
    assert np.allclose(y, c / math.sqrt(c * c + eps) * _val(g), rtol=1e-14, atol=0)


def test_rmsnorm_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(1024)
    ones = _bf16(np.ones(1024))
    y = oracle.rmsnorm(x, ones, 1e-6)
    assert abs(math.sqrt(np.mean(y * y)) - 1.0) < 1e-6       # RMS = 1 - O(eps)
    y2 = oracle.rmsnorm(x * 37.5, ones, 1e-6)
    assert np.allclose(y, y2, rtol=1e-6)


def test_rmsnorm_gain_is_elementwise():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(128)
    g = _bf16(1.0 + 0.1 * rng.standard_normal(128))
    a = oracle.rmsnorm(x, g, 1e-6)
    b = oracle.rmsnorm(x, _bf16(np.ones(128)), 1e-6)
    assert np.allclose(a, b * _val(g), rtol=1e-14)


# -------------------------------------------------------------------- GEMV
def test_gemv_matches_numpy_matmul():
    rng = np.random.default_rng(2)
    W = _bf16(rng.standard_normal((96, 320)) * 0.02)
    x = rng.standard_normal(320)
    y = oracle.gemv(W, x)
    ref = _val(W) @ x
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_gemv_identity_and_transposed_operand_fails():
    eye = _bf16(np.eye(48))
    x = np.arange(48, dtype=np.float64)
    assert np.array_equal(oracle.gemv(eye, x), x)
    # a plausible mistake (x^T W instead of W x) would not reproduce W[2,:] . x
    rng = np.random.default_rng(3)
    W = _bf16(rng.standard_normal((8, 16)))
    xx = rng.standard_normal(16)
    assert math.isclose(oracle.gemv(W, xx)[2], float(_val(W)[2] @ xx), rel_tol=1e-12)


# -------------------------------------------------------------------- RoPE
def test_rope_position_zero_is_identity():
    rng = np.random.default_rng(4)
    x = rng.standard_normal(128)
    assert np.array_equal(oracle.rope(x, 0, 1e6), x)


def test_rope_preserves_norm():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(128)
    for p in (1, 17, 795, 4095, 32767):
        assert math.isclose(np.linalg.norm(oracle.rope(x, p, 1e6)), np.linalg.norm(x), rel_tol=1e-12)


def test_rope_two_dim_is_rotation_by_p_radians():
    # D = 2: one pair (x0, x1) with inv_freq = 1 -> rotation by angle p
    for p in (1, 2, 5, 100):
        y = oracle.rope(np.array([1.0, 0.0]), p, 1e6)
        assert np.allclose(y, [math.cos(p), math.sin(p)], atol=1e-12)


def test_rope_pairs_i_with_i_plus_half():
    # only element 0 set: after rotation only elements 0 and D/2 are non-zero
    x = np.zeros(64)
    x[0] = 1.0
    y = oracle.rope(x, 3, 1e6)
    nz = np.nonzero(np.abs(y) > 1e-15)[0].tolist()
    assert nz == [0, 32]
    # the highest-index pair turns slowest: inv_freq = theta^(-(D-2)/D)
    x = np.zeros(64)
    x[31] = 1.0
    y = oracle.rope(x, 3, 1e6)
    ang = np.float32(3.0) * np.float32(1.0 / 1e6 ** (62 / 64))
    assert np.allclose([y[31], y[63]], [math.cos(ang), math.sin(ang)], atol=1e-12)


def test_rope_relative_position_property():
    rng = np.random.default_rng(6)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    base = np.dot(oracle.rope(q, 7, 1e6), oracle.rope(k, 3, 1e6))
    for shift in (10, 200, 700):
        other = np.dot(oracle.rope(q, 7 + shift, 1e6), oracle.rope(k, 3 + shift, 1e6))
        assert math.isclose(base, other, rel_tol=1e-4, abs_tol=1e-4)


# --------------------------------------------------------------- attention
def test_attention_single_key_returns_v_exactly():
    rng = np.random.default_rng(7)
    q = rng.standard_normal(128)
    K = _bf16(rng.standard_normal((1, 128)))
    V = _bf16(rng.standard_normal((1, 128)))
    out = oracle.attend(q, K, V, 1)
    assert np.array_equal(out, _val(V)[0])


def test_attention_identical_keys_give_mean_of_v():
    rng = np.random.default_rng(8)
    q = rng.standard_normal(64)
    K = _bf16(np.tile(rng.standard_normal(64), (9, 1)))
    V = _bf16(rng.standard_normal((9, 64)))
    out, probs = oracle.attend(q, K, V, 9, want_probs=True)
    assert np.allclose(probs, 1 / 9, rtol=1e-14)
    assert np.allclose(out, _val(V).mean(axis=0), rtol=1e-12, atol=1e-14)


def test_attention_probabilities_sum_to_one_and_match_torch_softmax():
    rng = np.random.default_rng(9)
    q = rng.standard_normal(128) * 3
    K = _bf16(rng.standard_normal((300, 128)))
    V = _bf16(rng.standard_normal((300, 128)))
    out, probs = oracle.attend(q, K, V, 257, want_probs=True)
    assert math.isclose(probs.sum(), 1.0, rel_tol=1e-13)
    s = torch.from_numpy(_val(K)[:257] @ q / math.sqrt(128))
    ref_p = torch.softmax(s, dim=0).numpy()
    assert np.allclose(probs, ref_p, rtol=1e-12, atol=1e-15)
    assert np.allclose(out, ref_p @ _val(V)[:257], rtol=1e-11, atol=1e-13)


def test_attention_reads_only_the_first_n_rows():
    rng = np.random.default_rng(10)
    q = rng.standard_normal(64)
    K = _bf16(rng.standard_normal((20, 64)))
    V = _bf16(rng.standard_normal((20, 64)))
    a = oracle.attend(q, K, V, 5)
    K2, V2 = K.copy(), V.copy()
    K2[5:] = _bf16(rng.standard_normal((15, 64)))
    V2[5:] = _bf16(rng.standard_normal((15, 64)))
    assert np.array_equal(a, oracle.attend(q, K2, V2, 5))


def test_attention_fp8_reads_code_times_scale():
    rng = np.random.default_rng(11)
    q = rng.standard_normal(128)
    codes_k = rng.integers(0, 0x7E, (33, 128)).astype(np.uint8)
    codes_v = rng.integers(0x80, 0xFE, (33, 128)).astype(np.uint8)
    ks = rng.uniform(0.01, 0.03, 33).astype(np.float32)
    vs = rng.uniform(0.01, 0.03, 33).astype(np.float32)
    out = oracle.attend(q, codes_k, codes_v, 33, ks, vs)
    Kd = torch.from_numpy(codes_k).view(torch.float8_e4m3fn).double().numpy() * ks[:, None]
    Vd = torch.from_numpy(codes_v).view(torch.float8_e4m3fn).double().numpy() * vs[:, None]
    p = torch.softmax(torch.from_numpy(Kd @ q / math.sqrt(128)), 0).numpy()
    assert np.allclose(out, p @ Vd, rtol=1e-11, atol=1e-13)


# ------------------------------------------------------------ SwiGLU, argmax
def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    assert math.isclose(oracle.silu(1.0), 1 / (1 + math.exp(-1)), rel_tol=1e-15)
    assert math.isclose(oracle.silu(-2.0), -2 * torch.sigmoid(torch.tensor(-2.0, dtype=torch.float64)).item(), rel_tol=1e-14)
    assert math.isclose(oracle.silu(30.0), 30.0, rel_tol=1e-12)


def test_argmax_lowest_index_on_ties_and_margin():
    v = np.array([0.5, 2.0, -1.0, 2.0, 1.75])
    i, m = oracle.argmax(v)
    assert i == 1 and m == 0.0
    v = np.array([0.5, 2.0, -1.0, 1.0, 1.75])
    i, m = oracle.argmax(v)
    assert i == 1 and m == 0.25
    rng = np.random.default_rng(12)
    w = rng.standard_normal(151936)
    i, _ = oracle.argmax(w)
    assert i == int(np.argmax(w))
