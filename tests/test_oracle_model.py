"""Whole-step pins of the oracle: brute-force full causal recompute.

The oracle decodes one token at a time against its KV cache.  Here the same
token sequence is pushed through the whole decoder at once in matrix form,
without a cache: all positions' q/k/v, an explicit repeat_kv
(np.repeat over KV heads), a causal mask and a row softmax.  Matching
logits at every position pins the cache append, the positions, the mask,
the GQA grouping and the layer order together ("Qwen3-ASR -- Latency &
Bottleneck Analysis", 07 Root causes lists the per-layer ops; "Can CTC make
Qwen3-ASR faster?", 03 Speculative decoding: a causal target pass over known
positions gives the same logits as one-token steps)."""
import math

import numpy as np
import pytest
import torch

import oracle
from decoder_greedy_decode_b200 import synth
from conftest import oracle_cache, oracle_shape, oracle_weights


def _f(t):
    return t.double().numpy()


def _rms_rows(X, g, eps):
    return X / np.sqrt(np.mean(X * X, axis=-1, keepdims=True) + eps) * g


def _rope_rows(X, pos, theta):
    """X [T, heads, D]; rotate-half with fp32 inverse frequencies and angles."""
    D = X.shape[-1]
    inv = (1.0 / theta ** (np.arange(0, D, 2, dtype=np.float64) / D)).astype(np.float32)
    ang = (pos.astype(np.float32)[:, None] * inv[None, :]).astype(np.float64)   # [T, D/2]
    cos = np.concatenate([np.cos(ang), np.cos(ang)], -1)[:, None, :]
    sin = np.concatenate([np.sin(ang), np.sin(ang)], -1)[:, None, :]
    rot = np.concatenate([-X[..., D // 2:], X[..., :D // 2]], -1)
    return X * cos + rot * sin


def _store(x, kind):
    """What the cache keeps of fp64 rows x [..., D] (returned as fp64 values)."""
    if kind == "bf16":
        return torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    xf = x.astype(np.float32)
    amax = np.maximum(np.abs(xf).max(-1, keepdims=True), np.float32(2.0 ** -126))
    scale = (amax / np.float32(448.0)).astype(np.float32)
    q = (xf / scale).astype(np.float32)
    codes = torch.from_numpy(q).to(torch.float8_e4m3fn)
    return codes.double().numpy() * scale.astype(np.float64)


def brute_force(s, w, pre_k, pre_v, toks, n0, kind):
    """All logits [T, V] of the token sequence at positions n0..n0+T-1, with
    pre_k/pre_v [L, Hkv, n0, D] (fp64 values) as the rows before it."""
    T = len(toks)
    rep = s.n_q_heads // s.n_kv_heads
    X = _f(w["embed"])[toks]
    pos = np.arange(n0, n0 + T)
    for l, lw in enumerate(w["layers"]):
        Hn = _rms_rows(X, _f(lw["in_norm"]), s.rms_eps)
        Q = (Hn @ _f(lw["q"]).T).reshape(T, s.n_q_heads, s.head_dim)
        K = (Hn @ _f(lw["k"]).T).reshape(T, s.n_kv_heads, s.head_dim)
        V = (Hn @ _f(lw["v"]).T).reshape(T, s.n_kv_heads, s.head_dim)
        Q = _rope_rows(_rms_rows(Q, _f(lw["q_norm"]), s.rms_eps), pos, s.rope_theta)
        K = _rope_rows(_rms_rows(K, _f(lw["k_norm"]), s.rms_eps), pos, s.rope_theta)
        Ks = np.concatenate([pre_k[l], _store(K, kind).transpose(1, 0, 2)], axis=1)  # [Hkv, n0+T, D]
        Vs = np.concatenate([pre_v[l], _store(V, kind).transpose(1, 0, 2)], axis=1)
        Kr, Vr = np.repeat(Ks, rep, axis=0), np.repeat(Vs, rep, axis=0)               # repeat_kv
        S = np.einsum("thd,hjd->htj", Q, Kr) / math.sqrt(s.head_dim)
        mask = np.arange(n0 + T)[None, :] <= pos[:, None]                             # causal
        S = np.where(mask[None], S, -np.inf)
        A = np.exp(S - S.max(-1, keepdims=True))
        A /= A.sum(-1, keepdims=True)
        O = np.einsum("htj,hjd->thd", A, Vr).reshape(T, -1)
        X = X + O @ _f(lw["o"]).T
        Hn = _rms_rows(X, _f(lw["post_norm"]), s.rms_eps)
        G, U = Hn @ _f(lw["gate"]).T, Hn @ _f(lw["up"]).T
        X = X + (G / (1 + np.exp(-G)) * U) @ _f(lw["down"]).T
    return _rms_rows(X, _f(w["final_norm"]), s.rms_eps) @ _f(w["lm_head"]).T


def _decode(s, w, kv, sc, toks, n0):
    m = oracle.Model(oracle_shape(s), oracle_weights(w))
    cache = oracle_cache(kv, sc, 0)
    out = []
    for t, tok in enumerate(toks):
        out.append(m.step(cache, int(tok), n0 + t).logits)
    return np.stack(out), cache


SHAPES = [
    synth.TINY,
    synth.ModelShape(2, 96, 6, 2, 16, 160, 300),     # 3 query heads per KV head
    synth.ModelShape(1, 64, 4, 4, 16, 96, 200),      # one query head per KV head
]


@pytest.mark.parametrize("s", SHAPES, ids=["tiny", "rep3", "mha"])
@pytest.mark.parametrize("n0", [0, 5])
def test_cached_decode_equals_full_recompute_bf16(s, n0):
    w = synth.model_weights(s, seed=11, gain_std=0.1)
    kv, _ = synth.kv_prefill(s, 1, n0 + 8, [n0], seed=12)
    toks = synth.tokens(s.vocab, 7, seed=13).numpy()
    got, _ = _decode(s, w, kv, None, toks, n0)
    pre = kv[:, :, 0, :, :n0].double().numpy()
    ref = brute_force(s, w, pre[:, 0], pre[:, 1], toks, n0, "bf16")
    assert np.max(np.abs(got - ref)) < 1e-9


@pytest.mark.parametrize("n0", [0, 6])
def test_cached_decode_equals_full_recompute_fp8(n0):
    s = synth.TINY
    w = synth.model_weights(s, seed=21, gain_std=0.1)
    codes, scales = synth.kv_prefill(s, 1, n0 + 8, [n0], seed=22, kind="fp8")
    toks = synth.tokens(s.vocab, 6, seed=23).numpy()
    got, _ = _decode(s, w, codes, scales, toks, n0)
    deq = codes[:, :, 0, :, :n0].view(torch.float8_e4m3fn).double().numpy() \
        * scales[:, :, 0, :, :n0, None].double().numpy()
    ref = brute_force(s, w, deq[:, 0], deq[:, 1], toks, n0, "fp8")
    assert np.max(np.abs(got - ref)) < 1e-9


def test_step_writes_exactly_row_p_and_reports_new_kv():
    s = synth.TINY
    w = synth.model_weights(s, seed=31)
    kv, _ = synth.kv_prefill(s, 1, 40, [20], seed=32)
    m = oracle.Model(oracle_shape(s), oracle_weights(w))
    cache = oracle_cache(kv, None, 0)
    before = cache.kv.copy()
    r = m.step(cache, 7, 20, want_hidden=True, want_new_kv=True)
    changed = np.argwhere(np.any(before != cache.kv, axis=-1))
    assert set(changed[:, 3].tolist()) == {20}
    stored_k = oracle.bf16_round(r.new_k)                 # [L, Hkv, D]
    assert np.array_equal(cache.kv[:, 0, :, 20], stored_k)
    assert np.array_equal(cache.kv[:, 1, :, 20], oracle.bf16_round(r.new_v))
    assert r.hidden.shape == (s.n_layers + 1, s.hidden)
    assert np.array_equal(r.hidden[0], _f(w["embed"])[7])


def test_greedy_margin_and_argmax_agree():
    s = synth.TINY
    w = synth.model_weights(s, seed=41)
    kv, _ = synth.kv_prefill(s, 1, 16, [8], seed=42)
    m = oracle.Model(oracle_shape(s), oracle_weights(w))
    r = m.step(oracle_cache(kv, None, 0), 3, 8)
    srt = np.sort(r.logits)
    assert r.token == int(np.argmax(r.logits))
    assert math.isclose(r.margin, srt[-1] - srt[-2], rel_tol=1e-12)


def test_tied_embedding_is_one_buffer():
    s = synth.TINY
    w = synth.model_weights(s, seed=51, tied=True)
    assert w["lm_head"] is w["embed"]
