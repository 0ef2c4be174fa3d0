"""CPU oracle for the greedy decode step (test infrastructure only).

The oracle is the plain definition of one decode step of a Qwen3-style
decoder, written in C (``dec_oracle.c``) with every activation in double and
the weights / KV cache held in the bytes the system stores (bf16, or OCP FP8
E4M3 with an fp32 scale per row).  This module only builds that C file with
gcc and marshals numpy arrays into it.

Only the test suite, the package smoke check and the benchmark's CPU-baseline
leg may import this module.  The CUDA library never does, and this module
imports nothing from it.

Sources are cited in ``dec_oracle.c`` per function ("Qwen3-ASR -- Latency &
Bottleneck Analysis", 03 Decode and 07 Root causes; "Can CTC make Qwen3-ASR
faster?", 03 Greedy exactness; the Baseten Qwen3-ASR article, KV cache
quantization).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dec_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")

LAYER_KEYS = ("in_norm", "q", "k", "v", "q_norm", "k_norm", "o", "post_norm",
              "gate", "up", "down")


def build(force: bool = False) -> str:
    """Compile dec_oracle.c into oracle/_build/liboracle.so (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    os.makedirs(_LIB_DIR, exist_ok=True)
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P, I, D, F, U16, U8 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_double,
                               ctypes.c_float, ctypes.c_uint16, ctypes.c_uint8)
        L.or_bf16_to_double.argtypes, L.or_bf16_to_double.restype = [U16], D
        L.or_bf16_round.argtypes, L.or_bf16_round.restype = [D], U16
        L.or_e4m3_decode.argtypes, L.or_e4m3_decode.restype = [U8], D
        L.or_e4m3_encode.argtypes, L.or_e4m3_encode.restype = [D], U8
        L.or_e4m3_quantize_row.argtypes, L.or_e4m3_quantize_row.restype = [P, I, P], F
        L.or_rmsnorm.argtypes, L.or_rmsnorm.restype = [P, P, I, D, P], None
        L.or_gemv.argtypes, L.or_gemv.restype = [P, P, I, I, P], None
        L.or_rope.argtypes, L.or_rope.restype = [P, I, I, D], None
        L.or_silu.argtypes, L.or_silu.restype = [D], D
        L.or_attend.argtypes = [P, I, I, I, P, P, P, P, P, P, ctypes.c_size_t, P, P]
        L.or_attend.restype = None
        L.or_argmax.argtypes, L.or_argmax.restype = [P, I, P], I
        L.or_int8_quantize_row.argtypes = [P, I, P]
        L.or_int8_quantize_row.restype = F
        L.or_int8_quantize_rows.argtypes = [P, I, I, P, P]
        L.or_int8_quantize_rows.restype = None
        L.or_gemv_i8.argtypes, L.or_gemv_i8.restype = [P, P, P, I, I, P], None
        L.or_fp8w_quantize_rows.argtypes = [P, I, I, P, P]
        L.or_fp8w_quantize_rows.restype = None
        L.or_gemv_f8.argtypes, L.or_gemv_f8.restype = [P, P, P, I, I, P], None
        L.or_step.argtypes = [P, P, P, P, P, P, I, P, P, I, P, P, P, I, I, I, P, P, P, P, P]
        L.or_step.restype = I
        L.or_set_threads.argtypes, L.or_set_threads.restype = [I], None
        L.or_get_threads.argtypes, L.or_get_threads.restype = [], I
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> None:
    lib().or_set_threads(int(n))


def get_threads() -> int:
    return int(lib().or_get_threads())


# --------------------------------------------------------------- formats
def bf16_to_double(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    f = lib().or_bf16_to_double
    return np.array([f(int(v)) for v in b.ravel()], dtype=np.float64).reshape(b.shape)


def bf16_round(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    f = lib().or_bf16_round
    return np.array([f(float(v)) for v in x.ravel()], dtype=np.uint16).reshape(x.shape)


def e4m3_decode(codes) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8)
    f = lib().or_e4m3_decode
    return np.array([f(int(v)) for v in c.ravel()], dtype=np.float64).reshape(c.shape)


def e4m3_encode(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    f = lib().or_e4m3_encode
    return np.array([f(float(v)) for v in x.ravel()], dtype=np.uint8).reshape(x.shape)


def e4m3_quantize_row(x) -> tuple:
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.zeros(x.shape[-1], dtype=np.uint8)
    s = lib().or_e4m3_quantize_row(_p(x), x.shape[-1], _p(codes))
    return codes, float(s)


def int8_quantize_rows(W_bits) -> tuple:
    """Per-row symmetric int8 codes and fp32 scales of a bf16 matrix [rows, cols]
    (reading in dec_oracle.c, or_int8_quantize_row)."""
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    W2 = W.reshape(-1, W.shape[-1])
    codes = np.zeros(W2.shape, dtype=np.int8)
    scales = np.zeros(W2.shape[0], dtype=np.float32)
    lib().or_int8_quantize_rows(_p(W2), W2.shape[0], W2.shape[1], _p(codes), _p(scales))
    return codes.reshape(W.shape), scales.reshape(W.shape[:-1])


def fp8w_quantize_rows(W_bits) -> tuple:
    """Per-row E4M3 codes and fp32 scales of a bf16 matrix [rows, cols]
    (reading in dec_oracle.c, or_fp8w_quantize_rows)."""
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    W2 = W.reshape(-1, W.shape[-1])
    codes = np.zeros(W2.shape, dtype=np.uint8)
    scales = np.zeros(W2.shape[0], dtype=np.float32)
    lib().or_fp8w_quantize_rows(_p(W2), W2.shape[0], W2.shape[1], _p(codes), _p(scales))
    return codes.reshape(W.shape), scales.reshape(W.shape[:-1])


# ---------------------------------------------------------- building blocks
def rmsnorm(x, g_bits, eps: float) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    g = np.ascontiguousarray(g_bits, dtype=np.uint16)
    y = np.zeros_like(x)
    lib().or_rmsnorm(_p(x), _p(g), x.size, float(eps), _p(y))
    return y


def gemv(W_bits, x) -> np.ndarray:
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.zeros(W.shape[0], dtype=np.float64)
    lib().or_gemv(_p(W), _p(x), W.shape[0], W.shape[1], _p(y))
    return y


def gemv_i8(codes, scales, x) -> np.ndarray:
    C = np.ascontiguousarray(codes, dtype=np.int8)
    sc = np.ascontiguousarray(scales, dtype=np.float32)
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.zeros(C.shape[0], dtype=np.float64)
    lib().or_gemv_i8(_p(C), _p(sc), _p(x), C.shape[0], C.shape[1], _p(y))
    return y


def gemv_f8(codes, scales, x) -> np.ndarray:
    C = np.ascontiguousarray(codes, dtype=np.uint8)
    sc = np.ascontiguousarray(scales, dtype=np.float32)
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.zeros(C.shape[0], dtype=np.float64)
    lib().or_gemv_f8(_p(C), _p(sc), _p(x), C.shape[0], C.shape[1], _p(y))
    return y


def rope(x, p: int, theta: float) -> np.ndarray:
    y = np.array(x, dtype=np.float64, copy=True)
    lib().or_rope(_p(y), y.size, int(p), float(theta))
    return y


def silu(z: float) -> float:
    return float(lib().or_silu(float(z)))


def attend(q, K, V, n: Optional[int] = None, Kscale=None, Vscale=None,
           want_probs: bool = False):
    """Attention of one query q[D] over rows 0..n-1 of K/V [rows, D].

    K/V are uint16 bf16 bits, or uint8 E4M3 codes with per-row scales."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    d = q.size
    n = K.shape[0] if n is None else int(n)
    out = np.zeros(d, dtype=np.float64)
    probs = np.zeros(max(n, 1), dtype=np.float64) if want_probs else None
    L = lib()
    if K.dtype == np.uint16:
        K = np.ascontiguousarray(K)
        V = np.ascontiguousarray(V)
        L.or_attend(_p(q), d, n, 0, _p(K), _p(V), None, None, None, None, d, _p(out), _p(probs))
    else:
        K = np.ascontiguousarray(K, dtype=np.uint8)
        V = np.ascontiguousarray(V, dtype=np.uint8)
        ks = np.ascontiguousarray(Kscale, dtype=np.float32)
        vs = np.ascontiguousarray(Vscale, dtype=np.float32)
        L.or_attend(_p(q), d, n, 1, None, None, _p(K), _p(V), _p(ks), _p(vs), d, _p(out), _p(probs))
    return (out, probs[:n]) if want_probs else out


def argmax(v) -> tuple:
    v = np.ascontiguousarray(v, dtype=np.float64)
    m = ctypes.c_double(0.0)
    i = lib().or_argmax(_p(v), v.size, ctypes.byref(m))
    return int(i), float(m.value)


# ---------------------------------------------------------------- model
@dataclass
class Shape:
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rms_eps: float = 1e-6
    rope_theta: float = 1e6


PROJ_KEYS = ("q", "k", "v", "o", "gate", "up", "down")


@dataclass
class Weights:
    """bf16 bits (np.uint16) of every tensor; layer tensors keyed by LAYER_KEYS.

    kind "int8" / "fp8": the PROJ_KEYS tensors of every layer and lm_head are
    int8 / E4M3 codes, with fp32 row scales in `scales` (per layer, keyed by
    PROJ_KEYS) and `lm_scale`; the embedding and the norm gains stay bf16."""
    embed: np.ndarray
    lm_head: np.ndarray
    final_norm: np.ndarray
    layers: List[Dict[str, np.ndarray]]
    kind: str = "bf16"
    lm_scale: Optional[np.ndarray] = None
    scales: Optional[List[Dict[str, np.ndarray]]] = None


def _quantize_weights(w: Weights, rows_fn, kind: str) -> Weights:
    assert w.kind == "bf16"
    layers, scales = [], []
    for lw in w.layers:
        nl, ns = dict(lw), {}
        for key in PROJ_KEYS:
            nl[key], ns[key] = rows_fn(lw[key])
        layers.append(nl)
        scales.append(ns)
    lm, lms = rows_fn(w.lm_head)
    return Weights(embed=w.embed, lm_head=lm, final_norm=w.final_norm, layers=layers,
                   kind=kind, lm_scale=lms, scales=scales)


def quantize_weights_int8(w: Weights) -> Weights:
    """The int8 weight-only model of a bf16 one: every projection and lm_head
    quantised per row (int8_quantize_rows)."""
    return _quantize_weights(w, int8_quantize_rows, "int8")


def quantize_weights_fp8(w: Weights) -> Weights:
    """The E4M3 weight-only model of a bf16 one: every projection and lm_head
    quantised per row (fp8w_quantize_rows)."""
    return _quantize_weights(w, fp8w_quantize_rows, "fp8")


@dataclass
class Cache:
    """KV cache of ONE sequence: kind 'bf16' -> kv [L,2,Hkv,max_ctx,D] uint16;
    kind 'fp8' -> kv [L,2,Hkv,max_ctx,D] uint8 codes + scales [L,2,Hkv,max_ctx]."""
    kind: str
    kv: np.ndarray
    scales: Optional[np.ndarray] = None

    @property
    def max_ctx(self) -> int:
        return int(self.kv.shape[3])


@dataclass
class StepResult:
    token: int
    margin: float
    logits: np.ndarray
    hidden: Optional[np.ndarray] = None
    new_k: Optional[np.ndarray] = None
    new_v: Optional[np.ndarray] = None


class Model:
    """Holds the weights and the pointer table the C step function reads."""

    def __init__(self, shape: Shape, w: Weights):
        self.shape = shape
        self.w = w
        self._keep = []
        L = shape.n_layers
        i8 = w.kind in ("int8", "fp8")   # 8-bit codes with row scales
        if w.kind not in ("bf16", "int8", "fp8"):
            raise ValueError(w.kind)
        cdt = np.int8 if w.kind == "int8" else np.uint8
        ptrs = (ctypes.c_void_p * (L * len(LAYER_KEYS)))()
        sptrs = (ctypes.c_void_p * (L * len(LAYER_KEYS)))()
        for l, lw in enumerate(w.layers):
            for j, key in enumerate(LAYER_KEYS):
                proj = i8 and key in PROJ_KEYS
                a = np.ascontiguousarray(lw[key], dtype=cdt if proj else np.uint16)
                self._keep.append(a)
                ptrs[l * len(LAYER_KEYS) + j] = a.ctypes.data
                if proj:
                    sc = np.ascontiguousarray(w.scales[l][key], dtype=np.float32)
                    assert sc.shape == (a.shape[0],)
                    self._keep.append(sc)
                    sptrs[l * len(LAYER_KEYS) + j] = sc.ctypes.data
        self._ptrs = ptrs
        self._sptrs = sptrs
        self._wkind = {"bf16": 0, "int8": 1, "fp8": 2}[w.kind]
        self._emb = np.ascontiguousarray(w.embed, dtype=np.uint16)
        self._lm = np.ascontiguousarray(w.lm_head, dtype=cdt if i8 else np.uint16)
        self._lms = np.ascontiguousarray(w.lm_scale, dtype=np.float32) if i8 else None
        self._fn = np.ascontiguousarray(w.final_norm, dtype=np.uint16)
        s = shape
        self._sh = np.array([s.n_layers, s.hidden, s.n_q_heads, s.n_kv_heads, s.head_dim,
                             s.ffn, s.vocab], dtype=np.int32)
        self._shd = np.array([s.rms_eps, s.rope_theta], dtype=np.float64)

    def step(self, cache: Cache, token: int, pos: int, want_hidden: bool = False,
             want_new_kv: bool = False) -> StepResult:
        """One greedy decode step of one sequence; writes row `pos` of `cache`."""
        s = self.shape
        if not (0 <= pos < cache.max_ctx):
            raise ValueError("position outside the cache")
        if not (0 <= token < s.vocab):
            raise ValueError("token outside the vocabulary")
        logits = np.zeros(s.vocab, dtype=np.float64)
        hidden = np.zeros((s.n_layers + 1, s.hidden)) if want_hidden else None
        nk = np.zeros((s.n_layers, s.n_kv_heads, s.head_dim)) if want_new_kv else None
        nv = np.zeros_like(nk) if want_new_kv else None
        margin = ctypes.c_double(0.0)
        assert cache.kv.flags["C_CONTIGUOUS"]
        if cache.kind == "bf16":
            assert cache.kv.dtype == np.uint16
            kind, k16, k8, ks = 0, cache.kv, None, None
        elif cache.kind == "fp8":
            assert cache.kv.dtype == np.uint8 and cache.scales.flags["C_CONTIGUOUS"]
            kind, k16, k8, ks = 1, None, cache.kv, cache.scales
        else:
            raise ValueError(cache.kind)
        tok = lib().or_step(_p(self._sh), _p(self._shd), _p(self._emb), _p(self._lm),
                            _p(self._fn), ctypes.cast(self._ptrs, ctypes.c_void_p),
                            self._wkind, _p(self._lms),
                            ctypes.cast(self._sptrs, ctypes.c_void_p), kind,
                            _p(k16), _p(k8), _p(ks), cache.max_ctx, int(token), int(pos),
                            _p(logits), _p(hidden), _p(nk), _p(nv), ctypes.byref(margin))
        return StepResult(int(tok), float(margin.value), logits, hidden, nk, nv)


# ------------------------------------------------- input marshalling helpers
# Views of the seeded synthetic inputs (torch tensors from the input
# generators) in the oracle's numpy form: raw bytes only, no arithmetic.

def _bits16(t) -> np.ndarray:
    """The raw 16-bit patterns of a bf16 torch tensor as numpy uint16."""
    import torch
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def shape_from(s) -> Shape:
    """A model shape (any object with the Shape field names) as a Shape."""
    return Shape(s.n_layers, s.hidden, s.n_q_heads, s.n_kv_heads, s.head_dim, s.ffn, s.vocab,
                 s.rms_eps, s.rope_theta)


def weights_from(w) -> Weights:
    """{"embed", "lm_head", "final_norm", "layers": [dict per layer]} of bf16
    torch tensors as Weights of uint16 bit patterns."""
    layers = [{k: _bits16(t) for k, t in lw.items()} for lw in w["layers"]]
    return Weights(embed=_bits16(w["embed"]), lm_head=_bits16(w["lm_head"]),
                   final_norm=_bits16(w["final_norm"]), layers=layers)


def cache_from(kv, scales, b: int) -> Cache:
    """Sequence b of a [L, 2, B, Hkv, max_ctx, D] cache (bf16 values, or E4M3
    codes with fp32 scales [L, 2, B, Hkv, max_ctx]) as a Cache (a copy)."""
    if scales is None:
        return Cache("bf16", np.ascontiguousarray(_bits16(kv[:, :, b])))
    codes = np.ascontiguousarray(kv[:, :, b].cpu().numpy())
    sc = np.ascontiguousarray(scales[:, :, b].cpu().numpy())
    return Cache("fp8", codes, sc)
