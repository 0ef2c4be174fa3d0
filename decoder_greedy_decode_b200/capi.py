"""ctypes binding of libdec.so: the C ABI of include/dec.h, same names.

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of libdec.so.  There is no CPU fallback: if the library is missing the
import of this module's functions raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("DEC_LIBRARY", os.path.join(HERE, "libdec.so"))

DEC_KV_BF16 = 0
DEC_KV_FP8_E4M3 = 1
DEC_DEV_BAD_POSITION = 1
DEC_DEV_BAD_TOKEN = 2
DEC_DEV_TIMEOUT = 4
DEC_ERR_TOO_LARGE = -10
LW_ORDER = ("in_norm", "q", "k", "v", "q_norm", "k_norm", "o", "post_norm", "gate", "up", "down")

#: every symbol include/dec.h declares
EXPORTS = (
    "dec_init", "dec_free", "dec_kv_bytes", "dec_kv_scale_offset", "dec_kv_alloc", "dec_step",
    "dec_step_debug", "dec_step_host", "dec_check", "dec_set_timeout_ns", "dec_set_debug_stall",
    "dec_error_string", "dec_last_cuda_error", "dec_get_config",
    "dec_attention_workspace_bytes", "dec_attention", "dec_kv_quantize_e4m3",
    "dec_attention_noalloc", "dec_verify", "dec_accept_greedy", "dec_generate",
    "dec_init_int8", "dec_quantize_int8", "dec_init_fp8w", "dec_quantize_fp8w",
)
#: the projections an int8 handle holds as int8 codes + row scales
PROJ_KEYS = ("q", "k", "v", "o", "gate", "up", "down")


class dec_shape(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("hidden", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("ffn", ctypes.c_int),
                ("vocab", ctypes.c_int), ("rms_eps", ctypes.c_float),
                ("rope_theta", ctypes.c_float), ("max_batch", ctypes.c_int)]


class dec_weights(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("lm_head", ctypes.c_void_p),
                ("final_norm", ctypes.c_void_p), ("layers", ctypes.POINTER(ctypes.c_void_p))]


class dec_weights_int8(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("lm_head", ctypes.c_void_p),
                ("lm_head_scale", ctypes.c_void_p), ("final_norm", ctypes.c_void_p),
                ("layers", ctypes.POINTER(ctypes.c_void_p)),
                ("scales", ctypes.POINTER(ctypes.c_void_p))]


class dec_kv(ctypes.Structure):
    _fields_ = [("base", ctypes.c_void_p), ("bytes", ctypes.c_size_t), ("batch", ctypes.c_int),
                ("max_ctx", ctypes.c_int), ("dtype", ctypes.c_int)]


class DecError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {error_string(code)} ({code})"
                         + (f", cuda error {lib().dec_last_cuda_error()}" if code == -7 else ""))


_lib = None


def lib() -> ctypes.CDLL:
    """Load libdec.so (built in-tree by decoder_greedy_decode_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m decoder_greedy_decode_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, Z, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_ulonglong
        sig = {
            "dec_init": ([ctypes.POINTER(dec_shape), ctypes.POINTER(dec_weights), ctypes.POINTER(P)], I),
            "dec_free": ([P], None),
            "dec_kv_bytes": ([P, I, I, I], Z),
            "dec_kv_scale_offset": ([P, I, I, I], Z),
            "dec_kv_alloc": ([P, I, I, I, P, Z, ctypes.POINTER(dec_kv)], I),
            "dec_step": ([P, I, P, P, ctypes.POINTER(dec_kv), P, P, P], I),
            "dec_step_debug": ([P, I, P, P, ctypes.POINTER(dec_kv), P, P, P, P], I),
            "dec_step_host": ([P, I, P, P, ctypes.POINTER(dec_kv), P, P, P], I),
            "dec_check": ([P, P], I),
            "dec_set_timeout_ns": ([P, U64], I),
            "dec_set_debug_stall": ([P, I], I),
            "dec_error_string": ([I], ctypes.c_char_p),
            "dec_last_cuda_error": ([], I),
            "dec_get_config": ([P, ctypes.POINTER(I), ctypes.POINTER(I), ctypes.POINTER(I)], I),
            "dec_attention_workspace_bytes": ([I, I, I, I, I], Z),
            "dec_attention": ([I, I, I, I, P, P, P, I, P, P, P, Z, P, P], I),
            "dec_kv_quantize_e4m3": ([P, I, I, P, P, P], I),
            "dec_attention_noalloc": ([I, I, I, I, P, P, P, I, P, P, P, P], I),
            "dec_verify": ([P, I, P, P, I, ctypes.POINTER(dec_kv), P, P, P], I),
            "dec_accept_greedy": ([I, P, P, P, ctypes.POINTER(I)], I),
            "dec_generate": ([P, I, I, P, P, ctypes.POINTER(dec_kv), P, I, P], I),
            "dec_init_int8": ([ctypes.POINTER(dec_shape), ctypes.POINTER(dec_weights_int8),
                               ctypes.POINTER(P)], I),
            "dec_quantize_int8": ([P, I, I, P, P, P], I),
            "dec_init_fp8w": ([ctypes.POINTER(dec_shape), ctypes.POINTER(dec_weights_int8),
                               ctypes.POINTER(P)], I),
            "dec_quantize_fp8w": ([P, I, I, P, P, P], I),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes, f.restype = args, res
        _lib = L
    return _lib


def error_string(code: int) -> str:
    return lib().dec_error_string(int(code)).decode()


def _ok(rc: int, what: str) -> int:
    if rc < 0:
        raise DecError(rc, what)
    return rc


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return int(t.data_ptr()) if hasattr(t, "data_ptr") else int(t)


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    return int(getattr(stream, "cuda_stream", stream))


# ------------------------------------------------------------------ C ABI
def dec_init(shape: dec_shape, embed, lm_head, final_norm, layer_ptrs: Sequence[int]) -> int:
    arr = (ctypes.c_void_p * len(layer_ptrs))(*[int(p) for p in layer_ptrs])
    w = dec_weights(_ptr(embed), _ptr(lm_head), _ptr(final_norm),
                    ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)))
    h = ctypes.c_void_p()
    _ok(lib().dec_init(ctypes.byref(shape), ctypes.byref(w), ctypes.byref(h)), "dec_init")
    return h.value


def dec_init_int8(shape: dec_shape, embed, lm_head, lm_head_scale, final_norm,
                  layer_ptrs: Sequence[int], scale_ptrs: Sequence[Optional[int]],
                  entry: str = "dec_init_int8") -> int:
    """dec_init_int8, or with entry="dec_init_fp8w" the same call for E4M3
    codes."""
    arr = (ctypes.c_void_p * len(layer_ptrs))(*[int(p) for p in layer_ptrs])
    sarr = (ctypes.c_void_p * len(scale_ptrs))(*[None if p is None else int(p)
                                                 for p in scale_ptrs])
    w = dec_weights_int8(_ptr(embed), _ptr(lm_head), _ptr(lm_head_scale), _ptr(final_norm),
                         ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)),
                         ctypes.cast(sarr, ctypes.POINTER(ctypes.c_void_p)))
    h = ctypes.c_void_p()
    _ok(getattr(lib(), entry)(ctypes.byref(shape), ctypes.byref(w), ctypes.byref(h)), entry)
    return h.value


def dec_init_fp8w(shape: dec_shape, embed, lm_head, lm_head_scale, final_norm,
                  layer_ptrs: Sequence[int], scale_ptrs: Sequence[Optional[int]]) -> int:
    return dec_init_int8(shape, embed, lm_head, lm_head_scale, final_norm, layer_ptrs,
                         scale_ptrs, entry="dec_init_fp8w")


def dec_quantize_int8(w, rows: int, cols: int, codes, scales, stream=None) -> None:
    _ok(lib().dec_quantize_int8(_ptr(w), rows, cols, _ptr(codes), _ptr(scales),
                                _stream(stream)), "dec_quantize_int8")


def dec_quantize_fp8w(w, rows: int, cols: int, codes, scales, stream=None) -> None:
    _ok(lib().dec_quantize_fp8w(_ptr(w), rows, cols, _ptr(codes), _ptr(scales),
                                _stream(stream)), "dec_quantize_fp8w")


def dec_free(h: int) -> None:
    lib().dec_free(h)


def dec_kv_bytes(h: int, batch: int, max_ctx: int, dtype: int) -> int:
    return int(lib().dec_kv_bytes(h, batch, max_ctx, dtype))


def dec_kv_scale_offset(h: int, batch: int, max_ctx: int, dtype: int) -> int:
    return int(lib().dec_kv_scale_offset(h, batch, max_ctx, dtype))


def dec_kv_alloc(h: int, batch: int, max_ctx: int, dtype: int, buf, nbytes: int) -> dec_kv:
    kv = dec_kv()
    _ok(lib().dec_kv_alloc(h, batch, max_ctx, dtype, _ptr(buf), nbytes, ctypes.byref(kv)),
        "dec_kv_alloc")
    return kv


def dec_step(h: int, batch: int, token_ids, positions, kv: dec_kv, out_ids, out_logits=None,
             stream=None) -> None:
    _ok(lib().dec_step(h, batch, _ptr(token_ids), _ptr(positions), ctypes.byref(kv),
                       _ptr(out_ids), _ptr(out_logits), _stream(stream)), "dec_step")


def dec_verify(h: int, k: int, token_ids, positions, seq: int, kv: dec_kv, out_ids,
               out_logits=None, stream=None) -> None:
    _ok(lib().dec_verify(h, k, _ptr(token_ids), _ptr(positions), seq, ctypes.byref(kv),
                         _ptr(out_ids), _ptr(out_logits), _stream(stream)), "dec_verify")


def dec_generate(h: int, batch: int, n_steps: int, token_ids, positions, kv: dec_kv, out_ids,
                 eos: int = -1, stream=None) -> None:
    _ok(lib().dec_generate(h, batch, n_steps, _ptr(token_ids), _ptr(positions),
                           ctypes.byref(kv), _ptr(out_ids), int(eos), _stream(stream)),
        "dec_generate")


def dec_accept_greedy(tokens: Sequence[int], out_ids: Sequence[int]) -> list:
    """Greedy acceptance of a verified block (host lists): the emitted tokens."""
    k = len(tokens)
    t = (ctypes.c_int32 * k)(*[int(x) for x in tokens])
    o = (ctypes.c_int32 * k)(*[int(x) for x in out_ids])
    e = (ctypes.c_int32 * k)()
    n = ctypes.c_int()
    _ok(lib().dec_accept_greedy(k, t, o, e, ctypes.byref(n)), "dec_accept_greedy")
    return [int(e[i]) for i in range(n.value)]


def dec_step_debug(h: int, batch: int, token_ids, positions, kv: dec_kv, out_ids, out_logits,
                   hidden_out, stream=None) -> None:
    _ok(lib().dec_step_debug(h, batch, _ptr(token_ids), _ptr(positions), ctypes.byref(kv),
                             _ptr(out_ids), _ptr(out_logits), _ptr(hidden_out), _stream(stream)),
        "dec_step_debug")


def dec_step_host(h: int, batch: int, token_ids_host, positions_host, kv: dec_kv, out_ids_host,
                  out_logits_host=None, stream=None) -> None:
    _ok(lib().dec_step_host(h, batch, _ptr(token_ids_host), _ptr(positions_host),
                            ctypes.byref(kv), _ptr(out_ids_host), _ptr(out_logits_host),
                            _stream(stream)), "dec_step_host")


def dec_check(h: int, stream=None) -> int:
    return _ok(lib().dec_check(h, _stream(stream)), "dec_check")


def dec_set_timeout_ns(h: int, ns: int) -> None:
    _ok(lib().dec_set_timeout_ns(h, int(ns)), "dec_set_timeout_ns")


def dec_set_debug_stall(h: int, cta_plus_one: int) -> None:
    _ok(lib().dec_set_debug_stall(h, int(cta_plus_one)), "dec_set_debug_stall")


def dec_get_config(h: int) -> dict:
    c, s, b = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _ok(lib().dec_get_config(h, ctypes.byref(c), ctypes.byref(s), ctypes.byref(b)), "dec_get_config")
    return {"ctas": c.value, "ring_slots": s.value, "slot_bytes": b.value}


def dec_attention_workspace_bytes(batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                                  max_len: int) -> int:
    return int(lib().dec_attention_workspace_bytes(batch, n_q_heads, n_kv_heads, head_dim, max_len))


def dec_attention(batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int, q, k_cache,
                  v_cache, max_len: int, lengths, out, workspace, workspace_bytes: int,
                  status=None, stream=None) -> None:
    _ok(lib().dec_attention(batch, n_q_heads, n_kv_heads, head_dim, _ptr(q), _ptr(k_cache),
                            _ptr(v_cache), max_len, _ptr(lengths), _ptr(out), _ptr(workspace),
                            workspace_bytes, _ptr(status), _stream(stream)), "dec_attention")


def dec_kv_quantize_e4m3(x, rows: int, dim: int, codes, scales, stream=None) -> None:
    _ok(lib().dec_kv_quantize_e4m3(_ptr(x), rows, dim, _ptr(codes), _ptr(scales),
                                   _stream(stream)), "dec_kv_quantize_e4m3")


def dec_attention_noalloc(batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int, q, k_cache,
                          v_cache, max_len: int, lengths, out, status=None, stream=None) -> None:
    _ok(lib().dec_attention_noalloc(batch, n_q_heads, n_kv_heads, head_dim, _ptr(q), _ptr(k_cache),
                                    _ptr(v_cache), max_len, _ptr(lengths), _ptr(out), _ptr(status),
                                    _stream(stream)), "dec_attention_noalloc")
