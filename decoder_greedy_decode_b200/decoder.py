"""Convenience wrapper over the C ABI for PyTorch callers.

Marshalling only: torch provides device memory and streams, every step of the
decode path runs in libdec.so's kernels.
"""
from __future__ import annotations

from typing import Dict, Optional

import torch

from . import capi
from .synth import LAYER_KEYS, ModelShape

assert tuple(LAYER_KEYS) == tuple(capi.LW_ORDER)


def to_device(w: Dict[str, object], device: str = "cuda") -> Dict[str, object]:
    """Copy synth.model_weights(...) tensors to the device (keeps tying)."""
    emb = w["embed"].to(device)
    lm = emb if w["lm_head"] is w["embed"] else w["lm_head"].to(device)
    return {"embed": emb, "lm_head": lm, "final_norm": w["final_norm"].to(device),
            "layers": [{k: t.to(device) for k, t in lw.items()} for lw in w["layers"]]}


def quantize_int8(w: Dict[str, object], kind: str = "int8") -> Dict[str, object]:
    """Weight-only 8-bit copy of device weights (to_device(...) layout): every
    projection and lm_head quantised per output row by dec_quantize_int8
    (kind "int8": int8 codes) or dec_quantize_fp8w (kind "fp8": E4M3 codes),
    with fp32 row scales; embedding and norm gains shared."""
    def q(t):
        rows, cols = t.shape
        codes = torch.empty((rows, cols), dtype=torch.int8 if kind == "int8" else torch.uint8,
                            device=t.device)
        scales = torch.empty(rows, dtype=torch.float32, device=t.device)
        if kind == "int8":
            capi.dec_quantize_int8(t, rows, cols, codes, scales)
        else:
            capi.dec_quantize_fp8w(t, rows, cols, codes, scales)
        return codes, scales

    layers, scales = [], []
    for lw in w["layers"]:
        nl, ns = dict(lw), {}
        for key in capi.PROJ_KEYS:
            nl[key], ns[key] = q(lw[key])
        layers.append(nl)
        scales.append(ns)
    lm, lms = q(w["lm_head"])
    return {"kind": kind, "embed": w["embed"], "lm_head": lm, "lm_head_scale": lms,
            "final_norm": w["final_norm"], "layers": layers, "scales": scales}


def quantize_fp8w(w: Dict[str, object]) -> Dict[str, object]:
    """Weight-only E4M3 copy of device weights (quantize_int8 with E4M3 codes)."""
    return quantize_int8(w, kind="fp8")


class KVCache:
    """A caller-owned cache buffer (torch) bound through dec_kv_alloc."""

    def __init__(self, dec: "Decoder", batch: int, max_ctx: int, dtype: str = "bf16",
                 device: str = "cuda"):
        s = dec.shape
        self.dtype_code = capi.DEC_KV_BF16 if dtype == "bf16" else capi.DEC_KV_FP8_E4M3
        self.dtype = dtype
        self.batch, self.max_ctx = batch, max_ctx
        nbytes = capi.dec_kv_bytes(dec.h, batch, max_ctx, self.dtype_code)
        if nbytes == 0:
            raise ValueError("invalid KV size")
        self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        self.kv = capi.dec_kv_alloc(dec.h, batch, max_ctx, self.dtype_code, self.buf, nbytes)
        shp = (s.n_layers, 2, batch, s.n_kv_heads, max_ctx, s.head_dim)
        if dtype == "bf16":
            self.values = self.buf.view(torch.bfloat16).view(shp)
            self.codes = self.scales = None
        else:
            off = capi.dec_kv_scale_offset(dec.h, batch, max_ctx, self.dtype_code)
            n = 1
            for d in shp:
                n *= d
            self.values = None
            self.codes = self.buf[:n].view(shp)
            self.scales = self.buf[off:off + 4 * n // s.head_dim].view(torch.float32).view(shp[:-1])


class Decoder:
    """Owns one dec_handle for a model whose weights live in device tensors."""

    def __init__(self, shape: ModelShape, weights: Dict[str, object], max_batch: int = 1):
        self.shape = shape
        self.w = weights
        cs = capi.dec_shape(shape.n_layers, shape.hidden, shape.n_q_heads, shape.n_kv_heads,
                            shape.head_dim, shape.ffn, shape.vocab, shape.rms_eps,
                            shape.rope_theta, max_batch)
        ptrs = [weights["layers"][l][k].data_ptr() for l in range(shape.n_layers)
                for k in capi.LW_ORDER]
        if weights.get("kind") in ("int8", "fp8"):
            sptrs = [weights["scales"][l][k].data_ptr() if k in capi.PROJ_KEYS else None
                     for l in range(shape.n_layers) for k in capi.LW_ORDER]
            self.h = capi.dec_init_int8(cs, weights["embed"], weights["lm_head"],
                                        weights["lm_head_scale"], weights["final_norm"], ptrs,
                                        sptrs, entry="dec_init_int8" if weights["kind"] == "int8"
                                        else "dec_init_fp8w")
        else:
            self.h = capi.dec_init(cs, weights["embed"], weights["lm_head"],
                                   weights["final_norm"], ptrs)
        self.max_batch = max_batch

    def close(self) -> None:
        if getattr(self, "h", None):
            capi.dec_free(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def config(self) -> dict:
        return capi.dec_get_config(self.h)

    def kv_cache(self, batch: int, max_ctx: int, dtype: str = "bf16") -> KVCache:
        return KVCache(self, batch, max_ctx, dtype)

    def step(self, kv: KVCache, token_ids, positions, out_ids, logits=None, stream=None,
             batch: Optional[int] = None) -> None:
        b = int(token_ids.numel()) if batch is None else batch
        capi.dec_step(self.h, b, token_ids, positions, kv.kv, out_ids, logits, stream)

    def generate(self, kv: KVCache, token_ids, positions, out_ids, eos: int = -1,
                 stream=None) -> None:
        """out_ids.shape[0] greedy steps on the device; positions advance in place."""
        capi.dec_generate(self.h, int(token_ids.numel()), int(out_ids.shape[0]), token_ids,
                          positions, kv.kv, out_ids, eos, stream)

    def verify(self, kv: KVCache, token_ids, positions, seq: int, out_ids, logits=None,
               stream=None) -> None:
        """One step over k consecutive tokens of cache sequence `seq`
        (positions p0 .. p0+k-1): out_ids[i] is the greedy token after
        token_ids[i]."""
        capi.dec_verify(self.h, int(token_ids.numel()), token_ids, positions, seq, kv.kv,
                        out_ids, logits, stream)

    def step_debug(self, kv: KVCache, token_ids, positions, out_ids, logits, hidden,
                   stream=None) -> None:
        capi.dec_step_debug(self.h, int(token_ids.numel()), token_ids, positions, kv.kv,
                            out_ids, logits, hidden, stream)

    def step_host(self, kv: KVCache, token_ids_host, positions_host, out_ids_host,
                  logits_host=None, stream=None) -> None:
        capi.dec_step_host(self.h, int(token_ids_host.numel()), token_ids_host, positions_host,
                           kv.kv, out_ids_host, logits_host, stream)

    def check(self, stream=None) -> int:
        return capi.dec_check(self.h, stream)

    def set_timeout_ns(self, ns: int) -> None:
        capi.dec_set_timeout_ns(self.h, ns)

    def set_debug_stall(self, cta_plus_one: int) -> None:
        capi.dec_set_debug_stall(self.h, cta_plus_one)
