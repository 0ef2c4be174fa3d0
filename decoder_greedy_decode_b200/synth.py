"""Seeded synthetic inputs: weights, prefilled KV caches, tokens and lengths.

This module draws random numbers and nothing else: it holds none of the decode
step's arithmetic, so both the CUDA path and the CPU oracle can be fed from it.
Every tensor is drawn on the CPU with a seeded ``torch.Generator`` (so a CPU
test and a GPU run see the same bytes) and cast to bf16 by torch.

Workload shapes follow the pages' measurements: the Qwen3-ASR-0.6B decoder
profiled in "Qwen3-ASR -- Latency & Bottleneck Analysis" (28 layers,
hidden 1024, lm_head 1024->151936, a 795-token prompt followed by 130 greedy
tokens, 01 Method & setup and 03 Decode) and the 1.7B model of the Baseten
batch-transcription article (64 concurrent requests of 30 s windows).  The
pages measure real audio; synthetic random-init weights and N(0,1) caches of
the same shapes stand in for them.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence

import torch


@dataclass(frozen=True)
class ModelShape:
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rms_eps: float = 1e-6
    rope_theta: float = 1e6


#: 2 layers, hidden 256, 4/2 heads of 64, FFN 768, vocab 4096 (parity-only size)
TINY = ModelShape(2, 256, 4, 2, 64, 768, 4096)
#: Qwen3-ASR-0.6B text decoder shape
QWEN3_0_6B = ModelShape(28, 1024, 16, 8, 128, 3072, 151936)
#: Qwen3-ASR-1.7B text decoder shape
QWEN3_1_7B = ModelShape(28, 2048, 16, 8, 128, 6144, 151936)

LAYER_KEYS = ("in_norm", "q", "k", "v", "q_norm", "k_norm", "o", "post_norm",
              "gate", "up", "down")


def layer_shapes(s: ModelShape) -> Dict[str, tuple]:
    """[out, in] of every per-layer tensor (row-major, y = W x)."""
    nq, nkv = s.n_q_heads * s.head_dim, s.n_kv_heads * s.head_dim
    return {
        "in_norm": (s.hidden,), "q": (nq, s.hidden), "k": (nkv, s.hidden),
        "v": (nkv, s.hidden), "q_norm": (s.head_dim,), "k_norm": (s.head_dim,),
        "o": (s.hidden, nq), "post_norm": (s.hidden,), "gate": (s.ffn, s.hidden),
        "up": (s.ffn, s.hidden), "down": (s.hidden, s.ffn),
    }


def _normal(gen: torch.Generator, shape, std: float) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.bfloat16)
    flat = out.view(-1)
    chunk = 1 << 24
    for i in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - i)
        flat[i:i + n] = (torch.randn(n, generator=gen) * std).to(torch.bfloat16)
    return out


def _gain(gen: torch.Generator, n: int, gain_std: float) -> torch.Tensor:
    if gain_std == 0.0:
        return torch.ones(n, dtype=torch.bfloat16)
    return (1.0 + gain_std * torch.randn(n, generator=gen)).to(torch.bfloat16)


def model_weights(s: ModelShape, seed: int, std: float = 0.02, gain_std: float = 0.0,
                  tied: bool = False) -> Dict[str, object]:
    """Random-init bf16 weights ~N(0, std); RMSNorm gains 1.0 (or 1 + N(0, gain_std)).

    Returns {"embed", "lm_head", "final_norm", "layers": [dict per layer]}."""
    gen = torch.Generator().manual_seed(int(seed))
    embed = _normal(gen, (s.vocab, s.hidden), std)
    lm_head = embed if tied else _normal(gen, (s.vocab, s.hidden), std)
    final_norm = _gain(gen, s.hidden, gain_std)
    layers: List[Dict[str, torch.Tensor]] = []
    for _ in range(s.n_layers):
        lw = {}
        for key, shp in layer_shapes(s).items():
            lw[key] = _gain(gen, shp[0], gain_std) if len(shp) == 1 else _normal(gen, shp, std)
        layers.append(lw)
    return {"embed": embed, "lm_head": lm_head, "final_norm": final_norm, "layers": layers}


def kv_prefill(s: ModelShape, batch: int, max_ctx: int, lengths: Sequence[int], seed: int,
               kind: str = "bf16"):
    """A KV cache [L, 2, B, Hkv, max_ctx, D] whose first lengths[b] rows of every
    (layer, K/V, head) of sequence b are random; the rest are zero.

    kind 'bf16': N(0,1) values cast to bf16 -> (tensor bf16, None).
    kind 'fp8' : E4M3 codes of N(0,1)*32 drawn through torch's float8 cast and
                 per-row scales ~U[0.02, 0.04] -> (codes uint8, scales fp32
                 [L, 2, B, Hkv, max_ctx])."""
    gen = torch.Generator().manual_seed(int(seed))
    L, Hkv, D = s.n_layers, s.n_kv_heads, s.head_dim
    if kind == "bf16":
        kv = torch.zeros((L, 2, batch, Hkv, max_ctx, D), dtype=torch.bfloat16)
        for b, n in enumerate(lengths):
            if n > 0:
                kv[:, :, b, :, :n, :] = torch.randn((L, 2, Hkv, n, D), generator=gen).to(torch.bfloat16)
        return kv, None
    if kind == "fp8":
        codes = torch.zeros((L, 2, batch, Hkv, max_ctx, D), dtype=torch.uint8)
        scales = torch.zeros((L, 2, batch, Hkv, max_ctx), dtype=torch.float32)
        for b, n in enumerate(lengths):
            if n > 0:
                z = (torch.randn((L, 2, Hkv, n, D), generator=gen) * 32.0).to(torch.float8_e4m3fn)
                codes[:, :, b, :, :n, :] = z.view(torch.uint8)
                scales[:, :, b, :, :n] = 0.02 + 0.02 * torch.rand((L, 2, Hkv, n), generator=gen)
        return codes, scales
    raise ValueError(kind)


def kv_prefill_seq(s: ModelShape, max_ctx: int, n: int, seed: int, kind: str = "bf16"):
    """One sequence's cache planes [L, 2, Hkv, max_ctx, D] drawn from its own
    generator (seed), so that a large batch can be filled one sequence at a
    time and only the sampled sequences need a host copy.  Same value recipe
    as kv_prefill: first n rows random, the rest zero."""
    gen = torch.Generator().manual_seed(int(seed))
    L, Hkv, D = s.n_layers, s.n_kv_heads, s.head_dim
    if kind == "bf16":
        kv = torch.zeros((L, 2, Hkv, max_ctx, D), dtype=torch.bfloat16)
        if n > 0:
            kv[:, :, :, :n, :] = torch.randn((L, 2, Hkv, n, D), generator=gen).to(torch.bfloat16)
        return kv, None
    if kind == "fp8":
        codes = torch.zeros((L, 2, Hkv, max_ctx, D), dtype=torch.uint8)
        scales = torch.zeros((L, 2, Hkv, max_ctx), dtype=torch.float32)
        if n > 0:
            z = (torch.randn((L, 2, Hkv, n, D), generator=gen) * 32.0).to(torch.float8_e4m3fn)
            codes[:, :, :, :n, :] = z.view(torch.uint8)
            scales[:, :, :, :n] = 0.02 + 0.02 * torch.rand((L, 2, Hkv, n), generator=gen)
        return codes, scales
    raise ValueError(kind)


def tokens(vocab: int, batch: int, seed: int) -> torch.Tensor:
    """Start tokens uniform in [0, vocab), int32 [batch]."""
    gen = torch.Generator().manual_seed(int(seed))
    return torch.randint(0, vocab, (batch,), generator=gen, dtype=torch.int64).to(torch.int32)


def ragged_lengths(lo: int, hi: int, batch: int, seed: int) -> List[int]:
    """Per-sequence lengths uniform in [lo, hi] (inclusive)."""
    gen = torch.Generator().manual_seed(int(seed))
    return [int(v) for v in torch.randint(lo, hi + 1, (batch,), generator=gen)]


def attention_inputs(batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                     max_len: int, lengths: Sequence[int], seed: int):
    """Isolated decode-attention operands: q [B, Hq, D] bf16 ~N(0,1) and a cache
    [B, Hkv, max_len, D] for K and V each, rows < lengths[b] ~N(0,1) bf16."""
    gen = torch.Generator().manual_seed(int(seed))
    q = torch.randn((batch, n_q_heads, head_dim), generator=gen).to(torch.bfloat16)
    k = torch.zeros((batch, n_kv_heads, max_len, head_dim), dtype=torch.bfloat16)
    v = torch.zeros_like(k)
    for b, n in enumerate(lengths):
        if n > 0:
            k[b, :, :n] = torch.randn((n_kv_heads, n, head_dim), generator=gen).to(torch.bfloat16)
            v[b, :, :n] = torch.randn((n_kv_heads, n, head_dim), generator=gen).to(torch.bfloat16)
    return q, k, v


def bits16(t: torch.Tensor):
    """The raw 16-bit patterns of a bf16 tensor as a numpy uint16 array."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")
