"""Algorithmic byte counts of one decode step (the roofline numerators).

Per step the decoder must read every weight once, read the KV rows already
in the cache and write the new row, and read one embedding row per sequence.
Weights dominate at batch 1; the KV cache dominates at high concurrency
("Qwen3-ASR -- Latency & Bottleneck Analysis", 06 Bottleneck ranking: MLP
529MB/token and lm_head 311MB/token are memory-bound; Baseten Qwen3-ASR
article, KV cache quantization: decode attention reads the whole cache every
step)."""
from __future__ import annotations

from typing import Iterable, Sequence

BF16 = 2


def layer_weight_params(s) -> int:
    nq, nkv = s.n_q_heads * s.head_dim, s.n_kv_heads * s.head_dim
    qkv = (nq + 2 * nkv) * s.hidden
    o = s.hidden * nq
    mlp = 3 * s.hidden * s.ffn
    norms = 2 * s.hidden + 2 * s.head_dim
    return qkv + o + mlp + norms


def mlp_bytes_per_token(s) -> int:
    """Gate, up and down projections of every layer (bf16)."""
    return s.n_layers * 3 * s.hidden * s.ffn * BF16


def lm_head_bytes(s) -> int:
    return s.vocab * s.hidden * BF16


def projection_rows(s) -> int:
    """Output rows of one layer's seven projections (q, k, v, o, gate, up, down)."""
    nq, nkv = s.n_q_heads * s.head_dim, s.n_kv_heads * s.head_dim
    return nq + 2 * nkv + s.hidden + 2 * s.ffn + s.hidden


def weight_bytes(s, weights: str = "bf16") -> int:
    """Every weight the step reads once: layers + lm_head + final norm.

    weights "int8" / "fp8": the projections and lm_head as 8-bit codes (1
    byte each) plus one fp32 scale per output row; norm gains stay bf16."""
    if weights == "bf16":
        return (s.n_layers * layer_weight_params(s) + s.vocab * s.hidden + s.hidden) * BF16
    assert weights in ("int8", "fp8")
    norms = 2 * s.hidden + 2 * s.head_dim
    proj = layer_weight_params(s) - norms
    per_layer = proj + 4 * projection_rows(s) + norms * BF16
    return s.n_layers * per_layer + s.vocab * s.hidden + 4 * s.vocab + s.hidden * BF16


def kv_bytes_per_token(s, kind: str = "bf16") -> int:
    """Bytes one cached token occupies over all layers, K and V."""
    per_head = s.head_dim * BF16 if kind == "bf16" else s.head_dim + 4   # fp8 codes + fp32 scale
    return s.n_layers * 2 * s.n_kv_heads * per_head


def step_bytes(s, positions: Iterable[int], kind: str = "bf16", weights: str = "bf16") -> int:
    """Algorithmic bytes of one step: weights + for every sequence b the KV
    rows 0..p_b-1 read, row p_b written, and its embedding row."""
    positions = list(positions)
    kv = sum((int(p) + 1) * kv_bytes_per_token(s, kind) for p in positions)
    return weight_bytes(s, weights) + kv + len(positions) * s.hidden * BF16


def attention_bytes(lengths: Sequence[int], n_kv_heads: int, head_dim: int,
                    n_q_heads: int) -> int:
    """Isolated decode attention: K and V rows of every (sequence, KV head)
    read once (bf16), q read (bf16) and the output written (fp32)."""
    kv = sum(int(n) for n in lengths) * n_kv_heads * 2 * head_dim * BF16
    b = len(lengths)
    return kv + b * n_q_heads * head_dim * (BF16 + 4)


def step_flops(s, positions: Sequence[int]) -> int:
    """2 x multiply-adds of the projections, the lm_head and attention."""
    per_tok = 2 * (s.n_layers * (layer_weight_params(s) - 2 * s.hidden - 2 * s.head_dim)
                   + s.vocab * s.hidden)
    att = sum(2 * 2 * s.n_layers * s.n_q_heads * s.head_dim * (int(p) + 1) for p in positions)
    return per_tok * len(positions) + att
