"""Run decode steps of a seeded synthetic decoder for profiling (ncu) and
quick timing.

    python -m decoder_greedy_decode_b200.profile_step --layers 2 --batch 64 \
        --ctx 200,420 --steps 2

Weights have the 0.6B (default) or 1.7B widths with --layers layers; every
sequence's cache holds N(0,1) rows up to a context drawn in [lo, hi]; the
steps feed their own ids back.  --weights int8 / fp8 quantises every projection
and lm_head per row (dec_quantize_int8 / dec_quantize_fp8w) and runs the
weight-only 8-bit step.  Prints the device time per step of the --steps steps that
follow --warmup untimed ones."""
from __future__ import annotations

import argparse

import torch

from . import synth
from .decoder import Decoder, quantize_int8, to_device


def main() -> None:
    p = argparse.ArgumentParser()
    p.add_argument("--shape", choices=["0.6b", "1.7b"], default="0.6b")
    p.add_argument("--layers", type=int, default=28)
    p.add_argument("--batch", type=int, default=64)
    p.add_argument("--ctx", default="200,420")
    p.add_argument("--steps", type=int, default=2)
    p.add_argument("--warmup", type=int, default=0)
    p.add_argument("--kv", choices=["bf16", "fp8"], default="bf16")
    p.add_argument("--weights", choices=["bf16", "int8", "fp8"], default="bf16")
    a = p.parse_args()
    base = synth.QWEN3_0_6B if a.shape == "0.6b" else synth.QWEN3_1_7B
    s = synth.ModelShape(a.layers, base.hidden, base.n_q_heads, base.n_kv_heads, base.head_dim,
                         base.ffn, base.vocab)
    lo, hi = (int(x) for x in a.ctx.split(","))
    w = to_device(synth.model_weights(s, seed=2))
    if a.weights in ("int8", "fp8"):
        w = quantize_int8(w, kind=a.weights)
    dec = Decoder(s, w, max_batch=a.batch)
    max_ctx = (hi + a.warmup + a.steps + 15) // 16 * 16
    kv = dec.kv_cache(a.batch, max_ctx, a.kv)
    g = torch.Generator(device="cuda").manual_seed(1)
    if a.kv == "bf16":
        kv.values.normal_(generator=g)
    else:
        z = torch.randn(kv.codes.shape, generator=g, device="cuda") * 32.0
        kv.codes.copy_(z.to(torch.float8_e4m3fn).view(torch.uint8))
        kv.scales.uniform_(0.02, 0.04, generator=g)
    lengths = synth.ragged_lengths(lo, hi, a.batch, seed=3)
    base_pos = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    tok = torch.randint(0, s.vocab, (a.batch,), generator=g, dtype=torch.int32, device="cuda")
    for i in range(a.warmup):
        dec.step(kv, tok, base_pos + i, tok)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for i in range(a.steps):
        dec.step(kv, tok, base_pos + a.warmup + i, tok)
    e1.record()
    torch.cuda.synchronize()
    st = dec.check()
    if st != 0:
        raise SystemExit(f"device status {st}")
    print(f"{a.steps} steps, batch {a.batch}, {a.layers} layers, {a.weights} weights: "
          f"{e0.elapsed_time(e1) / a.steps * 1e3:.1f} us/step")
    dec.close()


if __name__ == "__main__":
    main()
