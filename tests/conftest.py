"""Shared test plumbing: the `gpu` marker and converters from the seeded
synthetic inputs to the oracle's numpy views."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def oracle_weights(w):
    """synth.model_weights(...) -> oracle.Weights of uint16 bf16 bits."""
    import oracle
    from decoder_greedy_decode_b200.synth import bits16
    layers = [{k: bits16(t) for k, t in lw.items()} for lw in w["layers"]]
    return oracle.Weights(embed=bits16(w["embed"]), lm_head=bits16(w["lm_head"]),
                          final_norm=bits16(w["final_norm"]), layers=layers)


def oracle_shape(s):
    import oracle
    return oracle.Shape(s.n_layers, s.hidden, s.n_q_heads, s.n_kv_heads, s.head_dim,
                        s.ffn, s.vocab, s.rms_eps, s.rope_theta)


def oracle_cache(kv, scales, b):
    """Sequence b of a [L,2,B,Hkv,max_ctx,D] cache as an oracle.Cache (a copy)."""
    import oracle
    from decoder_greedy_decode_b200.synth import bits16
    if scales is None:
        a = np.ascontiguousarray(bits16(kv[:, :, b]))
        return oracle.Cache("bf16", a)
    codes = np.ascontiguousarray(kv[:, :, b].numpy())
    sc = np.ascontiguousarray(scales[:, :, b].numpy())
    return oracle.Cache("fp8", codes, sc)
