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
    return oracle.weights_from(w)


def oracle_shape(s):
    import oracle
    return oracle.shape_from(s)


def oracle_cache(kv, scales, b):
    """Sequence b of a [L,2,B,Hkv,max_ctx,D] cache as an oracle.Cache (a copy)."""
    import oracle
    return oracle.cache_from(kv, scales, b)
