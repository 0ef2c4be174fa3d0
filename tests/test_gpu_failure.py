"""Failure detection on the GPU without a fault: a bounded device wait is made
to run out (one CTA withholds its share of an activation, so every other CTA's
wait on it times out).  The step must report DEC_DEV_TIMEOUT, emit -1, drain
and return; the context must stay usable for the next step."""
import numpy as np
import pytest
import torch

import oracle
from conftest import oracle_cache, oracle_shape, oracle_weights
from decoder_greedy_decode_b200 import capi, synth
from decoder_greedy_decode_b200.decoder import Decoder, to_device
from gpu_util import assert_close, i32

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    s = synth.TINY
    w = synth.model_weights(s, seed=61)
    kv_host, _ = synth.kv_prefill(s, 1, 64, [20], seed=62)
    dec = Decoder(s, to_device(w), 1)
    kv = dec.kv_cache(1, 64)
    kv.values.copy_(kv_host.cuda())
    dec.set_timeout_ns(50_000_000)                 # 50 ms
    dec.set_debug_stall(5)                         # CTA 4 withholds its o_proj rows of layer 0
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    dec.step(kv, i32([7]), i32([20]), out)
    assert dec.check() == capi.DEC_DEV_TIMEOUT
    assert int(out[0]) == -1
    # the same step again without the stall: same context, correct result (it
    # rewrites row 20, which the aborted step may have written in part)
    dec.set_debug_stall(0)
    m = oracle.Model(oracle_shape(s), oracle_weights(w))
    cache = oracle_cache(kv_host, None, 0)
    r = m.step(cache, 7, 20)
    logits = torch.zeros((1, s.vocab), dtype=torch.float32, device="cuda")
    dec.step(kv, i32([7]), i32([20]), out, logits)
    assert dec.check() == 0
    assert_close(logits.cpu().numpy()[0], r.logits, "after timeout")
    dec.close()
