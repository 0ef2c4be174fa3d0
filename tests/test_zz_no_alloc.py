"""dec_attention_noalloc: the attention entry point that allocates nothing.

It serves callers that must not allocate device memory on their call path
(another framework's execute callback, real-time loops, memory owned by
another allocator): its scratch is a fixed device array inside the library.
Its output must match the workspace entry point's, call after call, and a
request larger than that array must be refused without launching."""
import numpy as np
import pytest
import torch

from decoder_greedy_decode_b200 import capi, synth
from gpu_util import assert_close, i32

pytestmark = pytest.mark.gpu


def _inputs(B, L, seed):
    lengths = synth.ragged_lengths(L // 2, L, B, seed=seed)
    q, k, v = synth.attention_inputs(B, 16, 8, 128, L, lengths, seed=seed + 1)
    return lengths, q.cuda(), k.cuda(), v.cuda()


def _with_workspace(B, L, lengths, q, k, v):
    out = torch.full((B, 16, 128), float("nan"), dtype=torch.float32, device="cuda")
    nb = capi.dec_attention_workspace_bytes(B, 16, 8, 128, L)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    capi.dec_attention(B, 16, 8, 128, q, k, v, L, i32(lengths), out, ws, nb, st)
    torch.cuda.synchronize()
    assert int(st[0]) == 0
    return out


def _no_alloc(B, L, lengths, q, k, v):
    out = torch.full((B, 16, 128), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    capi.dec_attention_noalloc(B, 16, 8, 128, q, k, v, L, i32(lengths), out, st)
    torch.cuda.synchronize()
    assert int(st[0]) == 0
    return out


def test_no_alloc_attention_matches_workspace_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    for B, L, seed in ((8, 795, 3), (4, 4096, 7)):      # two calls in a row, different sizes
        lengths, q, k, v = _inputs(B, L, seed)
        ref = _with_workspace(B, L, lengths, q, k, v)
        got = _no_alloc(B, L, lengths, q, k, v)
        assert torch.isfinite(got).all()
        assert_close(got.cpu().numpy(), ref.cpu().numpy(), f"no-alloc B={B} L={L}")


def test_no_alloc_attention_refuses_requests_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B, L = 64, 32768
    q = torch.zeros((B, 16, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((1,), dtype=torch.bfloat16, device="cuda")    # never read: refused first
    out = torch.zeros((B, 16, 128), dtype=torch.float32, device="cuda")
    rc = capi.lib().dec_attention_noalloc(B, 16, 8, 128, q.data_ptr(), kv.data_ptr(), kv.data_ptr(),
                                          L, i32([L] * B).data_ptr(), out.data_ptr(), None,
                                          int(torch.cuda.current_stream().cuda_stream))
    assert rc == capi.DEC_ERR_TOO_LARGE
    assert "fixed scratch" in capi.error_string(rc)
    assert torch.count_nonzero(out) == 0
