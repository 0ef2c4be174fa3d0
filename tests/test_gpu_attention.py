"""Parity of the isolated split-K GQA decode attention and of the E4M3 row
quantiser against the CPU oracle.

Workload: 16 query heads / 8 KV heads of 128, bf16 Q/K/V ~N(0,1), contexts
L in {128, 795, 4096, 16384, 32768} x batch {1, 8, 64}, per-sequence lengths
uniform in [L/2, L] ("Qwen3-ASR -- Latency & Bottleneck Analysis", 07 Root
causes: 16 x 128 x ~925 decode attention; Baseten Qwen3-ASR article: 64
concurrent sequences, attention over the whole cache every step)."""
import numpy as np
import pytest
import torch

import oracle
from decoder_greedy_decode_b200 import capi, synth
from gpu_util import assert_close, i32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    capi.lib()


def _bits(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _run(B, Hq, Hkv, D, L, lengths, q, k, v):
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    nb = capi.dec_attention_workspace_bytes(B, Hq, Hkv, D, L)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    capi.dec_attention(B, Hq, Hkv, D, q, k, v, L, i32(lengths), out, ws, nb, st)
    torch.cuda.synchronize()
    assert int(st[0]) == 0
    return out, ws


def _check(B, Hq, Hkv, D, lengths, q, k, v, out, pairs):
    rep = Hq // Hkv
    qn = q.float().cpu().double().numpy()
    on = out.cpu().numpy()
    for b, h in pairs:
        g = h // rep
        ref = oracle.attend(qn[b, h], _bits(k[b, g]), _bits(v[b, g]), lengths[b])
        assert_close(on[b, h], ref, f"b={b} h={h} len={lengths[b]}")


# Every (L, B) cell of the measured grid.  Cells the oracle covers in a few
# seconds are compared on every (sequence, query head); the larger ones on
# sampled pairs that always include the first and last sequence and query
# head, the longest and the shortest sequence.
GRID_L = (128, 795, 4096, 16384, 32768)
GRID_B = (1, 8, 64)
FULL_ROWS = 1 << 19   # sum over compared pairs of the rows the oracle reads


@pytest.mark.parametrize("L", GRID_L)
@pytest.mark.parametrize("B", GRID_B)
def test_attention_grid_cell(L, B):
    Hq, Hkv, D = 16, 8, 128
    lengths = synth.ragged_lengths(L // 2, L, B, seed=L + B)
    g = torch.Generator(device="cuda").manual_seed(L * 7 + B)
    q = torch.randn((B, Hq, D), generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn((B, Hkv, L, D), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((B, Hkv, L, D), generator=g, device="cuda").to(torch.bfloat16)
    out, _ = _run(B, Hq, Hkv, D, L, lengths, q, k, v)
    assert torch.isfinite(out).all()
    if sum(lengths) * Hq <= FULL_ROWS:
        pairs = [(b, h) for b in range(B) for h in range(Hq)]
    else:
        rng = np.random.default_rng(L * 3 + B)
        bl, bs = int(np.argmax(lengths)), int(np.argmin(lengths))
        pairs = {(0, 0), (B - 1, Hq - 1), (bl, 1), (bs, Hq - 2)}
        pairs |= {(int(rng.integers(B)), int(rng.integers(Hq))) for _ in range(8)}
        pairs = sorted(pairs)
    _check(B, Hq, Hkv, D, lengths, q, k, v, out, pairs)
    # a second call on a fresh workspace gives the same bits
    out2, _ = _run(B, Hq, Hkv, D, L, lengths, q, k, v)
    assert torch.equal(out, out2)
    del k, v


def test_attention_other_shapes_and_edges():
    # head_dim 64, 4 query heads per KV head, lengths 1 and max
    B, Hq, Hkv, D, L = 3, 8, 2, 64, 200
    lengths = [1, 200, 77]
    q, k, v = synth.attention_inputs(B, Hq, Hkv, D, L, lengths, seed=99)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    out, _ = _run(B, Hq, Hkv, D, L, lengths, q, k, v)
    _check(B, Hq, Hkv, D, lengths, q, k, v, out, [(b, h) for b in range(B) for h in range(Hq)])
    # a single-row context returns V exactly
    vv = v[0, :, 0].float()
    for h in range(Hq):
        assert torch.equal(out[0, h], vv[h // (Hq // Hkv)])


def test_attention_bad_length_sets_status():
    B, Hq, Hkv, D, L = 2, 16, 8, 128, 64
    q, k, v = synth.attention_inputs(B, Hq, Hkv, D, L, [10, 10], seed=5)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    out = torch.zeros((B, Hq, D), dtype=torch.float32, device="cuda")
    nb = capi.dec_attention_workspace_bytes(B, Hq, Hkv, D, L)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    capi.dec_attention(B, Hq, Hkv, D, q, k, v, L, i32([10, 65]), out, ws, nb, st)
    torch.cuda.synchronize()
    assert int(st[0]) == capi.DEC_DEV_BAD_POSITION
    assert torch.count_nonzero(out[1]) == 0 and torch.isfinite(out[0]).all()


def test_quantize_e4m3_bit_exact_against_oracle():
    """Same fp32 inputs -> the same codes and scales, bit for bit: the integer
    decision is taken in fp32 on both sides."""
    rng = np.random.default_rng(0)
    rows = []
    rows.append(rng.standard_normal((200, 128)).astype(np.float32))
    rows.append((rng.standard_normal((20, 128)) * 1e-3).astype(np.float32))
    rows.append(np.zeros((2, 128), dtype=np.float32))
    # rows whose scaled values sit on E4M3 rounding midpoints
    mids = oracle.e4m3_decode(np.arange(0, 0x7E, dtype=np.uint8))
    mid = ((mids[:-1] + mids[1:]) / 2).astype(np.float32)
    r = np.zeros((1, 128), dtype=np.float32)
    r[0, :125] = mid[:125]
    r[0, 127] = 448.0
    rows.append(r)
    x = np.concatenate(rows)
    xd = torch.from_numpy(x).cuda()
    codes = torch.zeros(x.shape, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(x.shape[0], dtype=torch.float32, device="cuda")
    capi.dec_kv_quantize_e4m3(xd, x.shape[0], 128, codes, scales)
    torch.cuda.synchronize()
    c = codes.cpu().numpy()
    s = scales.cpu().numpy()
    for i in range(x.shape[0]):
        rc, rs = oracle.e4m3_quantize_row(x[i])
        assert np.float32(rs) == s[i], i
        assert np.array_equal(rc, c[i]), i
