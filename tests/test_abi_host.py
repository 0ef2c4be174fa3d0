"""The C-ABI library without a GPU: it loads, exports every symbol the header
declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

from decoder_greedy_decode_b200 import capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "dec.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(dec_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_binding_exports():
    assert _declared() == sorted(capi.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = capi.lib()
    for name in _declared():
        assert hasattr(L, name), name


def test_shape_validation_happens_on_host():
    bad = capi.dec_shape(28, 1000, 16, 8, 128, 3072, 151936, 1e-6, 1e6, 1)   # hidden % 256
    h = ctypes.c_void_p()
    w = capi.dec_weights(1, 1, 1, None)
    rc = capi.lib().dec_init(ctypes.byref(bad), ctypes.byref(w), ctypes.byref(h))
    assert rc == -2 and not h.value
    bad = capi.dec_shape(28, 1024, 16, 6, 128, 3072, 151936, 1e-6, 1e6, 1)    # 16 % 6
    assert capi.lib().dec_init(ctypes.byref(bad), ctypes.byref(w), ctypes.byref(h)) == -2
    bad = capi.dec_shape(28, 1024, 16, 8, 96, 3072, 151936, 1e-6, 1e6, 1)     # head_dim 96
    assert capi.lib().dec_init(ctypes.byref(bad), ctypes.byref(w), ctypes.byref(h)) == -2
    bad = capi.dec_shape(28, 1024, 16, 8, 128, 3072, 151936, 1e-6, 1e6, 0)    # batch 0
    assert capi.lib().dec_init(ctypes.byref(bad), ctypes.byref(w), ctypes.byref(h)) == -3


def test_null_arguments():
    L = capi.lib()
    assert L.dec_step(None, 1, None, None, None, None, None, None) == -1
    assert L.dec_check(None, None) == -1
    assert L.dec_kv_bytes(None, 1, 64, 0) == 0
    assert L.dec_attention(1, 16, 8, 128, None, None, None, 64, None, None, None, 0, None, None) == -1
    assert L.dec_attention_workspace_bytes(1, 16, 6, 128, 64) == 0
    assert L.dec_kv_quantize_e4m3(None, 1, 128, None, None, None) == -1


def test_attention_rejects_no_query_heads():
    """n_q_heads < 1 is a shape error in both attention entry points, decided on
    the host before any CUDA call (the pointers are fake and never read)."""
    L = capi.lib()
    p = 1 << 20
    for hq in (0, -8):
        assert L.dec_attention_workspace_bytes(1, hq, 8, 128, 64) == 0
        assert L.dec_attention(1, hq, 8, 128, p, p, p, 64, p, p, p, 1 << 20, None, None) == -2
        assert L.dec_attention_noalloc(1, hq, 8, 128, p, p, p, 64, p, p, None, None) == -2


def test_error_strings():
    assert capi.error_string(0) == "ok"
    assert "NULL" in capi.error_string(-1)
    s = capi.error_string(capi.DEC_DEV_TIMEOUT | capi.DEC_DEV_BAD_TOKEN)
    assert "token" in s and "wait" in s


def _int8_weights(L, aligned=True, null_scale_at=None, norm_scale_null=True):
    """A dec_weights_int8 of fake device addresses (never dereferenced: the
    checks under test run on the host before any CUDA call)."""
    base = 1 << 20
    ptrs = [base + 256 * i + (0 if aligned else 4) for i in range(L * len(capi.LW_ORDER))]
    scales = []
    for i in range(L * len(capi.LW_ORDER)):
        key = capi.LW_ORDER[i % len(capi.LW_ORDER)]
        p = (1 << 24) + 64 * i if key in capi.PROJ_KEYS else (None if norm_scale_null else 1 << 26)
        scales.append(None if i == null_scale_at else p)
    arr = (ctypes.c_void_p * len(ptrs))(*ptrs)
    sarr = (ctypes.c_void_p * len(scales))(*scales)
    w = capi.dec_weights_int8(1 << 28, 1 << 29, 1 << 30, 1 << 27,
                              ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)),
                              ctypes.cast(sarr, ctypes.POINTER(ctypes.c_void_p)))
    return w, (arr, sarr)


@pytest.mark.parametrize("entry", ["dec_init_int8", "dec_init_fp8w"])
def test_8bit_init_checks_on_host(entry):
    """dec_init_int8 / dec_init_fp8w: shape first, then max_batch <= 64, NULL
    pointers (a projection's scale array is required, a norm slot's is not),
    alignment."""
    init = getattr(capi.lib(), entry)
    h = ctypes.c_void_p()
    ok_shape = capi.dec_shape(2, 256, 4, 2, 64, 768, 4096, 1e-6, 1e6, 1)
    w, keep = _int8_weights(2)
    bad = capi.dec_shape(2, 200, 4, 2, 64, 768, 4096, 1e-6, 1e6, 1)
    assert init(ctypes.byref(bad), ctypes.byref(w), ctypes.byref(h)) == -2
    big = capi.dec_shape(2, 256, 4, 2, 64, 768, 4096, 1e-6, 1e6, 65)
    assert init(ctypes.byref(big), ctypes.byref(w), ctypes.byref(h)) == -3
    q_of_layer1 = len(capi.LW_ORDER) + capi.LW_ORDER.index("q")
    w2, keep2 = _int8_weights(2, null_scale_at=q_of_layer1)
    assert init(ctypes.byref(ok_shape), ctypes.byref(w2), ctypes.byref(h)) == -1
    w3, keep3 = _int8_weights(2, aligned=False)
    assert init(ctypes.byref(ok_shape), ctypes.byref(w3), ctypes.byref(h)) == -6
    w4 = capi.dec_weights_int8(1 << 28, 1 << 29, None, 1 << 27, w.layers, w.scales)
    assert init(ctypes.byref(ok_shape), ctypes.byref(w4), ctypes.byref(h)) == -1
    w5 = capi.dec_weights_int8(1 << 28, 1 << 29, (1 << 30) + 2, 1 << 27, w.layers, w.scales)
    assert init(ctypes.byref(ok_shape), ctypes.byref(w5), ctypes.byref(h)) == -6
    assert not h.value


@pytest.mark.parametrize("entry", ["dec_quantize_int8", "dec_quantize_fp8w"])
def test_8bit_quantizer_checks_on_host(entry):
    q = getattr(capi.lib(), entry)
    assert q(None, 4, 16, 1 << 20, 1 << 21, None) == -1
    assert q(1 << 20, 4, 20, 1 << 21, 1 << 22, None) == -9    # cols % 8
    assert q(1 << 20, -1, 16, 1 << 21, 1 << 22, None) == -9
    assert q((1 << 20) + 8, 4, 16, 1 << 21, 1 << 22, None) == -6  # w 16 B
    assert q(1 << 20, 4, 16, (1 << 21) + 4, 1 << 22, None) == -6  # codes 8 B
    assert q(1 << 20, 0, 16, 1 << 21, 1 << 22, None) == 0      # no rows: no-op
