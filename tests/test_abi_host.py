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


def test_error_strings():
    assert capi.error_string(0) == "ok"
    assert "NULL" in capi.error_string(-1)
    s = capi.error_string(capi.DEC_DEV_TIMEOUT | capi.DEC_DEV_BAD_TOKEN)
    assert "token" in s and "wait" in s
