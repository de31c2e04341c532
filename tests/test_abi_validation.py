"""Host-side argument checks of every entry point, on the CPU: each call below
is rejected before anything is launched (so no device is needed), with the
status the header documents for it."""
import ctypes
import math
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

OK, INVALID, UNSUPPORTED, WORKSPACE, CAPACITY, CUDA = range(6)


@pytest.fixture(scope="module")
def lib():
    from hybrid_precision_attention_b200 import build
    h = ctypes.CDLL(build.build())
    from hybrid_precision_attention_b200.hq import HqCacheStruct
    P, I, S, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
    CP = ctypes.POINTER(HqCacheStruct)
    for name, args in (("hq_select_vlines", [CP, P, I, P, I, P, P, S, P]),
                       ("hq_pack_merge", [CP, P, P, I, P, S, P]),
                       ("hq_decode_attn", [CP, P, P, P, P, F, P, S, P]),
                       ("hq_prefill_attn", [I, I, I, I, I, P, P, P, P, I, I, I, I, F, P, P, S, P]),
                       ("hq_prefill_workspace_bytes", [I, I, I, I, I, I]),
                       ("hq_workspace_bytes", [CP, I, I]),
                       ("hq_status_str", [I]),
                       ("hq_last_error", [])):
        getattr(h, name).argtypes = args
    for name in ("hq_select_vlines", "hq_pack_merge", "hq_decode_attn", "hq_prefill_attn"):
        getattr(h, name).restype = I
    h.hq_prefill_workspace_bytes.restype = S
    h.hq_workspace_bytes.restype = S
    h.hq_status_str.restype = ctypes.c_char_p
    h.hq_last_error.restype = ctypes.c_char_p
    h.Cache = HqCacheStruct
    return h


@pytest.fixture(scope="module")
def mem():
    buf = ctypes.create_string_buffer(1 << 16)
    base = (ctypes.addressof(buf) + 255) & ~255
    return buf, base


def _cache(lib, base, **kw):
    c = lib.Cache(1, 32, 8, 128, 128, 500, 1024, 64, *([base] * 9))
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_select_rejections(lib, mem):
    _, a = mem
    c = _cache(lib, a)
    ws_need = lib.hq_workspace_bytes(ctypes.byref(c), 0, 0)
    assert ws_need > 0
    sel = lambda *args: lib.hq_select_vlines(ctypes.byref(c), *args)
    assert sel(a + 4, 512, a, 64, None, a, ws_need, None) == INVALID       # misaligned dense K
    assert sel(a, 512, a, 0, None, a, ws_need, None) == INVALID           # no queries
    assert sel(a, 512, a, 65, None, a, ws_need, None) == INVALID          # more than the query buffer
    assert sel(a, 32, a, 64, None, a, ws_need, None) == INVALID           # more queries than positions
    assert sel(a, 2048, a, 64, None, a, ws_need, None) == CAPACITY        # prefix longer than cap
    assert sel(None, 0, a, 64, None, a, ws_need, None) == INVALID         # external queries in decode mode
    assert sel(None, 0, None, 0, a + 8, a, ws_need, None) == INVALID      # misaligned scores
    assert sel(None, 0, None, 0, None, None, ws_need, None) == WORKSPACE  # no workspace
    assert sel(None, 0, None, 0, None, a, ws_need - 1, None) == WORKSPACE # workspace too small


def test_pack_merge_rejections(lib, mem):
    _, a = mem
    c = _cache(lib, a)
    need = lib.hq_workspace_bytes(ctypes.byref(c), 1, 0)
    pm = lambda *args: lib.hq_pack_merge(ctypes.byref(c), *args)
    assert pm(a, None, 512, a, need, None) == INVALID       # K without V
    assert pm(a, a, 0, a, need, None) == INVALID            # empty prefix
    assert pm(a, a, 4096, a, need, None) == CAPACITY        # prefix longer than cap
    assert pm(None, None, 0, a, need - 1, None) == WORKSPACE


def test_decode_rejections(lib, mem):
    _, a = mem
    c = _cache(lib, a)
    need = lib.hq_workspace_bytes(ctypes.byref(c), 2, 0)
    assert need > 0
    dec = lambda *args: lib.hq_decode_attn(ctypes.byref(c), *args)
    s = 1 / math.sqrt(128)
    assert dec(a + 2, a, a, a, s, a, need, None) == INVALID      # misaligned q
    assert dec(a, a, a, None, s, a, need, None) == INVALID       # no output
    assert dec(a, a, a, a, 0.0, a, need, None) == INVALID        # scale not positive
    assert dec(a, a, a, a, float("nan"), a, need, None) == INVALID
    assert dec(a, a, a, a, s, a, need - 1, None) == WORKSPACE
    bad = _cache(lib, a, Hq=72)                                   # GQA 9 > HQ_MAX_GQA
    assert lib.hq_decode_attn(ctypes.byref(bad), a, a, a, a, s, a, need, None) == UNSUPPORTED


def test_prefill_rejections(lib, mem):
    _, a = mem
    need = lib.hq_prefill_workspace_bytes(1, 32, 8, 1000, 128, 64)
    assert need > 0
    # the gathered vertical-line rows are sized by the row stride, not by L
    assert lib.hq_prefill_workspace_bytes(1, 32, 8, 1000, 128, 1000) > need
    assert lib.hq_prefill_workspace_bytes(1, 32, 8, 1000, 128, -1) == 0
    assert lib.hq_prefill_workspace_bytes(1, 32, 8, 1000, 64, 64) == 0
    assert lib.hq_prefill_workspace_bytes(1, 30, 8, 1000, 128, 64) == 0
    s = 1 / math.sqrt(128)
    pf = lambda B, Hq, Hkv, L, D, n_vl, stride, W, sc, ws, wsb, vl=a, q=a, fmt=0: lib.hq_prefill_attn(
        B, Hq, Hkv, L, D, q, a, a, vl, n_vl, stride, W, fmt, sc, a, ws, wsb, None)
    assert pf(1, 32, 8, 1000, 64, 0, 0, 128, s, a, need) == UNSUPPORTED   # head size
    assert pf(1, 30, 8, 1000, 128, 0, 0, 128, s, a, need) == INVALID      # Hq not a multiple of Hkv
    assert pf(1, 32, 8, 0, 128, 0, 0, 128, s, a, need) == INVALID         # empty prompt
    assert pf(1, 32, 8, 1000, 128, 0, 0, -1, s, a, need) == INVALID       # negative window
    assert pf(1, 32, 8, 1000, 128, 0, 0, 128, -s, a, need) == INVALID     # negative scale
    assert pf(1, 32, 8, 1000, 128, 10, 8, 128, s, a, need) == INVALID     # more lines than the row stride
    assert pf(1, 32, 8, 1000, 128, 10, 16, 128, s, a, need, vl=None) == INVALID  # lines without positions
    assert pf(1, 32, 8, 1000, 128, 0, 0, 128, s, a, need, q=a + 4) == INVALID    # misaligned Q
    assert pf(1, 32, 8, 1000, 128, 0, 0, 128, s, a, need - 1) == WORKSPACE
    assert pf(1, 32, 8, 1000, 128, 0, 0, 128, s, a, need, fmt=2) == INVALID         # unknown Q.K format


def test_status_strings(lib):
    names = [lib.hq_status_str(i) for i in range(6)]
    assert names[0] == b"ok" and len(set(names)) == 6
    assert lib.hq_status_str(99) == b"unknown status"
    assert isinstance(lib.hq_last_error(), bytes)  # a C string, empty until a CUDA step fails on this thread
