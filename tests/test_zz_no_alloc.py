"""The allocation-free decode entry point, checked against the workspace one.

hq_decode_attn_noalloc is for callers that may not allocate device memory,
such as a plugin inside a serving engine that owns all device memory, or a
latency-critical loop where cudaMalloc / cudaFree would synchronise the
device; it keeps its scratch in a fixed array inside the library.  Through the
C ABI, two decode steps in a row must give the same output as hq_decode_attn
on an identical cache, within the decode tolerance the other GPU tests use.
This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from hybrid_precision_attention_b200 import synth
from tests._gpu import DEC_MAXABS, DEC_RELL2, dev, hq

pytestmark = pytest.mark.gpu


def _prefilled_cache(lay, L):
    H = hq()
    c = H.HybridCache(1, 32, 8, L + 256, 128, 500)
    H.hq_select_vlines(c, dev(lay.k), dev(lay.q_tail))
    H.hq_pack_merge(c, dev(lay.k), dev(lay.v))
    return c


def test_noalloc_decode_matches_workspace_decode():
    H = hq()
    L = 4096
    lay = synth.planted_layer(21, 1, 32, 8, L)
    ref_cache = _prefilled_cache(lay, L)
    na_cache = _prefilled_cache(lay, L)
    q, k, v = synth.decode_tokens(21, 1, 32, 8, 2)
    for t in range(2):   # two calls in a row: the shared scratch must not carry anything over
        want = H.hq_decode_attn(ref_cache, dev(q[t]), dev(k[t]), dev(v[t]))
        got = H.hq_decode_attn_noalloc(na_cache, dev(q[t]), dev(k[t]), dev(v[t]))
        torch.cuda.synchronize()
        a = want.float().cpu().numpy().astype(np.float64)
        b = got.float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(b))
        assert np.abs(a - b).max() <= DEC_MAXABS
        assert np.linalg.norm(a - b) / np.linalg.norm(a) <= DEC_RELL2
        for c in (ref_cache, na_cache):
            st = c.state()
            assert st["err"] == 0 and st["T"] == L + t + 1, st


def test_noalloc_rejections_and_a_large_then_small_cache():
    """Host-side rejections (nothing launched, state untouched), a cache whose
    decode workspace exceeds the fixed array, then a small cache after a large
    one on the shared array, still equal to the workspace path."""
    import ctypes
    import math
    H = hq()
    lib = H._lib
    s = 1 / math.sqrt(128)
    L = 1024
    lay = synth.planted_layer(22, 1, 32, 8, L)
    small = _prefilled_cache(lay, L)
    ref = _prefilled_cache(lay, L)
    q, k, v = synth.decode_tokens(22, 1, 32, 8, 3)
    qd, kd, vd = dev(q[0]), dev(k[0]), dev(v[0])
    out = torch.empty_like(qd)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    call = lambda c, qq, sc, oo=out: lib.hq_decode_attn_noalloc(ctypes.byref(c.c), qq, P(kd), P(vd), oo, ctypes.c_float(sc),
                                                                  H._stream(None))
    assert call(small, ctypes.c_void_p(qd.data_ptr() + 2), s, P(out)) == 1      # misaligned q: HQ_ERR_INVALID
    assert call(small, P(qd), s, None) == 1                                      # no output
    assert call(small, P(qd), 0.0, P(out)) == 1                                  # scale not positive
    assert call(small, P(qd), float("nan"), P(out)) == 1
    # a cache whose decode workspace exceeds the array: B * Hkv = 1024 units of split partials
    big = H.HybridCache(128, 64, 8, 128, 128, 500)
    assert H._lib.hq_workspace_bytes(ctypes.byref(big.c), H.OP_DECODE, 0) > 4 << 20
    qb = torch.zeros((128, 64, 128), dtype=torch.float16, device="cuda")
    kb = torch.zeros((128, 8, 128), dtype=torch.float16, device="cuda")
    ob = torch.empty_like(qb)
    st = lib.hq_decode_attn_noalloc(ctypes.byref(big.c), P(qb), P(kb), P(kb), P(ob), ctypes.c_float(s), H._stream(None))
    assert st == 3                                                               # HQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert big.state()["T"] == 0 and small.state()["T"] == L and small.state()["err"] == 0
    # a large cache that fits (more splits and units than the small one), then the small one again
    mid = _prefilled_cache(synth.planted_layer(23, 1, 32, 8, 4096), 4096)
    qm, km, vm = synth.decode_tokens(23, 1, 32, 8, 1)
    H.hq_decode_attn_noalloc(mid, dev(qm[0]), dev(km[0]), dev(vm[0]))
    for t in range(3):
        want = H.hq_decode_attn(ref, dev(q[t]), dev(k[t]), dev(v[t]))
        got = H.hq_decode_attn_noalloc(small, dev(q[t]), dev(k[t]), dev(v[t]))
        torch.cuda.synchronize()
        a = want.float().cpu().numpy().astype(np.float64)
        b = got.float().cpu().numpy().astype(np.float64)
        assert np.abs(a - b).max() <= DEC_MAXABS
        assert np.linalg.norm(a - b) / np.linalg.norm(a) <= DEC_RELL2
    assert small.state()["T"] == L + 3 and small.state()["err"] == 0 and mid.state()["T"] == 4097
