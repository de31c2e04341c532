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
