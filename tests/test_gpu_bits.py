"""GPU parity of the other code widths of the decode cache (README Mode
reference: K8V8, K4V2, K2V4 beside K4V4), through the C ABI.

Each width runs the whole hot path against the oracle cache of the same width
(oracle.hybrid.HybridCacheRef with k_bits / v_bits): prefix install (the
selection, then the packed records bit-exact), decode steps within the decode
tolerances, a full 64-token period, reselection (scores and set) and merge
(records, VL rows and bitmap bit-exact), decode after the merge.  A per-layer
V width (the README's v_bits_fn) is a cache per layer with its own widths.
"""
import numpy as np
import pytest

from hybrid_precision_attention_b200 import synth
from tests._gpu import Pair, check_decode, dev, hq
from tests.test_gpu_varlen import Ragged

pytestmark = pytest.mark.gpu

WIDTHS = [(8, 8), (4, 2), (2, 4), (4, 4)]


@pytest.mark.parametrize("kb,vb", WIDTHS)
@pytest.mark.parametrize("B,Hq,Hkv,L,W", [
    (2, 8, 2, 1000, 100),      # ragged tiles, GQA 4
    (1, 32, 8, 4096, 128),     # Llama-3.1-8B attention shape
    (1, 16, 2, 333, 64),       # GQA 8, a partial last tile
])
def test_widths_period(kb, vb, B, Hq, Hkv, L, W):
    p = Pair(B, Hq, Hkv, L, W, 500, cap=L + 200, seed=L + kb * 10 + vb, k_bits=kb, v_bits=vb)
    p.init()
    q, k, v = synth.decode_tokens(L + kb, B, Hq, Hkv, 70)
    for t in range(64):
        if t % 9 == 0 or t == 63:
            out, ref = p.decode(q[t], k[t], v[t])
            check_decode(out, ref, f"K{kb}V{vb} step {t}")
        else:
            hq().hq_decode_attn(p.g, dev(q[t]), dev(k[t]), dev(v[t]))
            p.r.append(q[t], k[t], v[t])
    p.reselect_merge()
    for t in range(64, 67):
        out, ref = p.decode(q[t], k[t], v[t])
        check_decode(out, ref, f"K{kb}V{vb} after merge, step {t}")


@pytest.mark.slow
@pytest.mark.parametrize("kb,vb", [(8, 8), (4, 2), (2, 4)])
def test_widths_full_size_32k(kb, vb):
    """The 32K decode layer (B=1, Hq=32, Hkv=8) at each width: install, one step, a
    period with every 16th step checked, reselect + merge, one step."""
    B, Hq, Hkv, L, W = 1, 32, 8, 32768, 128
    p = Pair(B, Hq, Hkv, L, W, 500, cap=L + 128, seed=3, k_bits=kb, v_bits=vb)
    p.init()
    q, k, v = synth.decode_tokens(3, B, Hq, Hkv, 65)
    for t in range(64):
        if t % 16 == 0 or t == 63:
            out, ref = p.decode(q[t], k[t], v[t])
            check_decode(out, ref, f"K{kb}V{vb} step {t}")
        else:
            hq().hq_decode_attn(p.g, dev(q[t]), dev(k[t]), dev(v[t]))
            p.r.append(q[t], k[t], v[t])
    p.reselect_merge()
    out, ref = p.decode(q[64], k[64], v[64])
    check_decode(out, ref, f"K{kb}V{vb} after merge")


@pytest.mark.parametrize("kb,vb", [(8, 8), (2, 4), (4, 2)])
def test_widths_ragged_paged_batch(kb, vb):
    """Three sequences of 200, 700 and 1000 tokens (GQA 4, W = 64) in a shuffled
    page pool at each width (K8V8 pages hold two 32-position sub-pages): one
    install per sequence, a batched period, reselection and merge, three more
    steps, every sequence against its own oracle."""
    rg = Ragged([200, 700, 1000], 8, 2, 64, 500, cap=1300, seed=40 + kb + vb, k_bits=kb, v_bits=vb)
    for b in range(rg.B):
        rg.install(b)
        rg.check_store(b)
    q, k, v = synth.decode_tokens(41, rg.B, 8, 2, 67)
    for t in range(64):
        rg.decode(q[t], k[t], v[t], check=(t % 13 == 0 or t == 63))
    rg.reselect_merge()
    for t in range(64, 67):
        rg.decode(q[t], k[t], v[t])


@pytest.mark.parametrize("kb,vb", [(8, 8), (2, 4)])
def test_widths_running_scores(kb, vb):
    """Running column-mass scores at the other widths: two periods, the summed
    scores and the sets they choose against the oracle's running sums."""
    p = Pair(1, 8, 2, 900, 64, 500, cap=1200, seed=50 + kb, running=True, k_bits=kb, v_bits=vb)
    p.init()
    q, k, v = synth.decode_tokens(51, 1, 8, 2, 130)
    for period in range(2):
        for t in range(64 * period, 64 * period + 64):
            if t % 21 == 0:
                out, ref = p.decode(q[t], k[t], v[t])
                check_decode(out, ref, f"K{kb}V{vb} running, step {t}")
            else:
                hq().hq_decode_attn(p.g, dev(q[t]), dev(k[t]), dev(v[t]))
                p.r.append(q[t], k[t], v[t])
        p.reselect_merge()
    out, ref = p.decode(q[128], k[128], v[128])
    check_decode(out, ref, f"K{kb}V{vb} running, after two merges")


def test_widths_allocation_free_decode():
    """hq_decode_attn_noalloc on a K8V8 cache: the same step as the oracle's."""
    p = Pair(1, 32, 8, 2000, 128, 500, cap=2200, seed=60, k_bits=8, v_bits=8)
    p.init()
    q, k, v = synth.decode_tokens(61, 1, 32, 8, 3)
    H = hq()
    for t in range(3):
        out = H.hq_decode_attn_noalloc(p.g, dev(q[t]), dev(k[t]), dev(v[t]))
        ref = p.r.decode(q[t], k[t], v[t])
        st = p.g.state()
        assert st["err"] == 0 and st["T"] == p.r.T, st
        check_decode(out, ref, f"K8V8 allocation-free step {t}")
