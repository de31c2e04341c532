"""Pins for the oracle's hybrid-cache state machine, CPU only."""
import numpy as np
import pytest

from oracle import formats, hybrid, select
from hybrid_precision_attention_b200 import synth


def _cache(L=400, W=64, rho=500, B=2, Hq=4, Hkv=2, cap=600, seed=0):
    lay = synth.planted_layer(seed, B, Hq, Hkv, L)
    c = hybrid.HybridCacheRef(B, Hq, Hkv, W, rho, cap)
    vl, sc = c.init_from_prefix(lay.k, lay.v, lay.q_tail)
    return lay, c, vl, sc


def test_prefix_init_representation():
    lay, c, vl, _ = _cache()
    L, W = 400, 64
    assert c.T == L and c.n_packed == L - W
    for b in range(2):
        for h in range(2):
            assert len(vl[b][h]) == select.k_of(L - W, 500) and np.all(vl[b][h] < L - W)
            K, V = c.rep(b, h)
            # window rows and VL rows are the original FP16 values
            assert np.array_equal(K[L - W:], lay.k[b, h, L - W:].astype(np.float64))
            assert np.array_equal(K[vl[b][h]], lay.k[b, h, vl[b][h]].astype(np.float64))
            # every other row is its K4V4 dequantisation
            rest = np.setdiff1d(np.arange(L - W), vl[b][h])
            cc, s, z = formats.pack_k4v4(lay.v[b, h, rest])
            assert np.array_equal(V[rest], formats.dequant_k4v4(cc, s, z))


def test_staging_capacity_and_merge():
    lay, c, _, _ = _cache()
    qd, kd, vd = synth.decode_tokens(0, 2, 4, 2, 70)
    for t in range(64):
        c.decode(qd[t], kd[t], vd[t])
    with pytest.raises(RuntimeError):
        c.decode(qd[64], kd[64], vd[64])
    old_np = c.n_packed
    vl, sc = c.reselect()
    n = c.T - c.W
    assert all(len(vl[b][h]) == select.k_of(n, 500) for b in range(2) for h in range(2))
    c.merge(vl)
    assert c.n_packed == old_np + 64 == c.T - c.W
    # positions that left the window got the K4V4 record of their FP16 value
    # (here they are the prefix's last window, positions 336 .. 399)
    cc, s, z = formats.pack_k4v4(lay.k[0, 1, old_np:old_np + 64])
    assert old_np == 336 and np.array_equal(c.kq[0, 1, old_np:old_np + 64], cc)
    assert np.array_equal(c.ks[0, 1, old_np:old_np + 64], s) and np.array_equal(c.kz[0, 1, old_np:old_np + 64], z)
    c.decode(qd[64], kd[64], vd[64])


def test_promotion_and_demotion_rules():
    lay, c, vl0, _ = _cache(B=1, Hkv=1, Hq=2)
    b = h = 0
    old = set(int(p) for p in vl0[0][0])
    packed_not_vl = [p for p in range(c.n_packed) if p not in old][:3]
    keep = sorted(old)[:2]
    drop = sorted(old)[2]
    # a hand-made new set: two old lines, three promoted packed positions
    new = np.array(sorted(keep + packed_not_vl), np.int64)
    c.merge([[new]])
    K, V = c.rep(b, h)
    for p in keep:          # an old line keeps its FP16 row
        assert np.array_equal(K[p], lay.k[0, 0, p].astype(np.float64))
    for p in packed_not_vl:  # a promoted line is its dequantised record rounded once to FP16
        want = formats.dequant_k4v4_fp16(c.kq[0, 0, p], c.ks[0, 0, p], c.kz[0, 0, p]).astype(np.float64)
        assert np.array_equal(K[p], want)
    # a demoted line falls back to the record it got when it was first packed
    cc, s, z = formats.pack_k4v4(lay.k[0, 0, drop])
    assert np.array_equal(K[drop], formats.dequant_k4v4(cc, s, z))


def test_decode_uses_current_representation():
    lay, c, _, _ = _cache(B=1, Hkv=1, Hq=4)
    qd, kd, vd = synth.decode_tokens(1, 1, 4, 1, 3)
    from oracle.attention import attend
    for t in range(3):
        o = c.decode(qd[t], kd[t], vd[t])
        K, V = c.rep(0, 0)
        assert K.shape[0] == 400 + t + 1
        assert np.allclose(o[0], attend(qd[t, 0], K, V, 1 / np.sqrt(128)), rtol=0, atol=0)


def test_decode_from_an_empty_cache_closed_forms():
    """No prefix: the first step is a softmax over one key, so every query head
    returns its kv head's new V row exactly; the second step is a two-key
    softmax in closed form over the two FP16 rows (both still in the window)."""
    B, Hq, Hkv, W = 1, 4, 2, 8
    G = Hq // Hkv
    r = hybrid.HybridCacheRef(B, Hq, Hkv, W, 500, 64)
    q, k, v = synth.decode_tokens(4, B, Hq, Hkv, 2)
    o0 = r.decode(q[0], k[0], v[0])
    for h in range(Hq):
        assert np.array_equal(o0[0, h], v[0][0, h // G].astype(np.float64))
    o1 = r.decode(q[1], k[1], v[1])
    sm = 1.0 / np.sqrt(128)
    for h in range(Hq):
        kv = h // G
        K = np.stack([k[0][0, kv], k[1][0, kv]]).astype(np.float64)
        V = np.stack([v[0][0, kv], v[1][0, kv]]).astype(np.float64)
        s = K @ q[1][0, h].astype(np.float64) * sm
        p = np.exp(s - s.max())
        want = (p / p.sum()) @ V
        assert np.allclose(o1[0, h], want, rtol=1e-12, atol=1e-12)
    assert r.T == 2 and r.n_packed == 0
