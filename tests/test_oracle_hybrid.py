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


def _rep_by_hand(K16, packed_upto, vl_rows, upto):
    """Keys [0, upto) of one (b, kv head) built row by row from the raw FP16
    history: a vertical line gives its VL row, a packed position the
    dequantisation of the record its own FP16 value packs to, anything later
    its FP16 value (no call into the cache object)."""
    D = K16.shape[-1]
    out = np.empty((upto, D))
    for j in range(upto):
        if j in vl_rows:
            out[j] = vl_rows[j].astype(np.float64)
        elif j < packed_upto:
            c, s, z = formats.pack_k4v4(K16[j][None])
            out[j] = formats.dequant_k4v4(c, s, z)[0]
        else:
            out[j] = K16[j].astype(np.float64)
    return out


def _column_mass_by_hand(K, queries, n, sm):
    """queries: list of (position, q row); explicit loops over heads, queries and keys."""
    mass = np.zeros(n)
    for p, q in queries:
        logits = [sum(float(q[d]) * K[j, d] for d in range(K.shape[1])) * sm for j in range(p + 1)]
        mx = max(logits)
        w = [np.exp(x - mx) for x in logits]
        z = sum(w)
        for j in range(min(n, p + 1)):
            mass[j] += w[j] / z
    return mass


def test_reselect_brute_force_pre_merge():
    """Decode-mode reselection (HyQuant digest, method paragraph: the column mass
    of the buffered queries, recomputed every 64 tokens) against explicit loops.
    Every buffered query of every head of the group is paired with its own
    position (a query sees keys j <= its position only), the keys are taken in
    the representation they have before the merge (the positions about to leave
    the window are still FP16), and the k largest scores are kept."""
    B, Hq, Hkv, L, W, steps = 2, 4, 2, 24, 4, 6
    G = Hq // Hkv
    lay = synth.planted_layer(31, B, Hq, Hkv, L)
    c = hybrid.HybridCacheRef(B, Hq, Hkv, W, 2500, cap=64)
    vl0, _ = c.init_from_prefix(lay.k, lay.v, lay.q_tail)
    qd, kd, vd = synth.decode_tokens(31, B, Hq, Hkv, steps)
    for t in range(steps):
        c.decode(qd[t], kd[t], vd[t])
    T = L + steps
    assert c.T == T and c.n_packed == L - W and c.staged() == steps
    K16 = np.concatenate([lay.k, np.moveaxis(kd, 0, 2)], axis=2)      # [B, Hkv, T, D] raw history
    n = T - W
    kk = select.k_of(n, 2500)
    vl, scores = c.reselect()
    for b in range(B):
        for h in range(Hkv):
            rows = {int(p): lay.k[b, h, p] for p in vl0[b][h]}         # prefix VL rows are the dense rows
            K = _rep_by_hand(K16[b, h], L - W, rows, T)
            queries = [(L + t, qd[t, b, hh]) for hh in range(h * G, (h + 1) * G) for t in range(steps)]
            want = _column_mass_by_hand(K, queries, n, 1 / np.sqrt(128))
            assert np.allclose(scores[b][h], want, rtol=1e-11, atol=1e-14), (b, h)
            order = sorted(range(n), key=lambda j: (-want[j], j))[:kk]
            assert list(vl[b][h]) == sorted(order), (b, h)
    # the state is untouched by the reselection itself
    assert c.T == T and c.n_packed == L - W


def test_reselect_with_an_empty_query_buffer():
    """Right after a prefix install nothing is buffered: every score is zero and
    the stable top-k keeps the lowest k positions."""
    lay, c, _, _ = _cache(L=200, W=32, B=1, Hq=4, Hkv=2)
    assert c.qbuf == []
    vl, sc = c.reselect()
    n = 200 - 32
    for h in range(2):
        assert np.array_equal(sc[0][h], np.zeros(n))
        assert np.array_equal(vl[0][h], np.arange(select.k_of(n, 500)))


def test_merge_keeps_fp16_of_a_line_that_just_left_the_window():
    """A position that leaves the window at this merge and is selected as a
    vertical line keeps its FP16 value (it still has one), not its new record;
    this holds for a prefix position and for a decoded one alike."""
    lay, c, vl0, _ = _cache(L=300, W=40, B=1, Hq=2, Hkv=1)
    qd, kd, vd = synth.decode_tokens(2, 1, 2, 1, 64)
    for t in range(64):
        c.decode(qd[t], kd[t], vd[t])
    old_np = c.n_packed
    assert old_np == 260 and c.T == 364
    K16 = np.concatenate([lay.k[0, 0], kd[:, 0, 0]])
    V16 = np.concatenate([lay.v[0, 0], vd[:, 0, 0]])
    exited = [262, 290, 311]            # in [old_np, T - W) = [260, 324); 311 is a decoded token
    new = np.array(sorted(list(vl0[0][0][:3]) + exited), np.int64)
    c.merge([[new]])
    assert c.n_packed == 324
    K, V = c.rep(0, 0)
    for p in exited:
        assert np.array_equal(K[p], K16[p].astype(np.float64))
        assert np.array_equal(V[p], V16[p].astype(np.float64))
        # and that differs from the record the position now has
        deq = formats.dequant_k4v4(c.kq[0, 0, p], c.ks[0, 0, p], c.kz[0, 0, p])
        assert not np.array_equal(K[p], deq)
        cc, s, z = formats.pack_k4v4(K16[p])
        assert np.array_equal(c.kq[0, 0, p], cc)


def test_decode_against_loops_over_a_hand_built_cache():
    """Decode steps over a prefix with lines, window and staged tokens equal
    softmax loops over keys/values built row by row from the raw history."""
    B, Hq, Hkv, L, W = 1, 4, 2, 40, 8
    G = Hq // Hkv
    lay = synth.planted_layer(17, B, Hq, Hkv, L)
    c = hybrid.HybridCacheRef(B, Hq, Hkv, W, 1000, cap=64)
    vl0, _ = c.init_from_prefix(lay.k, lay.v, lay.q_tail)
    qd, kd, vd = synth.decode_tokens(17, B, Hq, Hkv, 3)
    from oracle.attention import attend_loops
    for t in range(3):
        o = c.decode(qd[t], kd[t], vd[t])
        T = L + t + 1
        for h in range(Hkv):
            K16 = np.concatenate([lay.k[0, h], kd[:t + 1, 0, h]])
            V16 = np.concatenate([lay.v[0, h], vd[:t + 1, 0, h]])
            K = _rep_by_hand(K16, L - W, {int(p): lay.k[0, h, p] for p in vl0[0][h]}, T)
            V = _rep_by_hand(V16, L - W, {int(p): lay.v[0, h, p] for p in vl0[0][h]}, T)
            want = attend_loops(qd[t, 0, h * G:(h + 1) * G], K, V, 1 / np.sqrt(128))
            assert np.allclose(o[0, h * G:(h + 1) * G], want, rtol=1e-11, atol=1e-13), (t, h)


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


def test_running_scores_accumulate_over_reselections():
    """accumulate=True (the running column-mass reading of README Overview
    item 1): the score of a position is the prefix selection's column mass
    plus the column mass of every later reselection, each taken from explicit
    loops over the keys as they were at that reselection; the set is the
    stable top-k of the running score.  Positions that entered the scored
    prefix later start from zero."""
    B, Hq, Hkv, L, W, steps = 1, 4, 2, 24, 4, 5
    G = Hq // Hkv
    sm = 1 / np.sqrt(128)
    lay = synth.planted_layer(37, B, Hq, Hkv, L)
    c = hybrid.HybridCacheRef(B, Hq, Hkv, W, 2500, cap=64, accumulate=True)
    vl0, sc0 = c.init_from_prefix(lay.k, lay.v, lay.q_tail)
    n0 = L - W
    nq = lay.q_tail.shape[2]
    running = np.zeros((Hkv, 64))
    for h in range(Hkv):
        K = lay.k[0, h].astype(np.float64)
        queries = [(L - nq + i, lay.q_tail[0, hh, i]) for hh in range(h * G, (h + 1) * G) for i in range(nq)]
        running[h, :n0] = _column_mass_by_hand(K, queries, n0, sm)
        assert np.allclose(c.acc[0, h, :n0], running[h, :n0], rtol=1e-11, atol=1e-14)
    qd, kd, vd = synth.decode_tokens(37, B, Hq, Hkv, 2 * steps)
    K16 = np.concatenate([lay.k, np.moveaxis(kd, 0, 2)], axis=2)
    vl_prev = {h: {int(p): lay.k[0, h, p] for p in vl0[0][h]} for h in range(Hkv)}
    for period in range(2):
        for t in range(period * steps, (period + 1) * steps):
            c.decode(qd[t], kd[t], vd[t])
        T = L + (period + 1) * steps
        n = T - W
        # keys as they are before this merge: the previous merge packed [0, n_packed)
        packed_upto = c.n_packed
        vl, scores = c.reselect()
        kk = select.k_of(n, 2500)
        for h in range(Hkv):
            K = _rep_by_hand(K16[0, h], packed_upto, vl_prev[h], T)
            buffered = list(range(0, (period + 1) * steps))
            queries = [(L + t, qd[t, 0, hh]) for hh in range(h * G, (h + 1) * G) for t in buffered]
            running[h, :n] += _column_mass_by_hand(K, queries, n, sm)
            assert np.allclose(scores[0][h], running[h, :n], rtol=1e-11, atol=1e-14), (period, h)
            order = sorted(range(n), key=lambda j: (-running[h, j], j))[:kk]
            assert list(vl[0][h]) == sorted(order)
        c.merge(vl)
        # rows of the new set: FP16 values for lines that had one, else dequantised records rounded once
        for h in range(Hkv):
            vl_prev[h] = {int(p): c.kf[0][h][r] for r, p in enumerate(vl[0][h])}


def test_running_scores_start_from_the_prefix_selection():
    """start_running_scores (a prefix installed with sets chosen elsewhere)
    gives the same running scores as init_from_prefix."""
    lay = synth.planted_layer(38, 1, 4, 2, 100)
    a = hybrid.HybridCacheRef(1, 4, 2, 16, 500, cap=128, accumulate=True)
    vl, _ = a.init_from_prefix(lay.k, lay.v, lay.q_tail)
    b = hybrid.HybridCacheRef(1, 4, 2, 16, 500, cap=128, accumulate=True)
    b.install_prefix(lay.k, lay.v, vl)
    b.start_running_scores(lay.k, lay.q_tail)
    assert np.array_equal(a.acc, b.acc)
