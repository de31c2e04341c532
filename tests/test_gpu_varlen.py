"""GPU parity of ragged (variable-length) batches over a paged K4V4 store,
through the C ABI.

Each sequence of the batch has its own lengths (its row of the state array)
and its own oracle cache (oracle.hybrid.HybridCacheRef with B = 1).  The pages
of the K4V4 store come from a pool in a shuffled order through the page table.
Prefixes of different lengths are installed one sequence at a time through
single-sequence descriptors; decode, reselection and merge then run over the
whole batch in one call each, every sequence checked against its own oracle:
decode outputs within the decode tolerances, selections against the oracle's
column mass, records, VL rows and bitmaps bit-exactly.
"""
import numpy as np
import pytest
import torch

from hybrid_precision_attention_b200 import synth
from oracle import hybrid, select as osel
from tests._gpu import (BAND_RTOL, BAND_RTOL_K2, SCORE_RTOL, SCORE_RTOL_K2, check_decode, check_selection, dev, hq,
                        sz_words)

pytestmark = pytest.mark.gpu


class Ragged:
    def __init__(self, lengths, Hq, Hkv, W, rho, cap, seed, paged=True, spare_pages=5, k_bits=4, v_bits=4):
        H = hq()
        self.lengths, self.Hq, self.Hkv, self.W, self.rho = list(lengths), Hq, Hkv, W, rho
        self.B = len(lengths)
        self.G = Hq // Hkv
        npg = ((cap + 127) // 128 * 128) // 64
        n_pages = self.B * Hkv * npg + spare_pages
        order = np.random.default_rng(seed).permutation(n_pages)[:self.B * Hkv * npg] if paged else None
        self.g = H.HybridCache(self.B, Hq, Hkv, cap, W, rho, paged=paged, n_pages=n_pages if paged else None,
                               page_order=order, k_bits=k_bits, v_bits=v_bits)
        self.refs = [hybrid.HybridCacheRef(1, Hq, Hkv, W, rho, self.g.cap, k_bits=k_bits, v_bits=v_bits)
                     for _ in lengths]
        # score bounds: 2-bit keys rebuild to larger values (tests/_gpu.py)
        self.tol = (SCORE_RTOL_K2, BAND_RTOL_K2) if k_bits == 2 else (SCORE_RTOL, BAND_RTOL)
        self.lays = [synth.planted_layer(seed + 10 * b, 1, Hq, Hkv, L) for b, L in enumerate(lengths)]

    def install(self, b, check=True):
        H = hq()
        lay = self.lays[b]
        s = self.g.slot(b)
        L = self.lengths[b]
        scores = torch.zeros((1, self.Hkv, self.g.cap), dtype=torch.float32, device="cuda")
        H.hq_select_vlines(s, dev(lay.k), dev(lay.q_tail), scores_out=scores)
        H.hq_pack_merge(s, dev(lay.k), dev(lay.v))
        torch.cuda.synchronize()
        st = self.g.state(b)
        n = max(L - self.W, 0)
        kk = osel.k_of(n, self.rho)
        assert st["T"] == L and st["n_packed"] == n and st["n_vl"] == kk and st["err"] == 0, st
        sel = s.vl_sel.cpu().numpy()
        vl = [[sel[0, h, :kk].astype(np.int64) for h in range(self.Hkv)]]
        if check:
            nq = lay.q_tail.shape[2]
            qpos = np.tile(np.arange(L - nq, L), self.G)
            gsc = scores.cpu().numpy()
            for h in range(self.Hkv):
                qs = lay.q_tail[0, h * self.G:(h + 1) * self.G].reshape(-1, 128).astype(np.float64)
                ref = osel.column_mass(lay.k[0, h].astype(np.float64), qs, qpos, n, 1 / np.sqrt(128))
                check_selection(gsc[0, h], vl[0][h], ref, kk, f"seq {b} install h{h}", *self.tol)
        self.refs[b].install_prefix(lay.k, lay.v, vl)

    def check_store(self, b):
        """Records, VL rows, positions and bitmap of sequence b, bit-exact (through the page table)."""
        r = self.refs[b]
        np_ = r.n_packed
        pk = self.g.packed()
        assert self.g.state(b)["n_packed"] == np_
        assert np.array_equal(pk["kq"][b, :, :np_], r.kq[0, :, :np_])
        assert np.array_equal(pk["vq"][b, :, :np_], r.vq[0, :, :np_])
        assert np.array_equal(pk["ksz"][b, :, :np_], sz_words(r.ks[0, :, :np_], r.kz[0, :, :np_]))
        assert np.array_equal(pk["vsz"][b, :, :np_], sz_words(r.vs[0, :, :np_], r.vz[0, :, :np_]))
        nvl = self.g.state(b)["n_vl"]
        kf, vf, pos = self.g.kf[b].cpu().numpy(), self.g.vf[b].cpu().numpy(), self.g.vl_pos[b].cpu().numpy()
        for h in range(self.Hkv):
            assert nvl == len(r.vl[0][h])
            assert np.array_equal(pos[h, :nvl], r.vl[0][h])
            assert np.array_equal(kf[h, :nvl].view(np.uint16), r.kf[0][h].view(np.uint16))
            assert np.array_equal(vf[h, :nvl].view(np.uint16), r.vf[0][h].view(np.uint16))
            assert np.array_equal(np.nonzero(pk["vl_bits"][b, h])[0], r.vl[0][h])

    def decode(self, q, k, v, active=None, check=True):
        """One batched decode step; `active` = sequences expected to take it (others are full)."""
        H = hq()
        active = list(range(self.B)) if active is None else active
        before = self.g.states()
        sentinel = torch.full((self.B, self.Hq, 128), 7.0, dtype=torch.float16, device="cuda")
        out = H.hq_decode_attn(self.g, dev(q), dev(k), dev(v), out=sentinel)
        torch.cuda.synchronize()
        after = self.g.states()
        for b in range(self.B):
            if b in active:
                assert after[b]["T"] == before[b]["T"] + 1 and after[b]["err"] == 0, (b, after[b])
                if check:
                    want = self.refs[b].decode(q[b:b + 1], k[b:b + 1], v[b:b + 1])
                    check_decode(out[b:b + 1], want, f"seq {b} T={after[b]['T']}")
                else:
                    self.refs[b].append(q[b:b + 1], k[b:b + 1], v[b:b + 1])
            else:
                assert after[b]["T"] == before[b]["T"] and after[b]["err"] & H.DEVERR_STAGING_FULL, (b, after[b])
                assert torch.all(out[b] == 7.0)
        return out

    def reselect_merge(self):
        H = hq()
        scores = torch.zeros((self.B, self.Hkv, self.g.cap), dtype=torch.float32, device="cuda")
        H.hq_select_vlines(self.g, scores_out=scores)
        torch.cuda.synchronize()
        sts = self.g.states()
        sel = self.g.vl_sel.cpu().numpy()
        gsc = scores.cpu().numpy()
        vls = []
        for b in range(self.B):
            r = self.refs[b]
            n = max(r.T - self.W, 0)
            kk = osel.k_of(n, self.rho)
            assert sts[b]["k_sel"] == kk, (b, sts[b], kk)
            vl = [[sel[b, h, :kk].astype(np.int64) for h in range(self.Hkv)]]
            _, ref_scores = r.reselect()
            for h in range(self.Hkv):
                check_selection(gsc[b, h], vl[0][h], ref_scores[0][h], kk, f"seq {b} reselect h{h}", *self.tol)
            vls.append(vl)
        H.hq_pack_merge(self.g)
        torch.cuda.synchronize()
        for b in range(self.B):
            self.refs[b].merge(vls[b])
            assert self.g.state(b)["err"] == 0, self.g.state(b)
            self.check_store(b)


def _tokens(seed, B, Hq, Hkv, n):
    return synth.decode_tokens(seed, B, Hq, Hkv, n)


def test_ragged_paged_batch_small():
    """Three sequences of 200, 700 and 1000 tokens (GQA 4, W = 64): installed
    one at a time, decoded together, one of them advanced alone until its
    staging area fills first (the batch call then skips and flags it while the
    others proceed), reselected and merged together, decoded again."""
    H = hq()
    Hq, Hkv, W = 8, 2, 64
    r = Ragged([200, 700, 1000], Hq, Hkv, W, 500, cap=1300, seed=41)
    for b in range(3):
        r.install(b)
        r.check_store(b)
    q, k, v = _tokens(41, 3, Hq, Hkv, 80)
    for t in range(4):
        r.decode(q[t], k[t], v[t])
    # sequence 1 alone through its single-sequence descriptor: 60 more tokens -> its staging is full
    s1 = r.g.slot(1)
    for t in range(4, 64):
        H.hq_decode_attn(s1, dev(q[t][1:2]), dev(k[t][1:2]), dev(v[t][1:2]))
        r.refs[1].append(q[t][1:2], k[t][1:2], v[t][1:2])
    torch.cuda.synchronize()
    assert r.g.state(1)["T"] == 764 and r.g.state(0)["T"] == 204
    r.decode(q[64], k[64], v[64], active=[0, 2])
    for b in range(3):
        r.g.state_t[b, H.STATE_ERR] = 0
    r.reselect_merge()
    assert [s["n_packed"] for s in r.g.states()] == [205 - W, 764 - W, 1005 - W]
    for t in range(65, 70):
        r.decode(q[t], k[t], v[t])


def test_page_table_entry_outside_the_pool_is_flagged():
    """A page-table entry outside [0, n_pages) is not followed: the sequence is
    flagged with HQ_DEVERR_PAGE (its output unspecified) and the other sequence
    is unaffected."""
    H = hq()
    Hq, Hkv, W = 8, 2, 32
    r = Ragged([300, 300], Hq, Hkv, W, 500, cap=400, seed=43)
    for b in range(2):
        r.install(b)
    r.g.page_table[1, 0, 2] = r.g.n_pages + 1000   # a page of sequence 1 that the scan reads
    q, k, v = _tokens(43, 2, Hq, Hkv, 1)
    out = H.hq_decode_attn(r.g, dev(q[0]), dev(k[0]), dev(v[0]))
    torch.cuda.synchronize()
    st = r.g.states()
    assert st[1]["err"] & H.DEVERR_PAGE and st[0]["err"] == 0
    want = r.refs[0].decode(q[0][0:1], k[0][0:1], v[0][0:1])
    check_decode(out[0:1], want, "unaffected sequence")


@pytest.mark.slow
def test_ragged_paged_batch_1k_3k_32k():
    """Lengths 1K, 3K and 32K in one batch (Llama-3.1-8B attention shape, W =
    128, rho = 5 %): decode steps checked every few tokens through a full
    64-token period, batched reselection + merge, decode after the merge."""
    Hq, Hkv, W = 32, 8, 128
    lengths = [1024, 3072, 32768]
    r = Ragged(lengths, Hq, Hkv, W, 500, cap=32768 + 256, seed=47)
    for b in range(3):
        r.install(b)
    for b in range(3):
        r.check_store(b)
    q, k, v = _tokens(47, 3, Hq, Hkv, 67)
    for t in range(64):
        r.decode(q[t], k[t], v[t], check=(t % 9 == 0 or t == 63))
    r.decode(q[64], k[64], v[64], active=[])        # every staging area is full now
    for b in range(3):
        r.g.state_t[b, hq().STATE_ERR] = 0
    r.reselect_merge()
    for t in range(65, 67):
        r.decode(q[t], k[t], v[t])


def test_ragged_batch_on_the_stream_k_grid():
    """Twelve sequences of 300 .. 2500 tokens with 4 kv heads (48 units: more
    than a quarter of the grid, so the decode cuts the batch's tile list into
    equal stream-K ranges whose segments cross sequences): one install per
    sequence, a batched period, reselection and merge, two more steps, every
    sequence against its own oracle."""
    lengths = [300, 2500, 700, 1200, 450, 2000, 900, 1600, 333, 1800, 1100, 640]
    rg = Ragged(lengths, 16, 4, 64, 500, cap=2700, seed=70)
    for b in range(rg.B):
        rg.install(b, check=(b % 4 == 0))
    q, k, v = _tokens(71, rg.B, 16, 4, 66)
    for t in range(64):
        rg.decode(q[t], k[t], v[t], check=(t % 16 == 0 or t == 63))
    rg.reselect_merge()
    for t in range(64, 66):
        rg.decode(q[t], k[t], v[t])


def test_one_sequence_reset_and_reused_in_a_running_batch():
    """A finished request's slot reused: sequence 1 of a ragged paged batch is
    reset through its single-sequence descriptor (its state row, its pages'
    bitmaps) and given a new prompt, while sequences 0 and 2 keep their
    caches; the batch then decodes on, every sequence against its own oracle."""
    rg = Ragged([600, 900, 300], 8, 2, 64, 500, cap=1200, seed=90)
    for b in range(rg.B):
        rg.install(b, check=False)
    q, k, v = _tokens(91, rg.B, 8, 2, 40)
    for t in range(20):
        rg.decode(q[t], k[t], v[t], check=(t == 19))
    H = hq()
    H.hq_cache_reset(rg.g.slot(1))
    torch.cuda.synchronize()
    st = rg.g.states()
    assert st[1]["T"] == 0 and st[1]["n_vl"] == 0 and not rg.g.packed()["vl_bits"][1].any(), st[1]
    assert st[0]["T"] == 620 and st[2]["T"] == 320, st
    rg.lengths[1] = 450
    rg.lays[1] = synth.planted_layer(92, 1, 8, 2, 450)
    rg.refs[1] = hybrid.HybridCacheRef(1, 8, 2, 64, 500, rg.g.cap)
    rg.install(1)
    rg.check_store(1)
    for t in range(20, 40):
        rg.decode(q[t], k[t], v[t], check=(t % 6 == 0 or t == 39))
    for b in range(rg.B):
        rg.check_store(b)
