"""Helpers shared by the GPU parity tests: run the CUDA path and the CPU oracle
on the same seeded inputs and compare them.

Tolerances (the reasoning is in the design notes):
  decode output        max-abs <= 2e-3 and rel-L2 <= 1e-3 against the float64 oracle
  column-mass scores   relative error <= SCORE_RTOL per score.  The kernel
                       rebuilds each packed key as fp16 (one rounding, <= 2^-11
                       relative per element, ~2e-4 nat on a logit) and sums
                       float32 exp2 weights; the measured worst case is ~2e-4,
                       so the bound is 5e-4 and the tie band twice that
                       With 2-bit keys the rebuilt values sit at the group's
                       four levels (min, min + span/3, ...), about 1.5 times the
                       RMS magnitude of 4-bit ones, and each logit's rounding
                       error grows with them: the measured worst case at 32K
                       is 7e-4, so the bound is SCORE_RTOL_K2 = 1e-3 (and the
                       tie band twice that)
  selected positions   exact when the GPU's own float32 scores are fed to the
                       oracle's stable top-k; against the oracle's float64
                       scores, a position may differ only inside the band
                       |s - s_k| <= BAND_RTOL * s_k
  packed bytes, scale/zero words, VL rows, VL positions: bit-exact
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import formats, hybrid, select as osel

SCORE_RTOL = 5e-4
BAND_RTOL = 1e-3
SCORE_RTOL_K2 = 1e-3
BAND_RTOL_K2 = 2e-3
DEC_MAXABS = 2e-3
DEC_RELL2 = 1e-3


def hq():
    from hybrid_precision_attention_b200 import hq as _hq
    return _hq


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def sz_words(scale, zero):
    """(scale, zero) fp16 arrays -> uint32 words as the cache stores them."""
    return scale.view(np.uint16).astype(np.uint32) | (zero.view(np.uint16).astype(np.uint32) << 16)


def check_decode(out_gpu: torch.Tensor, ref: np.ndarray, what=""):
    o = out_gpu.float().cpu().numpy().astype(np.float64)
    err = np.abs(o - ref)
    rel = np.linalg.norm(o - ref) / max(np.linalg.norm(ref), 1e-30)
    assert np.all(np.isfinite(o)), what
    assert err.max() <= DEC_MAXABS, f"{what} max-abs {err.max():.3e}"
    assert rel <= DEC_RELL2, f"{what} rel-L2 {rel:.3e}"
    return err.max(), rel


def check_selection(gpu_scores: np.ndarray, gpu_sel: np.ndarray, ref_scores: np.ndarray, k: int, what="",
                    rtol=SCORE_RTOL, band=BAND_RTOL):
    """gpu_scores/ref_scores over the n candidates of one (b, kv head); gpu_sel = the GPU's k positions."""
    n = ref_scores.shape[0]
    if n == 0:
        assert k == 0 and len(gpu_sel) == 0, what
        return 0.0
    g = gpu_scores[:n].astype(np.float64)
    rel = np.abs(g - ref_scores) / np.maximum(np.abs(ref_scores), 1e-30)
    assert rel.max() <= rtol, f"{what} score rel err {rel.max():.3e}"
    # the top-k stage is exact on the GPU's own scores
    want = osel.topk_stable(gpu_scores[:n].astype(np.float32), k)
    assert np.array_equal(np.sort(gpu_sel), gpu_sel), f"{what} not ascending"
    assert np.array_equal(gpu_sel, want), f"{what} top-k differs on the GPU's own scores"
    # against the float64 scores: differences only inside the tie band
    ref_sel = osel.topk_stable(ref_scores, k)
    if k > 0:
        sk = np.sort(ref_scores)[::-1][k - 1]
        diff = np.setxor1d(ref_sel, gpu_sel)
        assert np.all(np.abs(ref_scores[diff] - sk) <= band * sk), f"{what} selection differs outside the band"
    return rel.max()


class Pair:
    """A GPU cache and the oracle cache, kept on the same VL sets."""

    def __init__(self, B, Hq, Hkv, L, W, rho_bp, cap, seed=0, n_tail=64, running=False, k_bits=4, v_bits=4):
        self.lay = __import__("hybrid_precision_attention_b200.synth", fromlist=["x"]).planted_layer(seed, B, Hq, Hkv, L, n_tail=n_tail)
        self.B, self.Hq, self.Hkv, self.L, self.W, self.rho = B, Hq, Hkv, L, W, rho_bp
        self.running = running
        self.tol = (SCORE_RTOL_K2, BAND_RTOL_K2) if k_bits == 2 else (SCORE_RTOL, BAND_RTOL)
        H = hq()
        self.g = H.HybridCache(B, Hq, Hkv, cap, W, rho_bp, running_scores=running, k_bits=k_bits, v_bits=v_bits)
        self.r = hybrid.HybridCacheRef(B, Hq, Hkv, W, rho_bp, self.g.cap, accumulate=running, k_bits=k_bits, v_bits=v_bits)

    def init(self, check=True):
        H = hq()
        k, v, qt = dev(self.lay.k), dev(self.lay.v), dev(self.lay.q_tail)
        scores = torch.zeros((self.B, self.Hkv, self.g.cap), dtype=torch.float32, device="cuda")
        H.hq_select_vlines(self.g, k, qt, scores_out=scores)
        H.hq_pack_merge(self.g, k, v)
        torch.cuda.synchronize()
        st = self.g.state()
        n = max(self.L - self.W, 0)
        kk = osel.k_of(n, self.rho)
        assert st["k_sel"] == kk and st["T"] == self.L and st["n_packed"] == n and st["n_vl"] == kk and st["err"] == 0, st
        sel = self.g.vl_sel.cpu().numpy()
        gsc = scores.cpu().numpy()
        vl = [[sel[b, h, :kk].astype(np.int64) for h in range(self.Hkv)] for b in range(self.B)]
        if check:
            nq = self.lay.q_tail.shape[2]
            qpos = np.tile(np.arange(self.L - nq, self.L), self.Hq // self.Hkv)
            G = self.Hq // self.Hkv
            for b in range(self.B):
                for h in range(self.Hkv):
                    qs = self.lay.q_tail[b, h * G:(h + 1) * G].reshape(-1, 128).astype(np.float64)
                    ref = osel.column_mass(self.lay.k[b, h].astype(np.float64), qs, qpos, n, 1 / np.sqrt(128))
                    check_selection(gsc[b, h], vl[b][h], ref, kk, f"init b{b} h{h}", *self.tol)
        self.r.install_prefix(self.lay.k, self.lay.v, vl)
        if self.running:
            self.r.start_running_scores(self.lay.k, self.lay.q_tail)
        if check:
            self.check_state()
        return vl

    def check_state(self):
        """Packed records, VL store and bitmap: bit-exact against the oracle."""
        np_ = self.r.n_packed
        g = self.g
        assert g.state()["n_packed"] == np_
        pk = g.packed()
        kq = pk["kq"][:, :, :np_]
        vq = pk["vq"][:, :, :np_]
        assert np.array_equal(kq, self.r.kq[:, :, :np_]), "K codes differ"
        assert np.array_equal(vq, self.r.vq[:, :, :np_]), "V codes differ"
        ksz = pk["ksz"][:, :, :np_]
        vsz = pk["vsz"][:, :, :np_]
        assert np.array_equal(ksz, sz_words(self.r.ks[:, :, :np_], self.r.kz[:, :, :np_])), "K scale/zero differ"
        assert np.array_equal(vsz, sz_words(self.r.vs[:, :, :np_], self.r.vz[:, :, :np_])), "V scale/zero differ"
        nvl = g.state()["n_vl"]
        kf = g.kf.cpu().numpy()
        vf = g.vf.cpu().numpy()
        pos = g.vl_pos.cpu().numpy()
        bits_all = pk["vl_bits"]
        for b in range(self.B):
            for h in range(self.Hkv):
                assert nvl == len(self.r.vl[b][h])
                assert np.array_equal(pos[b, h, :nvl], self.r.vl[b][h])
                assert np.array_equal(kf[b, h, :nvl].view(np.uint16), self.r.kf[b][h].view(np.uint16)), "VL K rows differ"
                assert np.array_equal(vf[b, h, :nvl].view(np.uint16), self.r.vf[b][h].view(np.uint16)), "VL V rows differ"
                assert np.array_equal(np.nonzero(bits_all[b, h])[0], self.r.vl[b][h]), "VL bitmap differs"

    def decode(self, q, k, v):
        H = hq()
        out = H.hq_decode_attn(self.g, dev(q), dev(k), dev(v))
        ref = self.r.decode(q, k, v)
        st = self.g.state()
        assert st["err"] == 0 and st["T"] == self.r.T, st
        return out, ref

    def reselect_merge(self, check=True):
        H = hq()
        scores = torch.zeros((self.B, self.Hkv, self.g.cap), dtype=torch.float32, device="cuda")
        H.hq_select_vlines(self.g, scores_out=scores)
        torch.cuda.synchronize()
        st = self.g.state()
        n = max(self.r.T - self.W, 0)
        kk = osel.k_of(n, self.rho)
        assert st["k_sel"] == kk, (st, kk)
        sel = self.g.vl_sel.cpu().numpy()
        vl = [[sel[b, h, :kk].astype(np.int64) for h in range(self.Hkv)] for b in range(self.B)]
        if check or self.running:   # running scores: the oracle's sums must follow every reselection
            _, ref_scores = self.r.reselect()
            gsc = scores.cpu().numpy()
        if check:
            for b in range(self.B):
                for h in range(self.Hkv):
                    check_selection(gsc[b, h], vl[b][h], ref_scores[b][h], kk, f"reselect b{b} h{h}", *self.tol)
        H.hq_pack_merge(self.g)
        self.r.merge(vl)
        torch.cuda.synchronize()
        assert self.g.state()["err"] == 0, self.g.state()
        if check:
            self.check_state()
        return vl
