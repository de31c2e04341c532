"""The hybrid KV cache as a plain state machine.

TEST INFRASTRUCTURE ONLY (see the package docstring).

What the pages fix (HyQuant digest, method and prefill/decode paragraphs;
README Overview items 1 and 3, "Overhead"):

* three key classes: vertical-line (VL) positions and a recent window stay in
  FP16, every other position is stored K4V4 (or, with ``k_bits`` / ``v_bits``,
  the README's other code widths: K8V8, K4V2, K2V4);
* the VL set is chosen on the prefill's tail queries, then re-identified every
  64 tokens from at most 64 buffered FP16 queries — decode does not recompute
  global importance every step;
* new tokens go to a staging area first and are merged into the hybrid layout
  later.

Readings taken where the pages are silent (each listed in the design notes):

* the FP16 recent region is the last ``W`` positions at the last merge plus the
  staged tokens, so it holds between ``W`` and ``W + 64`` tokens; a decode
  step with 64 staged tokens is refused until a reselect + merge;
* a position gets its K4V4 record once, from its FP16 value, when it leaves
  the recent region (prefix init packs ``[0, L - W)``); the record is kept when
  the position later enters or leaves the VL set;
* a VL row holds the position's current FP16 value when it has one (recent
  region or previous VL set), otherwise the dequantised record rounded once to
  FP16;
* reselection uses the keys' pre-merge representation, then the merge packs the
  positions that left the window and installs the new VL set;
* VL sets are per (batch, kv head) (the KV layout is per kv head under GQA) and
  the column mass sums over the group's query heads;
* scores are recomputed at each reselection from the buffered queries; with
  ``accumulate=True`` (the other reading of the README's "running column-mass
  score") each reselection instead adds its column mass to a running score
  per position, started from the prefix selection's column mass, and the
  top-k runs on the running scores.
"""
from __future__ import annotations

import numpy as np

from . import formats, select
from .attention import attend

STAGE = 64      # staged tokens before a merge, and the reselection period
QBUF = 64       # buffered queries used by the column-mass estimate


class HybridCacheRef:
    def __init__(self, B: int, Hq: int, Hkv: int, W: int, rho_bp: int, cap: int, D: int = 128,
                 accumulate: bool = False, k_bits: int = 4, v_bits: int = 4):
        assert Hq % Hkv == 0 and D % formats.GROUP == 0
        self.B, self.Hq, self.Hkv, self.D, self.W, self.rho_bp, self.cap = B, Hq, Hkv, D, W, rho_bp, cap
        self.G = Hq // Hkv
        self.sm_scale = 1.0 / np.sqrt(D)
        self.k16 = np.zeros((B, Hkv, cap, D), np.float16)      # FP16 value of each position while it has one
        self.v16 = np.zeros((B, Hkv, cap, D), np.float16)
        assert k_bits in formats.BITS and v_bits in formats.BITS
        self.k_bits, self.v_bits = k_bits, v_bits
        self.kq = np.zeros((B, Hkv, cap, D * k_bits // 8), np.uint8)
        self.vq = np.zeros((B, Hkv, cap, D * v_bits // 8), np.uint8)
        self.ks = np.zeros((B, Hkv, cap, D // formats.GROUP), np.float16)
        self.kz = np.zeros_like(self.ks)
        self.vs = np.zeros_like(self.ks)
        self.vz = np.zeros_like(self.ks)
        self.vl = [[np.zeros(0, np.int64) for _ in range(Hkv)] for _ in range(B)]
        self.kf = [[np.zeros((0, D), np.float16) for _ in range(Hkv)] for _ in range(B)]
        self.vf = [[np.zeros((0, D), np.float16) for _ in range(Hkv)] for _ in range(B)]
        self.T = 0
        self.n_packed = 0
        self.qbuf = []          # list of (position, q [B, Hq, D] float16), newest last
        self.accumulate = accumulate
        self.acc = np.zeros((B, Hkv, cap))   # running column mass per position (accumulate=True)

    # ------------------------------------------------------------------ helpers
    def _pack_range(self, lo: int, hi: int):
        if hi <= lo:
            return
        for arr16, q, s, z, bits in ((self.k16, self.kq, self.ks, self.kz, self.k_bits),
                                     (self.v16, self.vq, self.vs, self.vz, self.v_bits)):
            c, sc, ze = formats.pack_bits(arr16[:, :, lo:hi], bits)
            q[:, :, lo:hi], s[:, :, lo:hi], z[:, :, lo:hi] = c, sc, ze

    def rep(self, b: int, h: int, upto: int = None):
        """Keys and values [0, upto) of (b, kv head h) in their current representation (float64)."""
        T = self.T if upto is None else upto
        np_ = min(self.n_packed, T)
        K = np.empty((T, self.D))
        V = np.empty((T, self.D))
        K[:np_] = formats.dequant_bits(self.kq[b, h, :np_], self.ks[b, h, :np_], self.kz[b, h, :np_], self.k_bits)
        V[:np_] = formats.dequant_bits(self.vq[b, h, :np_], self.vs[b, h, :np_], self.vz[b, h, :np_], self.v_bits)
        vl = self.vl[b][h]
        K[vl] = self.kf[b][h].astype(np.float64)
        V[vl] = self.vf[b][h].astype(np.float64)
        K[np_:T] = self.k16[b, h, np_:T]
        V[np_:T] = self.v16[b, h, np_:T]
        return K, V

    def fp16_region(self):
        return self.n_packed, self.T

    # ------------------------------------------------------------------ prefix
    def init_from_prefix(self, K16, V16, q_tail):
        """Install a prefix of L tokens.  Selects VL lines on the tail queries
        (keys all FP16), packs [0, L - W) and keeps [L - W, L) in FP16."""
        B, Hkv, L, D = K16.shape
        n = max(L - self.W, 0)
        nq = q_tail.shape[2]
        qpos = np.tile(np.arange(L - nq, L), self.G)
        scores = [[None] * Hkv for _ in range(B)]
        new_vl = [[None] * Hkv for _ in range(B)]
        for b in range(B):
            for h in range(Hkv):
                qs = q_tail[b, h * self.G:(h + 1) * self.G].reshape(-1, D).astype(np.float64)
                new_vl[b][h], scores[b][h] = select.select_vlines(K16[b, h].astype(np.float64), qs, qpos, n, self.rho_bp, self.sm_scale)
        self.install_prefix(K16, V16, new_vl)
        self._start_running(scores, n)
        return new_vl, scores

    def _start_running(self, scores, n):
        self.acc[:] = 0.0
        for b in range(self.B):
            for h in range(self.Hkv):
                self.acc[b, h, :n] = scores[b][h]

    def start_running_scores(self, K16, q_tail):
        """The prefix selection's column mass (keys all FP16, the tail queries)
        as the starting running score, for a prefix installed with
        :meth:`install_prefix` (whose VL sets were chosen elsewhere)."""
        B, Hkv, L, D = K16.shape
        n = max(L - self.W, 0)
        nq = q_tail.shape[2]
        qpos = np.tile(np.arange(L - nq, L), self.G)
        sc = [[select.column_mass(K16[b, h].astype(np.float64),
                                  q_tail[b, h * self.G:(h + 1) * self.G].reshape(-1, D).astype(np.float64),
                                  qpos, n, self.sm_scale) for h in range(Hkv)] for b in range(B)]
        self._start_running(sc, n)
        return sc

    def install_prefix(self, K16, V16, vl_sets):
        """Install a prefix with given VL sets (the selection step done elsewhere)."""
        B, Hkv, L, D = K16.shape
        assert L <= self.cap
        self.k16[:, :, :L] = K16
        self.v16[:, :, :L] = V16
        self.T = L
        self.n_packed = 0
        self.vl = [[np.zeros(0, np.int64) for _ in range(Hkv)] for _ in range(B)]
        self.merge(vl_sets)
        self.qbuf = []

    # ------------------------------------------------------------------ decode
    def staged(self) -> int:
        return self.T - self.n_packed - self.W if self.T > 0 else 0

    def append(self, q, k_new, v_new):
        """The state change of a decode step (new token staged, query buffered)."""
        if self.T - self.n_packed >= self.W + STAGE:
            raise RuntimeError("staging full: reselect and merge first")
        t = self.T
        self.k16[:, :, t] = k_new
        self.v16[:, :, t] = v_new
        self.T = t + 1
        self.qbuf.append((t, np.array(q, np.float16)))
        self.qbuf = self.qbuf[-QBUF:]

    def decode(self, q, k_new, v_new):
        """One decode step: append (k_new, v_new) at position T and attend.

        q [B, Hq, D], k_new/v_new [B, Hkv, D] float16.  Returns float64 [B, Hq, D].
        """
        self.append(q, k_new, v_new)
        out = np.empty((self.B, self.Hq, self.D))
        for b in range(self.B):
            for h in range(self.Hkv):
                K, V = self.rep(b, h)
                out[b, h * self.G:(h + 1) * self.G] = attend(q[b, h * self.G:(h + 1) * self.G], K, V, self.sm_scale)
        return out

    # ------------------------------------------------------------------ reselect + merge
    def reselect(self):
        """Column-mass scores and new VL sets from the buffered queries."""
        n = max(self.T - self.W, 0)
        pos = np.array([p for p, _ in self.qbuf], np.int64)
        qs_all = np.stack([q for _, q in self.qbuf], axis=2) if self.qbuf else np.zeros((self.B, self.Hq, 0, self.D), np.float16)
        qpos = np.tile(pos, self.G)
        new_vl = [[None] * self.Hkv for _ in range(self.B)]
        scores = [[None] * self.Hkv for _ in range(self.B)]
        for b in range(self.B):
            for h in range(self.Hkv):
                K, _ = self.rep(b, h)
                qs = qs_all[b, h * self.G:(h + 1) * self.G].reshape(-1, self.D).astype(np.float64)
                if qs.shape[0] == 0:
                    mass = np.zeros(n)
                else:
                    mass = select.column_mass(K, qs, qpos, n, self.sm_scale)
                if self.accumulate:
                    self.acc[b, h, :n] += mass
                    mass = self.acc[b, h, :n].copy()
                scores[b][h] = mass
                new_vl[b][h] = select.topk_stable(mass, select.k_of(n, self.rho_bp))
        return new_vl, scores

    def merge(self, new_vl):
        """Pack the positions that left the window and install the new VL sets."""
        old_np = self.n_packed
        new_np = max(old_np, self.T - self.W)
        self._pack_range(old_np, new_np)
        for b in range(self.B):
            for h in range(self.Hkv):
                pos = np.asarray(new_vl[b][h], np.int64)
                assert np.all(pos < new_np) and np.all(np.diff(pos) > 0)
                kf = np.empty((len(pos), self.D), np.float16)
                vf = np.empty((len(pos), self.D), np.float16)
                old = {int(p): i for i, p in enumerate(self.vl[b][h])}
                for r, p in enumerate(pos):
                    p = int(p)
                    if p in old:
                        kf[r], vf[r] = self.kf[b][h][old[p]], self.vf[b][h][old[p]]
                    elif p >= old_np:
                        kf[r], vf[r] = self.k16[b, h, p], self.v16[b, h, p]
                    else:
                        kf[r] = formats.dequant_bits_fp16(self.kq[b, h, p], self.ks[b, h, p], self.kz[b, h, p], self.k_bits)
                        vf[r] = formats.dequant_bits_fp16(self.vq[b, h, p], self.vs[b, h, p], self.vz[b, h, p], self.v_bits)
                self.vl[b][h], self.kf[b][h], self.vf[b][h] = pos, kf, vf
        self.n_packed = new_np
