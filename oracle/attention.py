"""Attention over the hybrid representation: decode step and causal prefill.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Decode (HyQuant digest, prefill/decode paragraph; README Overview item 3):
the cache keeps the vertical-line keys/values and the recent tokens in FP16
and every other position as K4V4; the decode step is ordinary softmax
attention of the new query over every cached position plus the new token,
each key and value taken in its stored representation (dequantised where it
is K4V4).  The fused kernel never materialises an FP16 cache, but what it
computes is exactly this.

Prefill (digest, prefill/decode paragraph; README Overview item 2, "vquant_vert"
and "hybrid_full" in the Mode reference): one causal attention pass in which
key j of query i is

* a window key when ``i - W < j <= i``      -> FP16 Q, K, V;
* else a vertical-line key when j is in the set -> FP16 Q, K, V;
* else a quantised key                     -> FP8 e4m3 Q, K, V with per-block
  scales (see ``formats``);

and a single softmax covers all three classes.  A vertical-line key inside a
query's window is counted once, as a window key.  The oracle keeps the
softmax weights in float64; the GPU kernel's rounding of P is inside the
stated tolerance.
"""
from __future__ import annotations

import numpy as np

from . import formats


def attend(q: np.ndarray, keys: np.ndarray, vals: np.ndarray, sm_scale: float) -> np.ndarray:
    """softmax(q K^T * sm_scale) V in float64; q [M, D], keys/vals [N, D]."""
    q = np.asarray(q, np.float64)
    s = (q @ np.asarray(keys, np.float64).T) * float(sm_scale)
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p @ np.asarray(vals, np.float64)) / p.sum(axis=1, keepdims=True)


def attend_loops(q, keys, vals, sm_scale):
    """The same softmax written as explicit loops (for brute-force checks on tiny inputs)."""
    q = np.asarray(q, np.float64)
    keys = np.asarray(keys, np.float64)
    vals = np.asarray(vals, np.float64)
    M, D = q.shape
    N = keys.shape[0]
    out = np.zeros((M, vals.shape[1]))
    for i in range(M):
        logits = []
        for j in range(N):
            acc = 0.0
            for d in range(D):
                acc += q[i, d] * keys[j, d]
            logits.append(acc * sm_scale)
        mx = max(logits)
        w = [np.exp(x - mx) for x in logits]
        tot = sum(w)
        for j in range(N):
            out[i] += (w[j] / tot) * vals[j]
    return out


def prefill_head(q16, k16, v16, is_vl, W: int, sm_scale: float, rows=None, qt=None, kt=None, vt=None):
    """Hybrid causal prefill for one query head against its kv head.

    q16 [L, D], k16/v16 [L, D] float16; is_vl [L] bool (vertical-line keys).
    ``qt/kt/vt`` are the FP8-represented real values (float64); computed from
    the FP16 inputs when not given.  Returns float64 [len(rows), D].
    """
    L = k16.shape[0]
    if rows is None:
        rows = np.arange(L)
    rows = np.asarray(rows, np.int64)
    if qt is None:
        qt = formats.fp8_dequant(formats.fp8_quantize(q16, formats.fp8_block_scales(q16)), formats.fp8_block_scales(q16))
    if kt is None:
        sk = formats.fp8_block_scales(k16)
        kt = formats.fp8_dequant(formats.fp8_quantize(k16, sk), sk)
    if vt is None:
        sv = formats.fp8_block_scales(v16)
        vt = formats.fp8_dequant(formats.fp8_quantize(v16, sv), sv)
    q64 = q16.astype(np.float64)
    k64 = k16.astype(np.float64)
    v64 = v16.astype(np.float64)
    out = np.empty((len(rows), k16.shape[1]))
    chunk = 256
    for c0 in range(0, len(rows), chunk):
        i = rows[c0:c0 + chunk]
        nk = int(i.max()) + 1
        j = np.arange(nk)
        causal = j[None, :] <= i[:, None]
        window = causal & (j[None, :] > i[:, None] - W)
        hi = window | (causal & is_vl[None, :nk])          # FP16 class
        s16 = (q64[i] @ k64[:nk].T) * sm_scale
        s8 = (qt[i] @ kt[:nk].T) * sm_scale
        s = np.where(hi, s16, s8)
        s = np.where(causal, s, -np.inf)
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        o = (p * hi) @ v64[:nk] + (p * ~hi) @ vt[:nk]
        out[c0:c0 + chunk] = o / p.sum(axis=1, keepdims=True)
    return out


def prefill_ref(Q, K, V, vl_pos, W: int, sm_scale: float, rows=None, heads=None):
    """Hybrid causal prefill, float64.

    Q [B, Hq, L, D], K/V [B, Hkv, L, D] float16; vl_pos[b][h] = vertical-line
    positions of (b, kv head h).  ``rows`` (optional) restricts the query rows
    and ``heads`` (optional) is a list of (b, hq) pairs to evaluate.
    Returns a dict {(b, hq): float64 [rows, D]}.
    """
    B, Hq, L, D = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(Hq)]
    out = {}
    cache = {}
    for (b, hq) in heads:
        kvh = hq // G
        if (b, kvh) not in cache:
            sk = formats.fp8_block_scales(K[b, kvh])
            sv = formats.fp8_block_scales(V[b, kvh])
            kt = formats.fp8_dequant(formats.fp8_quantize(K[b, kvh], sk), sk)
            vt = formats.fp8_dequant(formats.fp8_quantize(V[b, kvh], sv), sv)
            is_vl = np.zeros(L, dtype=bool)
            is_vl[np.asarray(vl_pos[b][kvh], np.int64)] = True
            cache = {(b, kvh): (kt, vt, is_vl)}
        kt, vt, is_vl = cache[(b, kvh)]
        sq = formats.fp8_block_scales(Q[b, hq])
        qt = formats.fp8_dequant(formats.fp8_quantize(Q[b, hq], sq), sq)
        out[(b, hq)] = prefill_head(Q[b, hq], K[b, kvh], V[b, kvh], is_vl, W, sm_scale, rows=rows, qt=qt, kt=kt, vt=vt)
    return out
