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
  scales (see ``formats``), or, with ``qk_format="int8"`` (the README's
  INT8-QK / FP16-PV kernels), INT8 Q and K with per-block scales and FP16 V;

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


def low_precision(x16, fmt: str):
    """The real values a quantised tile holds for x16 [..., L, D] (float64): e4m3
    or int8 codes times their per-block scales."""
    if fmt == "int8":
        s = formats.int8_block_scales(x16)
        return formats.fp8_dequant(formats.int8_quantize(x16, s), s)
    s = formats.fp8_block_scales(x16)
    return formats.fp8_dequant(formats.fp8_quantize(x16, s), s)


def prefill_head(q16, k16, v16, is_vl, W: int, sm_scale: float, rows=None, qt=None, kt=None, vt=None,
                 qk_format: str = "e4m3"):
    """Hybrid causal prefill for one query head against its kv head.

    q16 [L, D], k16/v16 [L, D] float16; is_vl [L] bool (vertical-line keys).
    ``qt/kt/vt`` are the low-precision real values (float64) of the quantised
    tiles, computed from the FP16 inputs when not given: e4m3 Q, K, V, or with
    ``qk_format="int8"`` INT8 Q, K and FP16 V.  Returns float64 [len(rows), D].
    """
    assert qk_format in ("e4m3", "int8")
    L = k16.shape[0]
    if rows is None:
        rows = np.arange(L)
    rows = np.asarray(rows, np.int64)
    if qt is None:
        qt = low_precision(q16, qk_format)
    if kt is None:
        kt = low_precision(k16, qk_format)
    if vt is None:
        vt = low_precision(v16, "e4m3") if qk_format == "e4m3" else np.asarray(v16, np.float64)
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


def prefill_ref(Q, K, V, vl_pos, W: int, sm_scale: float, rows=None, heads=None, qk_format: str = "e4m3"):
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
            kt = low_precision(K[b, kvh], qk_format)
            vt = low_precision(V[b, kvh], "e4m3") if qk_format == "e4m3" else V[b, kvh].astype(np.float64)
            is_vl = np.zeros(L, dtype=bool)
            is_vl[np.asarray(vl_pos[b][kvh], np.int64)] = True
            cache = {(b, kvh): (kt, vt, is_vl)}
        kt, vt, is_vl = cache[(b, kvh)]
        qt = low_precision(Q[b, hq], qk_format)
        out[(b, hq)] = prefill_head(Q[b, hq], K[b, kvh], V[b, kvh], is_vl, W, sm_scale, rows=rows, qt=qt, kt=kt, vt=vt,
                                    qk_format=qk_format)
    return out
