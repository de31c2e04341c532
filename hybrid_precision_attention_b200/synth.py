"""Seeded synthetic inputs shaped like long-context attention with vertical lines.

This module only draws random numbers; it holds none of the method's
arithmetic (no packing, no selection, no attention).  Both the CUDA path and
the CPU checker take their inputs from here, so it must stay free of either.

Workload recipe (stands in for real-model attention maps, which need trained
weights): for every (batch, kv-head) pair

* ``u``  — a random unit direction in R^D, shared by the whole GQA group;
* ``K``  — N(0, 1) entries; a planted set of positions ({0} plus
  floor(0.03 * L) positions drawn without replacement from [1, L)) gets
  ``+4 * u`` added, which makes those columns collect more attention mass from
  every query (the "vertical lines" of the HyQuant digest, coverage paragraph);
* ``V``  — N(0, 1) entries;
* every query (all heads of the group) — N(0, 1) entries plus ``1 * u``.

All arrays are drawn in float32 from ``numpy.random.default_rng([seed, tag])``
with one independent stream per tensor, then rounded to float16 (RN).  The
independent streams let a caller draw, say, only the decode-step tokens
without drawing the whole prefix.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

PLANT_FRAC = 0.03
KEY_SHIFT = 4.0
QUERY_SHIFT = 1.0

_TAG_U, _TAG_K, _TAG_PLANT, _TAG_V, _TAG_QTAIL, _TAG_QFULL, _TAG_STEPS = range(7)


def _rng(seed: int, tag: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tag)])


def directions(seed: int, B: int, Hkv: int, D: int = 128) -> np.ndarray:
    """Unit vectors ``u`` [B, Hkv, D] float32, one per (batch, kv head)."""
    u = _rng(seed, _TAG_U).standard_normal((B, Hkv, D), dtype=np.float32)
    u /= np.linalg.norm(u, axis=-1, keepdims=True)
    return u


def planted_positions(seed: int, B: int, Hkv: int, L: int) -> list:
    """Planted vertical-line positions, a sorted int64 array per (b, kv head)."""
    rng = _rng(seed, _TAG_PLANT)
    n_extra = int(PLANT_FRAC * L)
    out = []
    for _b in range(B):
        row = []
        for _h in range(Hkv):
            extra = rng.choice(np.arange(1, L), size=min(n_extra, max(L - 1, 0)), replace=False) if L > 1 else np.zeros(0, np.int64)
            row.append(np.sort(np.concatenate([[0], extra]).astype(np.int64)) if L > 0 else np.zeros(0, np.int64))
        out.append(row)
    return out


def _queries(rng: np.random.Generator, u: np.ndarray, B: int, Hq: int, n: int, D: int) -> np.ndarray:
    Hkv = u.shape[1]
    G = Hq // Hkv
    q = rng.standard_normal((B, Hq, n, D), dtype=np.float32)
    q += QUERY_SHIFT * np.repeat(u, G, axis=1)[:, :, None, :]
    return q.astype(np.float16)


@dataclass
class PlantedLayer:
    k: np.ndarray        # [B, Hkv, L, D] float16
    v: np.ndarray        # [B, Hkv, L, D] float16
    q_tail: np.ndarray   # [B, Hq, n_tail, D] float16, positions L-n_tail .. L-1
    u: np.ndarray        # [B, Hkv, D] float32
    planted: list        # planted positions per (b, kv head)


def planted_layer(seed: int, B: int, Hq: int, Hkv: int, L: int, D: int = 128, n_tail: int = 64) -> PlantedLayer:
    """One attention layer's prefix K/V plus the selection queries at its tail."""
    u = directions(seed, B, Hkv, D)
    k = _rng(seed, _TAG_K).standard_normal((B, Hkv, L, D), dtype=np.float32)
    planted = planted_positions(seed, B, Hkv, L)
    for b in range(B):
        for h in range(Hkv):
            k[b, h, planted[b][h]] += KEY_SHIFT * u[b, h]
    v = _rng(seed, _TAG_V).standard_normal((B, Hkv, L, D), dtype=np.float32)
    nq = min(n_tail, L)
    q_tail = _queries(_rng(seed, _TAG_QTAIL), u, B, Hq, nq, D)
    return PlantedLayer(k.astype(np.float16), v.astype(np.float16), q_tail, u, planted)


def full_queries(seed: int, B: int, Hq: int, Hkv: int, L: int, D: int = 128) -> np.ndarray:
    """Prefill queries [B, Hq, L, D] float16 drawn by the same rule."""
    u = directions(seed, B, Hkv, D)
    return _queries(_rng(seed, _TAG_QFULL), u, B, Hq, L, D)


def decode_tokens(seed: int, B: int, Hq: int, Hkv: int, steps: int, D: int = 128):
    """Per-step decode inputs: q [steps, B, Hq, D], k, v [steps, B, Hkv, D] float16.

    New tokens are never planted; their queries follow the same rule as the
    prefix queries.
    """
    u = directions(seed, B, Hkv, D)
    rng = _rng(seed, _TAG_STEPS)
    G = Hq // Hkv
    q = rng.standard_normal((steps, B, Hq, D), dtype=np.float32)
    q += QUERY_SHIFT * np.repeat(u, G, axis=1)[None]
    k = rng.standard_normal((steps, B, Hkv, D), dtype=np.float32)
    v = rng.standard_normal((steps, B, Hkv, D), dtype=np.float32)
    return q.astype(np.float16), k.astype(np.float16), v.astype(np.float16)


def planted_layer_device(seed: int, B: int, Hq: int, Hkv: int, L: int, device, D: int = 128, n_tail: int = 64):
    """Device-side variant of :func:`planted_layer` for layers too large to draw on the host.

    Same recipe, drawn with ``torch.Generator`` on ``device`` (different numbers
    than the host variant).  Returns torch float16 tensors (k, v, q_tail) and the
    float32 directions ``u``.
    """
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000003 + 17)
    u = torch.randn((B, Hkv, D), generator=g, device=device, dtype=torch.float32)
    u /= u.norm(dim=-1, keepdim=True)
    k = torch.randn((B, Hkv, L, D), generator=g, device=device, dtype=torch.float32)
    n_extra = int(PLANT_FRAC * L)
    if L > 1:
        # planted rows: position 0 plus n_extra distinct positions in [1, L)
        scores = torch.rand((B, Hkv, L - 1), generator=g, device=device)
        extra = scores.topk(n_extra, dim=-1).indices + 1 if n_extra > 0 else torch.zeros((B, Hkv, 0), dtype=torch.long, device=device)
        pos = torch.cat([torch.zeros((B, Hkv, 1), dtype=torch.long, device=device), extra], dim=-1)
        k.scatter_add_(2, pos[..., None].expand(-1, -1, -1, D), (KEY_SHIFT * u)[:, :, None, :].expand(-1, -1, pos.shape[-1], -1).contiguous())
    kh = k.to(torch.float16)
    del k
    v = torch.randn((B, Hkv, L, D), generator=g, device=device, dtype=torch.float32).to(torch.float16)
    G = Hq // Hkv
    nq = min(n_tail, L)
    q = torch.randn((B, Hq, nq, D), generator=g, device=device, dtype=torch.float32)
    q += QUERY_SHIFT * u.repeat_interleave(G, dim=1)[:, :, None, :]
    return kh, v, q.to(torch.float16), u
