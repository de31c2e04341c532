"""Vertical-line selection: column-mass scores and the top-rho set.

TEST INFRASTRUCTURE ONLY (see the package docstring).

HyQuant digest (agihunt.info, method paragraph): key positions are split into
a vertical-line set, the most recent fixed window and the quantised rest; the
vertical-line score of a key is the accumulated attention mass along its
column; the set is the top-rho (default 5 %) of the non-window prefix; it is
recomputed every 64 tokens from at most 64 cached FP16 query vectors.  The
README (Overview item 1) calls it a running column-mass score; this oracle
recomputes it at each reselection from the buffered queries.

Definitions used here, per (batch, kv head):

* buffered queries ``q_i`` (every query head of the GQA group, every buffered
  position ``p_i``), keys ``k_j`` in their current representation;
* ``a_{h,i,j} = softmax_j( q_{h,i} . k_j * sm_scale )`` over ``j <= p_i``;
* ``score_j = sum_{h,i} a_{h,i,j}`` for ``j`` in the non-window prefix
  ``[0, n)``, ``n = T - W``;
* ``k = ceil(rho * n)`` computed in integer basis points,
  ``k = (n * rho_bp + 9999) // 10000`` (so 5 % of 32640 is exactly 1632);
* the set is the ``k`` largest scores, ties going to the lower position,
  reported in ascending position order.
"""
from __future__ import annotations

import numpy as np


def k_of(n: int, rho_bp: int) -> int:
    """Number of vertical lines for a non-window prefix of ``n`` positions."""
    if n <= 0 or rho_bp <= 0:
        return 0
    return min(int(n), (int(n) * int(rho_bp) + 9999) // 10000)


def column_mass(keys: np.ndarray, queries: np.ndarray, qpos: np.ndarray, n: int, sm_scale: float) -> np.ndarray:
    """Column-mass scores (float64 [n]).

    keys     [Lk, D] float64 — keys 0 .. Lk-1 in their current representation
    queries  [M, D]  float64 — all buffered queries of the group (heads x positions)
    qpos     [M]     int     — position of each query; key j is visible iff j <= qpos
    """
    keys = np.asarray(keys, np.float64)
    queries = np.asarray(queries, np.float64)
    qpos = np.asarray(qpos, np.int64)
    Lk = keys.shape[0]
    if n <= 0:
        return np.zeros(0)
    s = (queries @ keys.T) * float(sm_scale)
    visible = np.arange(Lk)[None, :] <= qpos[:, None]
    s = np.where(visible, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    a = p / p.sum(axis=1, keepdims=True)
    return a[:, :n].sum(axis=0)


def topk_stable(scores: np.ndarray, k: int) -> np.ndarray:
    """Positions of the k largest scores (ties -> lower position), ascending."""
    scores = np.asarray(scores)
    if k <= 0:
        return np.zeros(0, dtype=np.int64)
    order = np.argsort(-scores, kind="stable")[:k]
    return np.sort(order).astype(np.int64)


def select_vlines(keys, queries, qpos, n: int, rho_bp: int, sm_scale: float):
    """Scores and the selected set for one (batch, kv head)."""
    sc = column_mass(keys, queries, qpos, n, sm_scale)
    return topk_stable(sc, k_of(n, rho_bp)), sc
