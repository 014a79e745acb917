"""Workload diagnostics: the three observations the PIVOT paper builds on
(Introduction, "Key observations (Figure 2)"), measured on dense indexer rows.

  O1 (local)           adjacent queries' top-k overlap |T_t & T_t+1| / k, and
                       the share of top-k common to a whole group |&_G T_t| / k;
  O2 (group-shareable) the group's top-k union |U_G T_t| / k;
  O3 (sparse)          cumulative share of the (ReLU-weighted, positive) score
                       mass held by a row's best m keys, at m = k/4, k/2, 3k/4, k.

Host-side analysis of index / score rows (numpy); the rows themselves come
from the library's dense indexer (or the oracle).  Rows are -1 padded; only
rows whose prefix holds at least k keys count.
"""
from __future__ import annotations

from typing import Dict, Iterable, Sequence

import numpy as np


def _full_rows(idx: np.ndarray, k: int) -> np.ndarray:
    """Row positions t whose prefix has >= k keys (t + 1 >= k)."""
    L = idx.shape[0]
    return np.arange(k - 1, L)


def adjacent_overlap(idx: np.ndarray, k: int) -> float:
    """O1: mean over t of |T_t & T_{t+1}| / k (rows t, t+1 both full)."""
    rows = _full_rows(idx, k)
    rows = rows[rows + 1 < idx.shape[0]]
    if rows.size == 0:
        return float("nan")
    vals = [np.intersect1d(idx[t], idx[t + 1], assume_unique=True).size / k for t in rows]
    return float(np.mean(vals))


def _groups(idx: np.ndarray, k: int, g: int) -> Iterable[np.ndarray]:
    L = idx.shape[0]
    for i in range(L // g):
        t0 = i * g
        if t0 + 1 >= k:  # every member full
            yield idx[t0:t0 + g]


def group_intersection(idx: np.ndarray, k: int, g: int) -> float:
    """O1 across a group: mean over full groups of |&_{t in G} T_t| / k."""
    vals = []
    for rows in _groups(idx, k, g):
        common = rows[0]
        for r in rows[1:]:
            common = np.intersect1d(common, r, assume_unique=True)
        vals.append(common.size / k)
    return float(np.mean(vals)) if vals else float("nan")


def group_union(idx: np.ndarray, k: int, g: int) -> float:
    """O2: mean over full groups of |U_{t in G} T_t| / k (between 1 and g)."""
    vals = [np.unique(rows).size / k for rows in _groups(idx, k, g)]
    return float(np.mean(vals)) if vals else float("nan")


def score_mass(scores: np.ndarray, ms: Sequence[int]) -> Dict[int, float]:
    """O3: rows of a query's scores over its whole prefix, in any order (NaN /
    -inf padded); for each m, the mean over rows of the share of the positive
    score mass held by the best m scores."""
    s = np.where(np.isfinite(scores), scores, 0.0)
    s = -np.sort(-np.maximum(s, 0.0), axis=1)  # descending
    total = s.sum(axis=1)
    keep = total > 0
    csum = np.cumsum(s[keep], axis=1)
    out = {}
    for m in ms:
        m_ = min(m, s.shape[1])
        out[int(m)] = float(np.mean(csum[:, m_ - 1] / total[keep])) if keep.any() else float("nan")
    return out


def summary(idx: np.ndarray, k: int, full_scores: np.ndarray = None,
            gs: Sequence[int] = (4, 8, 16)) -> dict:
    """All three observations for one sequence's dense rows."""
    out = {"k": k, "O1_adjacent_overlap": adjacent_overlap(idx, k),
           "O1_group4_common": group_intersection(idx, k, 4),
           "O2_union_over_k": {g: group_union(idx, k, g) for g in gs}}
    if full_scores is not None:
        out["O3_mass_at"] = score_mass(full_scores, (k // 4, k // 2, 3 * k // 4, k))
    return out


__all__ = ["adjacent_overlap", "group_intersection", "group_union", "score_mass", "summary"]
