"""Comparator between the CUDA library's index rows and the CPU oracle.

Tolerance (fp32 accumulation of bf16 inputs vs the oracle's double):
    |x_gpu - x_oracle| <= 1e-4 + 2e-3 * |x_oracle|.
A row passes iff
  * it holds exactly n valid entries (the rest -1), no duplicates, all in the
    eligible set E (this covers the causal mask and candidate membership);
  * with theta the oracle's n-th best score over E, every GPU entry outside
    the oracle's top-n has score >= theta - tol(theta), and every oracle
    entry the GPU left out has score <= theta + tol(theta) (swaps only
    between near-ties at the boundary);
  * returned scores match the oracle's within tol, elementwise.
"""
from __future__ import annotations

import numpy as np

ABS, REL = 1e-4, 2e-3


def tol(x):
    return ABS + REL * np.abs(x)


def check_row(row_idx, row_sc, elig_keys, elig_f, n, orc, what=""):
    """Returns a list of failure strings (empty when the row passes)."""
    fails = []
    row_idx = np.asarray(row_idx)
    nv = int((row_idx >= 0).sum())
    if not (row_idx[:nv] >= 0).all() or not (row_idx[nv:] == -1).all():
        fails.append(f"{what}: valid entries not first / bad padding")
        return fails
    A = row_idx[:nv].astype(np.int64)
    if nv != n:
        fails.append(f"{what}: {nv} valid entries, expected {n}")
        return fails
    if np.unique(A).size != A.size:
        fails.append(f"{what}: duplicate indices")
        return fails
    order = np.argsort(elig_keys, kind="stable")
    ks = np.asarray(elig_keys, np.int64)[order]
    fs = np.asarray(elig_f, np.float64)[order]
    pos = np.searchsorted(ks, A)
    inside = (pos < ks.size) & (ks[np.minimum(pos, ks.size - 1)] == A)
    if not inside.all():
        fails.append(f"{what}: {int((~inside).sum())} indices outside the eligible set, e.g. {A[~inside][:5]}")
        return fails
    if n == 0:
        return fails
    fa = fs[pos]
    Bk, Bv = orc.topn(fs, n, ks)
    theta = Bv[-1]
    inB = np.isin(A, Bk)
    bad_in = fa[~inB] < theta - tol(theta)
    if bad_in.any():
        fails.append(f"{what}: {int(bad_in.sum())} GPU entries below theta={theta:.6g} "
                     f"(min {fa[~inB].min():.6g})")
    missing = ~np.isin(Bk, A)
    bad_out = Bv[missing] > theta + tol(theta)
    if bad_out.any():
        fails.append(f"{what}: {int(bad_out.sum())} oracle entries above theta missing (max {Bv[missing].max():.6g})")
    if row_sc is not None:
        sc = np.asarray(row_sc, np.float64)[:nv]
        err = np.abs(sc - fa) > tol(fa)
        if err.any():
            i = int(np.argmax(np.abs(sc - fa)))
            fails.append(f"{what}: {int(err.sum())} scores off (worst gpu {sc[i]:.7g} vs oracle {fa[i]:.7g})")
    return fails


def summarize(fails, limit=12):
    return "\n".join(fails[:limit]) + (f"\n... {len(fails)} failures" if len(fails) > limit else "")
