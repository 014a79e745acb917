"""ctypes wrapper of the plain-C double-precision PIVOT oracle (pivot_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
CPU-baseline leg may import this module; the library's product path never
does.  Inputs are the same host arrays handed to the GPU (bf16 as uint16 bit
patterns, or float32).

Parity unpinned by the pages (conventions, see the C file's header): the
bf16 rounding of the pooled query, and the decode member positions.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pivot_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile pivot_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.orc_dense.argtypes = [P, P, P, I32, I64, I32, I32, I32, I64, I64, P, P]
        L.orc_reuse.argtypes = [P, P, P, I32, I64, I32, I32, I32, I32, I64, I64, P, P]
        L.orc_refine.argtypes = [P, P, P, I32, I64, I32, I32, I32, I32, I32, I64, I64, P, P, P, P, P]
        L.orc_decode.argtypes = [P, P, P, P, I32, I32, I32, I32, I32, I32, I32, I64, I64, P, P, P,
                                 P, P]
        L.orc_proxy.argtypes = [P, P, I32, I32, I32, P, I32, P, P]
        L.orc_query_row.argtypes = [P, P, I32, I32, I32, I64, P, P]
        L.orc_scores.argtypes = [P, P, I32, I32, P, I32, P, I64, I64, P]
        L.orc_proxy_scores.argtypes = [P, P, P, I32, I64, I32, I32, I32, I64, P]
        L.orc_proxy_scores.restype = I64
        L.orc_scores_batch.argtypes = [P, P, I64, I32, I32, P, I32, P, P, P, I64, P]
        L.orc_topn.argtypes = [P, P, I64, I64, P, P]
        L.orc_topn.restype = I64
        L.orc_threads.restype = I32
        L.orc_set_threads.argtypes = [I32]
        L.orc_set_aggregation.argtypes = [I32]
        _ = D
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dt(arr: np.ndarray) -> int:
    if arr.dtype == np.uint16:
        return 0
    if arr.dtype == np.float32:
        return 1
    raise TypeError(f"q/k must be uint16 (bf16 bits) or float32, got {arr.dtype}")


def _c(a, dtype=None):
    return np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))


def threads() -> int:
    return int(lib().orc_threads())


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


AGGREGATION = {"mean": 0, "first": 1, "last": 2}


def set_aggregation(mode: str) -> None:
    """Proxy aggregation of the PIVOT calls that follow: "mean" (Eq. 4), "first" or "last"."""
    lib().orc_set_aggregation(AGGREGATION[mode])


def dense(q, w, k, topk, t0=0, t1=None):
    """Eq. (1) + TopK for query rows [t0, t1).  Returns (idx int32, scores f64) [(t1-t0), topk]."""
    q, w, k = _c(q), _c(w, np.float32), _c(k)
    L, H, d = q.shape
    t1 = L if t1 is None else t1
    idx = np.empty((t1 - t0, topk), np.int32)
    val = np.empty((t1 - t0, topk), np.float64)
    lib().orc_dense(_p(q), _p(w), _p(k), _dt(q), L, H, d, topk, t0, t1, _p(idx), _p(val))
    return idx, val


def reuse(q, w, k, topk, g, g0=0, g1=None):
    """Eq. (4)-(6) for prefill groups [g0, g1).  Rows are the groups' member positions."""
    q, w, k = _c(q), _c(w, np.float32), _c(k)
    L, H, d = q.shape
    G = (L + g - 1) // g
    g1 = G if g1 is None else g1
    rows = min(g1 * g, L) - g0 * g
    idx = np.empty((rows, topk), np.int32)
    val = np.empty((rows, topk), np.float64)
    lib().orc_reuse(_p(q), _p(w), _p(k), _dt(q), L, H, d, topk, g, g0, g1, _p(idx), _p(val))
    return idx, val


def refine(q, w, k, topk, c, g, g0=0, g1=None, cand_in=None):
    """Eq. (4),(5),(7)-(9) for prefill groups [g0, g1).

    Returns (idx, scores, cand, cand_scores); cand/cand_scores are the oracle's
    C_i in rank order ([(g1-g0), c], -1 / NaN padded).  With ``cand_in`` the
    given sets replace C_i (cand_scores is then NaN)."""
    q, w, k = _c(q), _c(w, np.float32), _c(k)
    L, H, d = q.shape
    G = (L + g - 1) // g
    g1 = G if g1 is None else g1
    rows = min(g1 * g, L) - g0 * g
    idx = np.empty((rows, topk), np.int32)
    val = np.empty((rows, topk), np.float64)
    cand = np.empty((g1 - g0, c), np.int32)
    cval = np.empty((g1 - g0, c), np.float64)
    ci = None if cand_in is None else _c(cand_in, np.int32)
    lib().orc_refine(_p(q), _p(w), _p(k), _dt(q), L, H, d, topk, c, g, g0, g1, _p(ci), _p(idx),
                     _p(val), _p(cand), _p(cval))
    return idx, val, cand, cval


def decode(q, w, kc, offsets, topk, c, g, variant, b0=0, b1=None, cand_in=None):
    """Eq. (3)-(9) for an MTP decode batch; variant 0 = Reuse, 1 = Refine."""
    q, w, kc = _c(q), _c(w, np.float32), _c(kc)
    off = _c(offsets, np.int64)
    B = off.size - 1
    b1 = B if b1 is None else b1
    H, d = q.shape[1], q.shape[2]
    idx = np.empty(((b1 - b0) * g, topk), np.int32)
    val = np.empty(((b1 - b0) * g, topk), np.float64)
    cand = np.empty((b1 - b0, c), np.int32)
    cval = np.empty((b1 - b0, c), np.float64)
    ci = None if cand_in is None else _c(cand_in, np.int32)
    lib().orc_decode(_p(q), _p(w), _p(kc), _p(off), _dt(q), H, d, topk, c, g, variant, b0, b1,
                     _p(ci), _p(idx), _p(val), _p(cand), _p(cval))
    return idx, val, cand, cval


def query_row(q, w, row):
    """Widened (double) query row q[row] [H*d] and w[row] [H]."""
    q, w = _c(q), _c(w, np.float32)
    _, H, d = q.shape
    qv = np.empty(H * d, np.float64)
    wv = np.empty(H, np.float64)
    lib().orc_query_row(_p(q), _p(w), _dt(q), H, d, row, _p(qv), _p(wv))
    return qv, wv


def proxy(q, w, rows):
    """Eq. (4) over the given member rows: (q-bar rounded to the input dtype, w-bar), as doubles."""
    q, w = _c(q), _c(w, np.float32)
    _, H, d = q.shape
    r = _c(np.asarray(rows), np.int64)
    qb = np.empty(H * d, np.float64)
    wb = np.empty(H, np.float64)
    lib().orc_proxy(_p(q), _p(w), _dt(q), H, d, _p(r), r.size, _p(qb), _p(wb))
    return qb, wb


def scores(qv, wv, k, keys=None, key_lo=0, n=None, H=None, d=None):
    """Eq. (1)/(5)/(8) score of one (query or proxy) [H*d], [H] against key rows."""
    k = _c(k)
    d = k.shape[1] if d is None else d
    H = wv.size if H is None else H
    qv, wv = _c(qv, np.float64), _c(wv, np.float64)
    kk = None if keys is None else _c(np.asarray(keys), np.int64)
    n = (kk.size if kk is not None else k.shape[0] - key_lo) if n is None else n
    out = np.empty(n, np.float64)
    lib().orc_scores(_p(qv), _p(wv), H, d, _p(k), _dt(k), _p(kk), key_lo, n, _p(out))
    return out


def proxy_scores(q, w, k, g, i):
    """Eq. (4)+(5): proxy scores of prefill group i over s <= e_i."""
    q, w, k = _c(q), _c(w, np.float32), _c(k)
    L, H, d = q.shape
    e = min(i * g + g, L) - 1
    out = np.empty(e + 1, np.float64)
    lib().orc_proxy_scores(_p(q), _p(w), _p(k), _dt(q), L, H, d, g, i, _p(out))
    return out


def topn(f, n, idx=None):
    """TopK by full sort (score desc, index asc): returns (key indices, scores) in rank order."""
    f = _c(f, np.float64)
    ii = None if idx is None else _c(np.asarray(idx), np.int64)
    out = np.empty(max(1, min(n, f.size)), np.int64)
    val = np.empty_like(out, dtype=np.float64)
    cnt = lib().orc_topn(_p(f), _p(ii), f.size, n, _p(out), _p(val))
    return out[:cnt], val[:cnt]


def scores_batch(qv, wv, k, key_rows=None, plen=None, key_base=None, m=None):
    """Scores of n vectors against key lists (key_rows [n,m], -1 = none) or
    prefixes (plen [n]); returns [n, m] float64 with NaN where undefined."""
    k = _c(k)
    qv, wv = _c(qv, np.float64), _c(wv, np.float64)
    n, H = wv.shape
    d = k.shape[1]
    kr = None if key_rows is None else _c(key_rows, np.int64)
    pl = None if plen is None else _c(plen, np.int64)
    kb = None if key_base is None else _c(key_base, np.int64)
    if m is None:
        m = kr.shape[1] if kr is not None else int(pl.max())
    out = np.empty((n, m), np.float64)
    lib().orc_scores_batch(_p(qv), _p(wv), n, H, d, _p(k), _dt(k), _p(kb), _p(kr), _p(pl), m, _p(out))
    return out


def query_rows(q, w, rows):
    """Widened query rows: ([n, H*d], [n, H]) doubles."""
    rows = list(rows)
    _, H, d = q.shape
    qv = np.empty((len(rows), H * d), np.float64)
    wv = np.empty((len(rows), H), np.float64)
    for i, r in enumerate(rows):
        qv[i], wv[i] = query_row(q, w, int(r))
    return qv, wv


def proxies(q, w, member_lists):
    """Eq. (4) proxies of several groups: ([n, H*d], [n, H]) doubles."""
    _, H, d = q.shape
    qv = np.empty((len(member_lists), H * d), np.float64)
    wv = np.empty((len(member_lists), H), np.float64)
    for i, rows in enumerate(member_lists):
        qv[i], wv[i] = proxy(q, w, rows)
    return qv, wv
