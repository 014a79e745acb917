"""PIVOT group-shared sparse-attention indexer for NVIDIA B200 (sm_100a).

Thin ctypes binding of ``libpivot.so`` (the C ABI in ``include/pivot.h``).
It only marshals arguments: every step of the indexer runs in the library's
CUDA kernels.  PyTorch provides device memory and streams.  There is no CPU
fallback: if the library is missing or a CUDA device is absent, calls raise.

PIVOT (picx.dev summary of the paper, Methodology, Eq. 1-9): the dense DSA
indexer scores I_{t,s} = sum_j w_{t,j} ReLU(q_{t,j} . k_s) and keeps the top k
keys per query; PIVOT pools each group of g queries into a mean proxy, scans
the prefix once per group, and either reuses the proxy top-k (Reuse) or
re-scores the proxy top-c per member (Refine).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpivot.so")

OP_DENSE, OP_REUSE, OP_REFINE = 0, 1, 2
BF16, F32 = 0, 1

STATUS = {
    0: "PIVOT_OK",
    1: "PIVOT_ERR_INVALID_ARG",
    2: "PIVOT_ERR_UNSUPPORTED_SHAPE",
    3: "PIVOT_ERR_WORKSPACE_TOO_SMALL",
    4: "PIVOT_ERR_CUDA",
    5: "PIVOT_ERR_DEVICE_TIMEOUT",
    6: "PIVOT_ERR_DEVICE_BOUNDS",
}

# every symbol include/pivot.h declares
EXPORTS = (
    "pivot_workspace_size", "pivot_indexer_dense", "pivot_reuse", "pivot_refine",
    "pivot_varlen_workspace_size", "pivot_reuse_varlen", "pivot_refine_varlen",
    "pivot_last_device_status", "pivot_status_string", "pivot_last_cuda_error", "pivot_path",
    "pivot_set_device_timeout_ns", "pivot_set_debug_flags", "pivot_set_profile_events", "pivot_version",
    "pivot_reuse_noalloc", "pivot_guardrail_dense", "pivot_reuse_guarded", "pivot_refine_guarded",
    "pivot_reuse_agg", "pivot_refine_agg", "pivot_indexer_dense_range", "pivot_reuse_range",
    "pivot_refine_range", "pivot_refine_host_workspace_size", "pivot_refine_host",
    "pivot_decode_shard_workspace_size", "pivot_decode_shard_select", "pivot_decode_merge_workspace_size",
    "pivot_decode_merge",
    "pivot_decode_shard_rescore", "pivot_decode_rowselect",
)

# proxy aggregation (PIVOT paper, Ablation Studies, Proxy aggregation, Table 2)
AGGREGATION = {"mean": 0, "first": 1, "last": 2}


class PivotError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}" + (f" ({detail})" if detail else ""))


_lib = None


def lib() -> ctypes.CDLL:
    """Load libpivot.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m top_token_selection_proxy_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        L.pivot_workspace_size.argtypes = [I, I64, I, I, I, I, I, I]
        L.pivot_workspace_size.restype = SZ
        L.pivot_varlen_workspace_size.argtypes = [I, I, P, I, I, I, I, I, I]
        L.pivot_varlen_workspace_size.restype = SZ
        L.pivot_indexer_dense.argtypes = [P, P, P, I64, I, I, I, I, P, P, P, SZ, P]
        L.pivot_reuse.argtypes = [P, P, P, I64, I, I, I, I, I, P, P, P, SZ, P]
        L.pivot_refine.argtypes = [P, P, P, I64, I, I, I, I, I, I, P, P, P, P, P, SZ, P]
        L.pivot_reuse_varlen.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, P, P, SZ, P]
        L.pivot_refine_varlen.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, P, P, SZ, P]
        L.pivot_indexer_dense_range.argtypes = [P, P, P, I64, I, I, I, I, I64, I64, P, P, P, SZ, P]
        L.pivot_reuse_range.argtypes = [P, P, P, I64, I, I, I, I, I, I64, I64, P, P, P, SZ, P]
        L.pivot_refine_range.argtypes = [P, P, P, I64, I, I, I, I, I, I, I64, I64, P, P, P, P, P, SZ, P]
        L.pivot_reuse_agg.argtypes = [P, P, P, I64, I, I, I, I, I, I, P, P, P, SZ, P]
        L.pivot_refine_agg.argtypes = [P, P, P, I64, I, I, I, I, I, I, I, P, P, P, P, P, SZ, P]
        L.pivot_refine_host_workspace_size.argtypes = [I64, I, I, I, I, I]
        L.pivot_refine_host_workspace_size.restype = SZ
        L.pivot_refine_host.argtypes = [P, P, P, I64, I, I, I, I, I, I, P, P, SZ, P]
        L.pivot_refine_host.restype = I
        L.pivot_guardrail_dense.argtypes = [I, I64, I, I]
        L.pivot_guardrail_dense.restype = I
        L.pivot_reuse_guarded.argtypes = [P, P, P, I64, I, I, I, I, I, P, P, P, SZ, P, P]
        L.pivot_refine_guarded.argtypes = [P, P, P, I64, I, I, I, I, I, I, P, P, P, P, P, SZ, P, P]
        L.pivot_decode_shard_workspace_size.argtypes = [I, I, P, I, I, I, I, I]
        L.pivot_decode_shard_workspace_size.restype = SZ
        L.pivot_decode_shard_select.argtypes = [I, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, SZ, P]
        L.pivot_decode_merge_workspace_size.argtypes = [I, I, I, I, I, I]
        L.pivot_decode_merge_workspace_size.restype = SZ
        L.pivot_decode_merge.argtypes = [I, P, I, P, P, I, I, I, I, P, P, P, P, P, P, P, P, SZ, P]
        L.pivot_decode_shard_rescore.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, SZ, P]
        L.pivot_decode_rowselect.argtypes = [P, P, P, I, I, I, I, P, P, P]
        for f in ("pivot_decode_shard_select", "pivot_decode_merge", "pivot_decode_shard_rescore",
                  "pivot_decode_rowselect"):
            getattr(L, f).restype = I
        for f in ("pivot_indexer_dense", "pivot_reuse", "pivot_refine", "pivot_reuse_varlen",
                  "pivot_refine_varlen", "pivot_last_device_status", "pivot_reuse_guarded",
                  "pivot_refine_guarded", "pivot_reuse_agg", "pivot_refine_agg", "pivot_indexer_dense_range",
                  "pivot_reuse_range", "pivot_refine_range"):
            getattr(L, f).restype = I
        L.pivot_last_device_status.argtypes = [P, P]
        L.pivot_status_string.argtypes = [I]
        L.pivot_status_string.restype = ctypes.c_char_p
        L.pivot_last_cuda_error.restype = ctypes.c_char_p
        L.pivot_path.argtypes = [I, I64, I, I, I, I, I, I]
        L.pivot_path.restype = I
        L.pivot_set_device_timeout_ns.argtypes = [ctypes.c_uint64]
        L.pivot_set_debug_flags.argtypes = [I]
        L.pivot_set_profile_events.argtypes = [P, I]
        L.pivot_version.restype = I
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"q/k must be bfloat16 or float32, got {t.dtype}")


def _check(st: int, where: str):
    if st != 0:
        raise PivotError(st, where, lib().pivot_last_cuda_error().decode())


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


class Workspace:
    """Caller-owned scratch for the library (a torch uint8 buffer that grows on demand)."""

    def __init__(self, device=None):
        self.device = device
        self.buf: Optional[torch.Tensor] = None

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device or "cuda")
        return self.buf


_default_ws: dict = {}


def _ws_for(ws: Optional[Workspace], dev) -> Workspace:
    if ws is not None:
        return ws
    key = str(dev)
    if key not in _default_ws:
        _default_ws[key] = Workspace(dev)
    return _default_ws[key]


def workspace_size(op: int, L: int, H: int, d: int, k: int, c: int, g: int, dtype: int = BF16) -> int:
    return int(lib().pivot_workspace_size(op, L, H, d, k, c, g, dtype))


def varlen_workspace_size(op: int, offsets_host, H: int, d: int, k: int, c: int, g: int, dtype: int = BF16) -> int:
    off = torch.as_tensor(offsets_host, dtype=torch.int64).contiguous()
    return int(lib().pivot_varlen_workspace_size(op, off.numel() - 1, ctypes.c_void_p(off.data_ptr()), H, d, k, c,
                                                 g, dtype))


def path(op: int, L: int, H: int, d: int, k: int, c: int, g: int, dtype: int = BF16) -> int:
    """1 = tcgen05 tensor-core path, 0 = CUDA-core path, -1 = rejected."""
    return int(lib().pivot_path(op, L, H, d, k, c, g, dtype))


def _prefill_common(q, w, k):
    _need_cuda(q, w, k)
    if q.dim() != 3 or w.dim() != 2 or k.dim() != 2:
        raise ValueError("expected q [L,H,d], w [L,H], k [L,d]")
    L, H, d = q.shape
    if w.shape != (L, H) or k.shape != (L, d) or w.dtype != torch.float32 or k.dtype != q.dtype:
        raise ValueError("shape/dtype mismatch between q, w and k")
    return L, H, d, _dt(q)


def indexer_dense(q, w, k, topk: int, *, scores: bool = False, out=None, ws: Optional[Workspace] = None,
                  stream=None):
    """Eq. (1): dense indexer.  Returns (indices [L,topk] int32, scores [L,topk] f32 or None)."""
    L, H, d, dt = _prefill_common(q, w, k)
    idx = out if out is not None else torch.empty((L, topk), dtype=torch.int32, device=q.device)
    sc = torch.empty((L, topk), dtype=torch.float32, device=q.device) if scores else None
    nbytes = workspace_size(OP_DENSE, L, H, d, topk, topk, 1, dt)
    W = _ws_for(ws, q.device).get(nbytes)
    _check(lib().pivot_indexer_dense(_ptr(q), _ptr(w), _ptr(k), L, H, d, dt, topk, _ptr(idx), _ptr(sc), _ptr(W),
                                     W.numel(), _stream(stream)), "pivot_indexer_dense")
    return idx, sc


def reuse(q, w, k, topk: int, g: int, *, scores: bool = False, out=None, ws: Optional[Workspace] = None,
          stream=None, aggregation: str = "mean"):
    """Eq. (4)-(6): PIVOT-Reuse.  Returns (indices, proxy scores or None).
    ``aggregation``: "mean" (Eq. 4), "first" or "last" query proxy."""
    L, H, d, dt = _prefill_common(q, w, k)
    idx = out if out is not None else torch.empty((L, topk), dtype=torch.int32, device=q.device)
    sc = torch.empty((L, topk), dtype=torch.float32, device=q.device) if scores else None
    nbytes = workspace_size(OP_REUSE, L, H, d, topk, topk, g, dt)
    W = _ws_for(ws, q.device).get(nbytes)
    if aggregation == "mean":
        _check(lib().pivot_reuse(_ptr(q), _ptr(w), _ptr(k), L, H, d, dt, topk, g, _ptr(idx), _ptr(sc), _ptr(W),
                                 W.numel(), _stream(stream)), "pivot_reuse")
    else:
        _check(lib().pivot_reuse_agg(_ptr(q), _ptr(w), _ptr(k), L, H, d, dt, topk, g, AGGREGATION[aggregation],
                                     _ptr(idx), _ptr(sc), _ptr(W), W.numel(), _stream(stream)), "pivot_reuse_agg")
    return idx, sc


def refine(q, w, k, topk: int, c: int, g: int, *, scores: bool = False, cand=False, out=None,
           ws: Optional[Workspace] = None, stream=None, aggregation: str = "mean"):
    """Eq. (4),(5),(7)-(9): PIVOT-Refine.  Returns (indices, member scores|None, C|None, C scores|None).

    `cand` is False, True (allocate C) or a contiguous int32 [G, c] device tensor
    that receives C (any 4-byte aligned address)."""
    L, H, d, dt = _prefill_common(q, w, k)
    G = (L + g - 1) // g
    idx = out if out is not None else torch.empty((L, topk), dtype=torch.int32, device=q.device)
    sc = torch.empty((L, topk), dtype=torch.float32, device=q.device) if scores else None
    if isinstance(cand, torch.Tensor):
        if cand.dtype != torch.int32 or tuple(cand.shape) != (G, c) or not cand.is_contiguous() \
                or cand.device != q.device:
            raise ValueError("cand must be a contiguous int32 [G, c] tensor on q's device")
        cd = cand
    else:
        cd = torch.empty((G, c), dtype=torch.int32, device=q.device) if cand else None
    cs = torch.empty((G, c), dtype=torch.float32, device=q.device) if (cd is not None and scores) else None
    nbytes = workspace_size(OP_REFINE, L, H, d, topk, c, g, dt)
    W = _ws_for(ws, q.device).get(nbytes)
    if aggregation == "mean":
        _check(lib().pivot_refine(_ptr(q), _ptr(w), _ptr(k), L, H, d, dt, topk, c, g, _ptr(idx), _ptr(sc),
                                  _ptr(cd), _ptr(cs), _ptr(W), W.numel(), _stream(stream)), "pivot_refine")
    else:
        _check(lib().pivot_refine_agg(_ptr(q), _ptr(w), _ptr(k), L, H, d, dt, topk, c, g, AGGREGATION[aggregation],
                                      _ptr(idx), _ptr(sc), _ptr(cd), _ptr(cs), _ptr(W), W.numel(),
                                      _stream(stream)), "pivot_refine_agg")
    return idx, sc, cd, cs


def _range_common(q_rows, w_rows, k_prefix, L, g, g0, g1):
    _need_cuda(q_rows, w_rows, k_prefix)
    if q_rows.dim() != 3 or w_rows.shape != q_rows.shape[:2] or k_prefix.shape[1] != q_rows.shape[2]:
        raise ValueError("expected q_rows [rows, H, d], w_rows [rows, H], k_prefix [keys, d]")
    r0, r1 = g0 * g, min(g1 * g, L)
    if q_rows.shape[0] != r1 - r0 or k_prefix.shape[0] < r1:
        raise ValueError(f"groups [{g0}, {g1}) need {r1 - r0} query rows and {r1} key rows")
    return q_rows.shape[1], q_rows.shape[2], _dt(q_rows), r1 - r0


def indexer_dense_range(q_rows, w_rows, k_prefix, L: int, topk: int, t0: int, t1: int, *, scores: bool = False,
                        ws: Optional[Workspace] = None, stream=None):
    """Eq. (1) + TopK for query rows [t0, t1) of a length-L sequence (rows given, keys 0..t1-1)."""
    H, d, dt, n = _range_common(q_rows, w_rows, k_prefix, L, 1, t0, t1)
    idx = torch.empty((n, topk), dtype=torch.int32, device=q_rows.device)
    sc = torch.empty((n, topk), dtype=torch.float32, device=q_rows.device) if scores else None
    W = _ws_for(ws, q_rows.device).get(workspace_size(OP_DENSE, L, H, d, topk, topk, 1, dt))
    _check(lib().pivot_indexer_dense_range(_ptr(q_rows), _ptr(w_rows), _ptr(k_prefix), L, H, d, dt, topk, t0, t1,
                                           _ptr(idx), _ptr(sc), _ptr(W), W.numel(), _stream(stream)),
           "pivot_indexer_dense_range")
    return idx, sc


def reuse_range(q_rows, w_rows, k_prefix, L: int, topk: int, g: int, g0: int, g1: int, *, scores: bool = False,
                ws: Optional[Workspace] = None, stream=None):
    """PIVOT-Reuse for groups [g0, g1) of a length-L sequence (their rows given, keys 0..min(g1*g, L)-1)."""
    H, d, dt, n = _range_common(q_rows, w_rows, k_prefix, L, g, g0, g1)
    idx = torch.empty((n, topk), dtype=torch.int32, device=q_rows.device)
    sc = torch.empty((n, topk), dtype=torch.float32, device=q_rows.device) if scores else None
    W = _ws_for(ws, q_rows.device).get(workspace_size(OP_REUSE, L, H, d, topk, topk, g, dt))
    _check(lib().pivot_reuse_range(_ptr(q_rows), _ptr(w_rows), _ptr(k_prefix), L, H, d, dt, topk, g, g0, g1,
                                   _ptr(idx), _ptr(sc), _ptr(W), W.numel(), _stream(stream)), "pivot_reuse_range")
    return idx, sc


def refine_range(q_rows, w_rows, k_prefix, L: int, topk: int, c: int, g: int, g0: int, g1: int, *,
                 scores: bool = False, cand: bool = False, ws: Optional[Workspace] = None, stream=None):
    """PIVOT-Refine for groups [g0, g1) of a length-L sequence.  Returns (indices, scores, C, C scores)."""
    H, d, dt, n = _range_common(q_rows, w_rows, k_prefix, L, g, g0, g1)
    idx = torch.empty((n, topk), dtype=torch.int32, device=q_rows.device)
    sc = torch.empty((n, topk), dtype=torch.float32, device=q_rows.device) if scores else None
    cd = torch.empty((g1 - g0, c), dtype=torch.int32, device=q_rows.device) if cand else None
    cs = torch.empty((g1 - g0, c), dtype=torch.float32, device=q_rows.device) if (cand and scores) else None
    W = _ws_for(ws, q_rows.device).get(workspace_size(OP_REFINE, L, H, d, topk, c, g, dt))
    _check(lib().pivot_refine_range(_ptr(q_rows), _ptr(w_rows), _ptr(k_prefix), L, H, d, dt, topk, c, g, g0, g1,
                                    _ptr(idx), _ptr(sc), _ptr(cd), _ptr(cs), _ptr(W), W.numel(), _stream(stream)),
           "pivot_refine_range")
    return idx, sc, cd, cs


def group_chunks(L: int, g: int, chunks: int):
    """[(t0, t1)]: rows [0, L) cut into at most `chunks` runs of whole groups of g."""
    if L <= 0 or g <= 0 or chunks <= 0:
        raise ValueError("L, g and chunks must be positive")
    G = (L + g - 1) // g
    per = (G + chunks - 1) // chunks
    return [(i * g, min(L, (i + per) * g)) for i in range(0, G, per)]


def refine_host(q_host, w_host, k_host, topk: int, c: int, g: int, *, out_host, chunks: int = 8,
                ws: Optional[Workspace] = None, device=None, stream=None):
    """PIVOT-Refine of one prefill sequence held in pinned host memory (pivot_refine_host).

    q_host [L, H, d] bf16, w_host [L, H] fp32, k_host [L, d] bf16 and out_host [L, topk] int32
    are pinned CPU tensors.  The library copies the keys and weights, then the queries in
    `chunks` runs of whole groups (from the sequence's end to its start, heaviest first),
    indexes each run with the group-range call as soon as it has landed and copies its rows
    back while later runs are still in flight.  The rows equal
    those of one `refine` call.  Asynchronous: the stream is ordered after the last copy back,
    so synchronise it before reading out_host."""
    for t, dt_ in ((q_host, torch.bfloat16), (w_host, torch.float32), (k_host, torch.bfloat16),
                   (out_host, torch.int32)):
        if t.is_cuda or not t.is_pinned() or not t.is_contiguous() or t.dtype != dt_:
            raise ValueError("q/w/k/out must be contiguous pinned CPU tensors (bf16, fp32, bf16, int32)")
    L, H, d = q_host.shape
    if w_host.shape != (L, H) or k_host.shape != (L, d) or out_host.shape != (L, topk):
        raise ValueError("expected q [L,H,d], w [L,H], k [L,d], out [L,topk]")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if dev.type != "cuda" or dev.index is None:
        raise ValueError("device must name one CUDA device, e.g. 'cuda:0'")
    with torch.cuda.device(dev):  # the C call works on the calling thread's current device
        nbytes = int(lib().pivot_refine_host_workspace_size(L, H, d, topk, c, g))
        if nbytes == 0:
            raise PivotError(2, "pivot_refine_host_workspace_size")
        W = _ws_for(ws, dev).get(nbytes)
        s = torch.cuda.current_stream(dev) if stream is None else stream
        _check(lib().pivot_refine_host(_ptr(q_host), _ptr(w_host), _ptr(k_host), L, H, d, topk, c, g, chunks,
                                       _ptr(out_host), _ptr(W), W.numel(), ctypes.c_void_p(s.cuda_stream)),
               "pivot_refine_host")
    return out_host


# the earlier name of refine_host
refine_streamed = refine_host


def guardrail_dense(op: int, L: int, c: int, g: int) -> bool:
    """The guardrail's choice (PIVOT paper, Efficiency Results, Figure 4): True when the
    dense indexer needs no more work than op (OP_REUSE or OP_REFINE) on a prefill of L."""
    r = lib().pivot_guardrail_dense(op, L, c, g)
    if r < 0:
        raise ValueError("invalid guardrail arguments")
    return bool(r)


def reuse_guarded(q, w, k, topk: int, g: int, *, scores: bool = False, ws: Optional[Workspace] = None,
                  stream=None):
    """PIVOT-Reuse behind the guardrail.  Returns (indices, scores|None, ran_dense)."""
    L, H, d, dt = _prefill_common(q, w, k)
    idx = torch.empty((L, topk), dtype=torch.int32, device=q.device)
    sc = torch.empty((L, topk), dtype=torch.float32, device=q.device) if scores else None
    dense = guardrail_dense(OP_REUSE, L, topk, g)
    nbytes = workspace_size(OP_DENSE if dense else OP_REUSE, L, H, d, topk, topk, g, dt)
    W = _ws_for(ws, q.device).get(nbytes)
    path = ctypes.c_int(-1)
    _check(lib().pivot_reuse_guarded(_ptr(q), _ptr(w), _ptr(k), L, H, d, dt, topk, g, _ptr(idx), _ptr(sc), _ptr(W),
                                     W.numel(), _stream(stream), ctypes.byref(path)), "pivot_reuse_guarded")
    return idx, sc, path.value == 1


def refine_guarded(q, w, k, topk: int, c: int, g: int, *, scores: bool = False, ws: Optional[Workspace] = None,
                   stream=None):
    """PIVOT-Refine behind the guardrail.  Returns (indices, scores|None, ran_dense)."""
    L, H, d, dt = _prefill_common(q, w, k)
    idx = torch.empty((L, topk), dtype=torch.int32, device=q.device)
    sc = torch.empty((L, topk), dtype=torch.float32, device=q.device) if scores else None
    dense = guardrail_dense(OP_REFINE, L, c, g)
    nbytes = workspace_size(OP_DENSE if dense else OP_REFINE, L, H, d, topk, c, g, dt)
    W = _ws_for(ws, q.device).get(nbytes)
    path = ctypes.c_int(-1)
    _check(lib().pivot_refine_guarded(_ptr(q), _ptr(w), _ptr(k), L, H, d, dt, topk, c, g, _ptr(idx), _ptr(sc), None,
                                      None, _ptr(W), W.numel(), _stream(stream), ctypes.byref(path)),
           "pivot_refine_guarded")
    return idx, sc, path.value == 1


def _varlen_common(q, w, kc, offsets, g):
    _need_cuda(q, w, kc)
    off_h = offsets.host if isinstance(offsets, DeviceOffsets) else torch.as_tensor(offsets, dtype=torch.int64).cpu().contiguous()
    B = off_h.numel() - 1
    if q.dim() != 3 or q.shape[0] != B * g or w.shape != (B * g, q.shape[1]) or kc.shape[1] != q.shape[2]:
        raise ValueError("expected q [B*g,H,d], w [B*g,H], k_cache [sum P, d]")
    return B, q.shape[1], q.shape[2], _dt(q), off_h


def _offsets_dev(off_h, device, stream):
    """The offsets on the device, copied on the call's stream from pinned memory without
    blocking the host (the launches that follow are queued behind the copy)."""
    s = torch.cuda.current_stream(device) if stream is None else stream
    with torch.cuda.stream(s):
        return off_h.pin_memory().to(device, non_blocking=True)


def reuse_varlen(q, w, k_cache, offsets, topk: int, g: int, *, scores: bool = False,
                 ws: Optional[Workspace] = None, stream=None):
    """Eq. (3)-(6) for a batch of MTP decode groups.  Returns (indices [B*g,topk], scores|None)."""
    B, H, d, dt, off_h = _varlen_common(q, w, k_cache, offsets, g)
    off_d = _offsets_pair(offsets, q.device, stream)[1] if isinstance(offsets, DeviceOffsets) else \
        _offsets_dev(off_h, q.device, stream)
    idx = torch.empty((B * g, topk), dtype=torch.int32, device=q.device)
    sc = torch.empty((B * g, topk), dtype=torch.float32, device=q.device) if scores else None
    nbytes = varlen_workspace_size(OP_REUSE, off_h, H, d, topk, topk, g, dt)
    W = _ws_for(ws, q.device).get(nbytes)
    _check(lib().pivot_reuse_varlen(_ptr(q), _ptr(w), _ptr(k_cache), _ptr(off_d), _ptr(off_h), B, H, d, dt, topk,
                                    g, _ptr(idx), _ptr(sc), _ptr(W), W.numel(), _stream(stream)),
           "pivot_reuse_varlen")
    return idx, sc


def refine_varlen(q, w, k_cache, offsets, topk: int, c: int, g: int, *, scores: bool = False, cand: bool = False,
                  ws: Optional[Workspace] = None, stream=None):
    """Eq. (3)-(5),(7)-(9) for a batch of MTP decode groups."""
    B, H, d, dt, off_h = _varlen_common(q, w, k_cache, offsets, g)
    off_d = _offsets_pair(offsets, q.device, stream)[1] if isinstance(offsets, DeviceOffsets) else \
        _offsets_dev(off_h, q.device, stream)
    idx = torch.empty((B * g, topk), dtype=torch.int32, device=q.device)
    sc = torch.empty((B * g, topk), dtype=torch.float32, device=q.device) if scores else None
    cd = torch.empty((B, c), dtype=torch.int32, device=q.device) if cand else None
    cs = torch.empty((B, c), dtype=torch.float32, device=q.device) if (cand and scores) else None
    nbytes = varlen_workspace_size(OP_REFINE, off_h, H, d, topk, c, g, dt)
    W = _ws_for(ws, q.device).get(nbytes)
    _check(lib().pivot_refine_varlen(_ptr(q), _ptr(w), _ptr(k_cache), _ptr(off_d), _ptr(off_h), B, H, d, dt, topk,
                                     c, g, _ptr(idx), _ptr(sc), _ptr(cd), _ptr(cs), _ptr(W), W.numel(),
                                     _stream(stream)), "pivot_refine_varlen")
    return idx, sc, cd, cs


# ---------------------------------------------------------------- one long decode prefix over ranks
# The C ABI's four steps (pivot_decode_shard_select, _merge, _shard_rescore, _rowselect); the
# exchanges between them (an all-gather of the shard entries, an element-wise sum of the member
# score keys) belong to the caller: multigpu.decode_split_step runs them over torch.distributed.


class DeviceOffsets:
    """int64 offsets (or per-sequence positions) kept on the host and on one device, so that repeated
    calls pass them without copying; any of the decode split calls accepts one where it takes offsets
    or positions."""

    def __init__(self, values, device):
        self.host = torch.as_tensor(values, dtype=torch.int64).cpu().contiguous()
        self.dev = self.host.to(device)


def _offsets_pair(offsets, device, stream):
    if isinstance(offsets, DeviceOffsets):
        if offsets.dev.device != torch.device(device):
            raise ValueError(f"offsets live on {offsets.dev.device}, the call runs on {device}")
        return offsets.host, offsets.dev
    h = torch.as_tensor(offsets, dtype=torch.int64).cpu().contiguous()
    return h, _offsets_dev(h, device, stream)


def _positions_dev(values, device, stream):
    """Per-sequence int64 values on the device (copied from pinned memory without blocking)."""
    if isinstance(values, DeviceOffsets) or (isinstance(values, torch.Tensor) and values.is_cuda):
        d = values.dev if isinstance(values, DeviceOffsets) else values
        if d.device != torch.device(device):
            raise ValueError(f"positions live on {d.device}, the call runs on {device}")
        return d
    return _offsets_pair(values, device, stream)[1]


def decode_shard_select(op: int, q, w, k_shard, shard_offsets, pos_base, topk: int, c: int, g: int, *,
                        ws: Optional[Workspace] = None, stream=None):
    """Step 1: this rank's key shard of every sequence -> its exact top-n (n = k+g-1 for
    OP_REUSE, c for OP_REFINE) as packed int64 entries [B, n] with prefix positions (0 pads)."""
    _need_cuda(q, w, k_shard)
    sh, sd = _offsets_pair(shard_offsets, q.device, stream)
    pb = _positions_dev(pos_base, q.device, stream)
    B = sh.numel() - 1
    H, d = q.shape[1], q.shape[2]
    n = topk + g - 1 if op == OP_REUSE else c
    ent = torch.empty((B, n), dtype=torch.int64, device=q.device)
    nbytes = int(lib().pivot_decode_shard_workspace_size(op, B, _ptr(sh), H, d, topk, c, g))
    if nbytes == 0:
        raise PivotError(1, "decode_shard_select", "unsupported shape or offsets")
    W = _ws_for(ws, q.device).get(nbytes)
    _check(lib().pivot_decode_shard_select(op, _ptr(q), _ptr(w), _ptr(k_shard), _ptr(sd), _ptr(sh), _ptr(pb), B, H,
                                           d, _dt(q), topk, c, g, _ptr(ent), _ptr(W), W.numel(), _stream(stream)),
           "pivot_decode_shard_select")
    return ent


def decode_merge(op: int, entries, plen_offsets, topk: int, c: int, g: int, *, shard_offsets=None, pos_base=None,
                 scores: bool = False, ws: Optional[Workspace] = None, stream=None):
    """Step 3: entries [R, B, n] of all ranks -> OP_REUSE: (indices [B*g, k], scores|None);
    OP_REFINE: (C [B, c], C scores|None, C in this rank's shard rows [B, c] | None)."""
    _need_cuda(entries)
    R, B, n = entries.shape
    ph, pd = _offsets_pair(plen_offsets, entries.device, stream)
    dev = entries.device
    local = shard_offsets is not None
    sd = _offsets_pair(shard_offsets, dev, stream)[1] if local else None
    pb = _positions_dev(pos_base, dev, stream) if local else None
    nbytes = int(lib().pivot_decode_merge_workspace_size(op, R, B, topk, c, g))
    W = _ws_for(ws, dev).get(nbytes)
    idx = sc = cand = csc = cl = None
    if op == OP_REUSE:
        idx = torch.empty((B * g, topk), dtype=torch.int32, device=dev)
        sc = torch.empty((B * g, topk), dtype=torch.float32, device=dev) if scores else None
    else:
        cand = torch.empty((B, c), dtype=torch.int32, device=dev)
        csc = torch.empty((B, c), dtype=torch.float32, device=dev) if scores else None
        cl = torch.empty((B, c), dtype=torch.int32, device=dev) if local else None
    _check(lib().pivot_decode_merge(op, _ptr(entries), R, _ptr(pd), _ptr(ph), B, topk, c, g, _ptr(idx), _ptr(sc),
                                    _ptr(cand), _ptr(csc), _ptr(pb), _ptr(sd), _ptr(cl), _ptr(W), W.numel(),
                                    _stream(stream)), "pivot_decode_merge")
    return (idx, sc) if op == OP_REUSE else (cand, csc, cl)


def decode_shard_rescore(q, w, k_shard, shard_offsets, pos_base, plen_offsets, cand_local, topk: int, c: int,
                         g: int, *, ws: Optional[Workspace] = None, stream=None):
    """Step 4: Eq. (8) member score keys [B*g, c] (int32 bits of the uint32 keys) of the candidates
    this rank's shard holds; 0 for the others."""
    _need_cuda(q, w, k_shard, cand_local)
    sh, sd = _offsets_pair(shard_offsets, q.device, stream)
    pd = _offsets_pair(plen_offsets, q.device, stream)[1]
    pb = _positions_dev(pos_base, q.device, stream)
    B = sh.numel() - 1
    H, d = q.shape[1], q.shape[2]
    keys = torch.empty((B * g, c), dtype=torch.int32, device=q.device)
    W = _ws_for(ws, q.device).get(256)
    _check(lib().pivot_decode_shard_rescore(_ptr(q), _ptr(w), _ptr(k_shard), _ptr(sd), _ptr(sh), _ptr(pb), _ptr(pd),
                                            B, H, d, _dt(q), topk, c, g, _ptr(cand_local), _ptr(keys), _ptr(W),
                                            W.numel(), _stream(stream)), "pivot_decode_shard_rescore")
    return keys


def decode_rowselect(keys, cand, plen_offsets, topk: int, c: int, g: int, *, scores: bool = False, stream=None):
    """Step 6: Eq. (9) on the rank-summed keys -> (indices [B*g, k], scores|None)."""
    _need_cuda(keys, cand)
    B = cand.shape[0]
    pd = _offsets_pair(plen_offsets, keys.device, stream)[1]
    idx = torch.empty((B * g, topk), dtype=torch.int32, device=keys.device)
    sc = torch.empty((B * g, topk), dtype=torch.float32, device=keys.device) if scores else None
    _check(lib().pivot_decode_rowselect(_ptr(keys), _ptr(cand), _ptr(pd), B, topk, c, g, _ptr(idx), _ptr(sc),
                                        _stream(stream)), "pivot_decode_rowselect")
    return idx, sc


def last_device_status(ws: Workspace, stream=None) -> int:
    """Synchronise the stream and return the device status code of the last call on ``ws``."""
    return int(lib().pivot_last_device_status(_ptr(ws.buf), _stream(stream)))


def set_device_timeout_ns(ns: int) -> None:
    lib().pivot_set_device_timeout_ns(int(ns))


def set_debug_flags(flags: int) -> None:
    lib().pivot_set_debug_flags(int(flags))


class KernelTimer:
    """Records CUDA events between the library's kernel launches (on the call's
    stream): times of the scan kernel, the refine kernel and the row select of a
    prefill call; of the proxies + scan, the selection + emit, and the re-scoring +
    row select of a decode call."""

    def __init__(self):
        self.ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        s = torch.cuda.current_stream()
        for e in self.ev:
            e.record(s)  # creates the underlying cudaEvent_t
        torch.cuda.synchronize()
        self._arr = (ctypes.c_void_p * 4)(*[e.cuda_event for e in self.ev])

    def __enter__(self):
        lib().pivot_set_profile_events(self._arr, 4)
        return self

    def __exit__(self, *exc):
        lib().pivot_set_profile_events(None, 0)

    def ms(self):
        """The three phase times (ms) of the last call, in the order above (after a sync)."""
        e = self.ev
        return e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3])


__all__ = [
    "lib", "LIB_PATH", "EXPORTS", "PivotError", "Workspace", "workspace_size", "varlen_workspace_size", "path",
    "indexer_dense", "reuse", "refine", "reuse_varlen", "refine_varlen", "last_device_status",
    "guardrail_dense", "reuse_guarded", "refine_guarded", "AGGREGATION",
    "indexer_dense_range", "reuse_range", "refine_range",
    "group_chunks", "refine_host", "refine_streamed",
    "decode_shard_select", "decode_merge", "decode_shard_rescore", "decode_rowselect", "DeviceOffsets",
    "set_device_timeout_ns", "set_debug_flags", "KernelTimer", "OP_DENSE", "OP_REUSE", "OP_REFINE", "BF16", "F32",
    "STATUS",
]
