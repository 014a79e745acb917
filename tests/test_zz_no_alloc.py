"""pivot_reuse_noalloc: PIVOT-Reuse for callers that cannot allocate device
memory (their device memory belongs to a pool or planner they do not
control), with its scratch in a static device array instead of a caller
workspace.  Checked through the C ABI against pivot_reuse, the entry point
with a workspace, on two calls in a row (the array keeps the previous call's
contents, so the second call checks that what must start cleared is cleared),
and against the CPU oracle on every group.  This file is collected last on
purpose."""
import ctypes

import numpy as np
import pytest
import torch

import top_token_selection_proxy_b200 as P
from parity import check_row, summarize
from top_token_selection_proxy_b200 import inputs

pytestmark = pytest.mark.gpu

TOL_ABS, TOL_REL = 1e-4, 2e-3


def _dev(x):
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _noalloc(lib, q, w, k, topk, g):
    L, H, d = q.shape
    idx = torch.empty((L, topk), dtype=torch.int32, device=q.device)
    sc = torch.empty((L, topk), dtype=torch.float32, device=q.device)
    st = lib.pivot_reuse_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                                 ctypes.c_void_p(k.data_ptr()), ctypes.c_int64(L), H, d, P.BF16, topk, g,
                                 ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(sc.data_ptr()),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, idx, sc


def _same_rows(a_idx, a_sc, b_idx, b_sc):
    """Same index set per row, scores of common indices within the tests' tolerance;
    where sets differ, only near-ties at the row's boundary may swap."""
    for t in range(a_idx.shape[0]):
        va, vb = a_idx[t] >= 0, b_idx[t] >= 0
        assert va.sum() == vb.sum(), t
        da = dict(zip(a_idx[t][va].tolist(), a_sc[t][va].tolist()))
        db = dict(zip(b_idx[t][vb].tolist(), b_sc[t][vb].tolist()))
        for s in set(da) & set(db):
            assert abs(da[s] - db[s]) <= TOL_ABS + TOL_REL * abs(db[s]), (t, s)
        if set(da) != set(db):
            lo = min(db.values())
            for s in set(da) ^ set(db):
                v = da.get(s, db.get(s))
                assert abs(v - lo) <= TOL_ABS + TOL_REL * abs(lo), (t, s)


def _oracle_fails(orc, x, idx, sc, topk, g):
    """Every member row against the oracle's Eq. (4)-(6): proxy scores over s <= t."""
    L = x["q"].shape[0]
    G = (L + g - 1) // g
    mem = [list(range(i * g, min(i * g + g, L))) for i in range(G)]
    qv, wv = orc.proxies(x["q"], x["w"], mem)
    F = orc.scores_batch(qv, wv, x["k"], plen=np.array([m[-1] + 1 for m in mem]))
    fails = []
    for i, m in enumerate(mem):
        for t in m:
            fails += check_row(idx[t], sc[t], np.arange(t + 1), F[i, :t + 1], min(topk, t + 1), orc,
                               f"noalloc reuse t={t}")
    return fails


@pytest.mark.parametrize("L,topk,g", [(3001, 120, 8), (4000, 249, 8)])
def test_reuse_noalloc_matches_workspace_entry_point_twice(orc, L, topk, g):
    """k + g - 1 = 127 (several tiles and cut-backs) and = 256, the largest selection the
    static scratch takes (its sub-buffers run their cut-backs closest to full)."""
    from top_token_selection_proxy_b200 import build

    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = P.lib()
    H, d = 64, 128
    x = inputs.random_prefill(L, H, d, inputs.BF16, seed=4242 + topk)
    q, w, k = _dev(x["q"]), _dev(x["w"]), _dev(x["k"])
    ref_idx, ref_sc = P.reuse(q, w, k, topk, g, scores=True)
    torch.cuda.synchronize()
    ref_idx, ref_sc = ref_idx.cpu().numpy(), ref_sc.cpu().numpy()
    for call in range(2):
        st, idx, sc = _noalloc(lib, q, w, k, topk, g)
        assert st == 0, P.STATUS.get(st, st)
        torch.cuda.synchronize()
        idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
        _same_rows(idx, sc, ref_idx, ref_sc)
        fails = _oracle_fails(orc, x, idx, sc, topk, g)
        assert not fails, summarize(fails)


def test_reuse_noalloc_rejects_sizes_beyond_its_scratch():
    lib = P.lib()
    x = inputs.random_prefill(64, 64, 128, inputs.BF16, seed=1)
    q, w, k = _dev(x["q"]), _dev(x["w"]), _dev(x["k"])
    st, _, _ = _noalloc(lib, q, w, k, 250, 8)  # k + g - 1 = 257 > 256
    assert st == 2  # PIVOT_ERR_UNSUPPORTED_SHAPE
