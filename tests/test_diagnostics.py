"""The workload diagnostics (O1-O3) on hand-built rows with known values, and
(GPU) the same diagnostics from the library's dense rows against the oracle's."""
from __future__ import annotations

import numpy as np
import pytest

from top_token_selection_proxy_b200 import diagnostics as D


def _window_rows(L, k):
    # row t holds the k most recent keys t-k+1 .. t (full rows only), -1 padded otherwise
    idx = -np.ones((L, k), np.int32)
    for t in range(L):
        lo = max(0, t - k + 1)
        idx[t, : t + 1 - lo] = np.arange(lo, t + 1)
    return idx


def test_sliding_window_closed_forms():
    L, k = 200, 16
    idx = _window_rows(L, k)
    assert D.adjacent_overlap(idx, k) == pytest.approx((k - 1) / k)
    for g in (2, 4, 8):
        assert D.group_union(idx, k, g) == pytest.approx((k + g - 1) / k)
        assert D.group_intersection(idx, k, g) == pytest.approx((k - g + 1) / k)


def test_identical_rows_share_everything():
    L, k = 64, 8
    row = np.arange(k, dtype=np.int32) * 3
    idx = np.tile(row, (L, 1))
    assert D.adjacent_overlap(idx, k) == 1.0
    assert D.group_union(idx, k, 8) == 1.0
    assert D.group_intersection(idx, k, 4) == 1.0


def test_score_mass():
    s = np.array([[1.0, 4.0, -1.0, 2.0, 0.0, 3.0, -np.inf],
                  [5.0, 5.0, np.nan, 0.0, 0.0, 0.0, 0.0]])
    m = D.score_mass(s, (1, 2, 4))
    # row 0: positive mass 10 -> 0.4, 0.7, 1.0; row 1: mass 10 -> 0.5, 1.0, 1.0
    assert m[1] == pytest.approx((0.4 + 0.5) / 2)
    assert m[2] == pytest.approx((0.7 + 1.0) / 2)
    assert m[4] == pytest.approx(1.0)


@pytest.mark.gpu
def test_diagnostics_of_gpu_rows_match_oracle_rows(orc):
    import torch

    import top_token_selection_proxy_b200 as P
    from top_token_selection_proxy_b200 import inputs

    L, k = 1024, 64
    x = inputs.random_prefill(L, 64, 128, inputs.BF16, seed=91)
    dev = lambda a: (torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16) if a.dtype == np.uint16
                     else torch.from_numpy(np.ascontiguousarray(a)).cuda())
    gi, _ = P.indexer_dense(dev(x["q"]), dev(x["w"]), dev(x["k"]), k)
    _, gs = P.indexer_dense(dev(x["q"]), dev(x["w"]), dev(x["k"]), L, scores=True)
    torch.cuda.synchronize()
    oi, _ = orc.dense(x["q"], x["w"], x["k"], k)
    _, os_ = orc.dense(x["q"], x["w"], x["k"], L)
    a = D.summary(gi.cpu().numpy(), k, gs.cpu().numpy())
    b = D.summary(oi, k, os_)
    # the sets agree up to swaps of near-ties at the boundary: allow a couple of entries
    assert abs(a["O1_adjacent_overlap"] - b["O1_adjacent_overlap"]) <= 2 / k
    assert abs(a["O1_group4_common"] - b["O1_group4_common"]) <= 2 / k
    for g in (4, 8, 16):
        assert abs(a["O2_union_over_k"][g] - b["O2_union_over_k"][g]) <= 2 / k
    for m in a["O3_mass_at"]:
        assert a["O3_mass_at"][m] == pytest.approx(b["O3_mass_at"][m], rel=2e-3, abs=1e-4)
