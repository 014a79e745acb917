"""CPU-side checks of the C ABI: the library builds, loads and exports every
symbol include/pivot.h declares; host-side validation and sizing need no GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

import top_token_selection_proxy_b200 as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from top_token_selection_proxy_b200 import build

    build.build()
    return P.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "pivot.h")).read()
    return sorted(set(re.findall(r"PIVOT_API\s+[\w\s\*]+?\b(pivot_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(P.EXPORTS) == names


def test_version_and_status_strings(lib):
    assert lib.pivot_version() == 100
    for code, name in P.STATUS.items():
        assert lib.pivot_status_string(code).decode() == name


def test_workspace_sizes_positive_and_monotone(lib):
    a = P.workspace_size(P.OP_REFINE, 8192, 64, 128, 2048, 4096, 8)
    b = P.workspace_size(P.OP_REFINE, 131072, 64, 128, 2048, 4096, 8)
    assert 0 < a < b
    assert P.workspace_size(P.OP_DENSE, 512, 4, 32, 16, 16, 1, P.F32) > 0
    assert P.workspace_size(P.OP_REUSE, 100, 64, 128, 8, 8, 17) == 0  # g > 16 rejected
    assert P.workspace_size(P.OP_REFINE, 100, 64, 128, 8, 4, 4) == 0  # c < k rejected


def test_path_selection(lib):
    assert P.path(P.OP_REFINE, 131072, 64, 128, 2048, 4096, 8, P.BF16) == 1
    assert P.path(P.OP_DENSE, 131072, 64, 64, 2048, 2048, 1, P.BF16) == 1
    assert P.path(P.OP_REFINE, 512, 4, 32, 16, 32, 4, P.F32) == 0
    assert P.path(P.OP_REUSE, 512, 32, 128, 16, 16, 4, P.BF16) == 0
    assert P.path(P.OP_REUSE, 0, 64, 128, 16, 16, 4, P.BF16) == -1


def test_invalid_arguments_rejected_before_launch(lib):
    # null pointers, zero sizes, k > c, bad g: rejected on the host (no device needed)
    nul = None
    buf = ctypes.create_string_buffer(1024)
    ptr = ctypes.cast(buf, ctypes.c_void_p)
    assert lib.pivot_indexer_dense(nul, nul, nul, 16, 4, 32, 0, 4, nul, nul, nul, 0, nul) == 1
    assert lib.pivot_reuse(ptr, ptr, ptr, 0, 4, 32, 0, 4, 2, ptr, nul, ptr, 1024, nul) == 1
    assert lib.pivot_refine(ptr, ptr, ptr, 64, 4, 32, 0, 8, 4, 2, ptr, nul, nul, nul, ptr, 1024, nul) == 1
    assert lib.pivot_reuse(ptr, ptr, ptr, 64, 4, 32, 0, 4, 32, ptr, nul, ptr, 1024, nul) == 2
    assert lib.pivot_indexer_dense(ptr, ptr, ptr, 64, 4, 30, 0, 4, ptr, nul, ptr, 1024, nul) == 1  # d % 8
    off = np.array([0, 3, 10], np.int64)  # P_0 = 3 < g = 4
    assert lib.pivot_varlen_workspace_size(1, 2, off.ctypes.data_as(ctypes.c_void_p), 64, 128, 8, 8, 4, 0) == 0


def test_decode_split_entry_points_validate_on_the_host(lib):
    """The split decode's calls (one long prefix over GPUs) size their workspaces and reject bad
    arguments before any device work."""
    vp = ctypes.c_void_p
    shard = np.array([0, 1, 5, 9], np.int64)  # a shard may hold a single key of a sequence
    empty = np.array([0, 0, 4, 9], np.int64)  # ... but not none
    sz = lambda op, off, H=64, d=128: lib.pivot_decode_shard_workspace_size(op, 3, off.ctypes.data_as(vp), H, d,
                                                                            8, 16, 4)
    assert sz(P.OP_REUSE, shard) > 0 and sz(P.OP_REFINE, shard) > 0
    assert sz(P.OP_REFINE, empty) == 0
    assert sz(P.OP_DENSE, shard) == 0                      # Reuse or Refine only
    assert sz(P.OP_REFINE, shard, H=32) == 0              # tensor-core shape only
    m = [lib.pivot_decode_merge_workspace_size(P.OP_REFINE, R, 3, 8, 16, 4) for R in (1, 2, 4)]
    assert 0 < m[0] < m[1] < m[2]
    assert lib.pivot_decode_merge_workspace_size(P.OP_REFINE, 0, 3, 8, 16, 4) == 0
    assert lib.pivot_decode_merge_workspace_size(P.OP_REFINE, 2, 3, 8, 4, 4) == 0  # c < k
    buf = ctypes.create_string_buffer(1 << 16)
    ptr = ctypes.c_void_p((ctypes.addressof(buf) + 255) // 256 * 256)
    plen = np.array([0, 9, 20, 40], np.int64)
    short = np.array([0, 3, 20, 40], np.int64)  # P_0 = 3 < g = 4
    pl, sh = plen.ctypes.data_as(vp), short.ctypes.data_as(vp)
    # merge: null entries, a prefix shorter than g, Reuse without its output, workspace too small
    assert lib.pivot_decode_merge(P.OP_REUSE, None, 2, ptr, pl, 3, 8, 8, 4, ptr, None, None, None, None, None,
                                  None, ptr, 1 << 15, None) == 1
    assert lib.pivot_decode_merge(P.OP_REUSE, ptr, 2, ptr, sh, 3, 8, 8, 4, ptr, None, None, None, None, None,
                                  None, ptr, 1 << 15, None) == 1
    assert lib.pivot_decode_merge(P.OP_REUSE, ptr, 2, ptr, pl, 3, 8, 8, 4, None, None, None, None, None, None,
                                  None, ptr, 1 << 15, None) == 1
    assert lib.pivot_decode_merge(P.OP_REFINE, ptr, 2, ptr, pl, 3, 8, 16, 4, None, None, ptr, None, None, None,
                                  ptr, ptr, 1 << 15, None) == 1  # a local C needs this rank's shard
    assert lib.pivot_decode_merge(P.OP_REFINE, ptr, 2, ptr, pl, 3, 8, 16, 4, None, None, ptr, None, None, None,
                                  None, ptr, 256, None) == 3
    sp = shard.ctypes.data_as(vp)
    # shard select: dense is not a decode op; fp32 has no tensor-core path; null entries
    assert lib.pivot_decode_shard_select(P.OP_DENSE, ptr, ptr, ptr, ptr, sp, ptr, 3, 64, 128, P.BF16, 8, 16, 4,
                                         ptr, ptr, 1 << 15, None) == 1
    assert lib.pivot_decode_shard_select(P.OP_REFINE, ptr, ptr, ptr, ptr, sp, ptr, 3, 64, 128, P.F32, 8, 16, 4,
                                         ptr, ptr, 1 << 15, None) == 2
    assert lib.pivot_decode_shard_select(P.OP_REFINE, ptr, ptr, ptr, ptr, sp, ptr, 3, 64, 128, P.BF16, 8, 16, 4,
                                         None, ptr, 1 << 15, None) == 1
    assert lib.pivot_decode_shard_rescore(ptr, ptr, ptr, ptr, sp, ptr, ptr, 3, 64, 128, P.BF16, 8, 16, 4, None,
                                          ptr, ptr, 1 << 15, None) == 1
    assert lib.pivot_decode_rowselect(ptr, ptr, ptr, 3, 8, 4, 4, ptr, None, None) == 1  # c < k


def test_workspace_too_small_rejected(lib):
    buf = ctypes.create_string_buffer(4096)
    ptr = ctypes.c_void_p((ctypes.addressof(buf) + 15) // 16 * 16)
    st = lib.pivot_reuse(ptr, ptr, ptr, 1024, 64, 128, 0, 16, 4, ptr, None, ptr, 256, None)
    assert st == 3


# ---------------------------------------------------------------- guardrail decision (host logic)


def test_guardrail_decision():
    g_dense = P.lib().pivot_guardrail_dense
    # Reuse scans sum_i P_i keys: less than dense's L(L+1)/2 for any g >= 2; equal at g = 1
    for L in (1, 2, 100, 8192, 131072):
        assert g_dense(P.OP_REUSE, L, 16, 1) == 1
    for L in (2, 100, 8192, 131072):
        for g in (2, 4, 8, 16):
            assert g_dense(P.OP_REUSE, L, 16, g) == 0
    # Refine at L = 8192, g = 8, c = 4096, worked by hand: dense 8192*8193/2 = 33,558,528 key-row
    # products; scan 8*(1+...+1024) = 4,198,400; re-scoring 8*[8*(1+...+512) + 512*4096] =
    # 25,182,208; Refine total 29,380,608 < dense, so Refine is kept
    assert g_dense(P.OP_REFINE, 8192, 4096, 8) == 0
    # c >= L: every candidate set is the whole prefix, Refine only adds the scan to dense's work
    assert g_dense(P.OP_REFINE, 4096, 4096, 8) == 1
    assert g_dense(P.OP_REFINE, 3000, 4096, 8) == 1
    # long context: Refine's work grows like L*c, dense like L^2
    assert g_dense(P.OP_REFINE, 131072, 4096, 8) == 0
    # the choice flips once, from dense to Refine, as L grows (g = 8, c = 4096)
    picks = [g_dense(P.OP_REFINE, L, 4096, 8) for L in range(1000, 20000, 250)]
    flips = sum(1 for a, b in zip(picks, picks[1:]) if a != b)
    assert picks[0] == 1 and picks[-1] == 0 and flips == 1
    # invalid arguments
    assert g_dense(P.OP_DENSE, 100, 16, 8) == -1
    assert g_dense(P.OP_REFINE, 0, 16, 8) == -1
    assert g_dense(P.OP_REFINE, 100, 0, 8) == -1
    assert g_dense(P.OP_REUSE, 100, 16, 0) == -1


def test_group_chunks_cover_the_rows_in_whole_groups():
    from top_token_selection_proxy_b200 import group_chunks

    for L, g, n in ((6001, 8, 8), (6001, 8, 3), (64, 8, 8), (5, 8, 4), (131072, 8, 8), (100, 1, 7)):
        ch = group_chunks(L, g, n)
        assert 1 <= len(ch) <= n
        assert ch[0][0] == 0 and ch[-1][1] == L
        for (a0, a1), (b0, _) in zip(ch, ch[1:]):
            assert a1 == b0
        for t0, t1 in ch:
            assert t0 < t1 and t0 % g == 0 and (t1 % g == 0 or t1 == L)
    with pytest.raises(ValueError):
        group_chunks(0, 8, 2)


def test_decode_workspace_grows_with_the_cached_keys(lib):
    # tensor-core decode path: a 32-bit score key and a tie slot per cached key
    off_a = np.array([0, 20000, 50000], dtype=np.int64)
    off_b = np.array([0, 20000, 50000 + 100000], dtype=np.int64)
    for op, c in ((P.OP_REUSE, 2048), (P.OP_REFINE, 4096)):
        a = P.varlen_workspace_size(op, off_a, 64, 128, 2048, c, 4)
        b = P.varlen_workspace_size(op, off_b, 64, 128, 2048, c, 4)
        assert 0 < a and b - a >= 12 * 100000 - 8 * 256  # buffers start on 256-byte boundaries
    assert P.varlen_workspace_size(P.OP_REUSE, np.array([0, 3], dtype=np.int64), 64, 128, 8, 8, 4) == 0  # P_b < g
    assert P.varlen_workspace_size(P.OP_REUSE, np.array([5, 20], dtype=np.int64), 64, 128, 8, 8, 4) == 0  # off[0] != 0


def test_host_entry_point_checks_arguments_before_any_cuda_call(lib):
    """pivot_refine_host: argument and workspace checks happen on the host, before a stream,
    event or copy is touched (so they also hold on a machine without a GPU)."""
    buf = ctypes.create_string_buffer(4096 + 256)
    ws = ctypes.c_void_p((ctypes.addressof(buf) + 255) // 256 * 256)
    h = ctypes.cast(ctypes.create_string_buffer(64), ctypes.c_void_p)
    L, H, d, k, c, g = 1024, 64, 128, 16, 32, 8
    need = lib.pivot_refine_host_workspace_size(L, H, d, k, c, g)
    # the device copies of q, w, k and the output rows, then the refine workspace
    assert need >= L * H * d * 2 + L * H * 4 + L * d * 2 + L * k * 4 + \
        lib.pivot_workspace_size(2, L, H, d, k, c, g, 0)
    assert lib.pivot_refine_host_workspace_size(L, H, d, k, 8, g) == 0  # c < k
    args = (h, h, h, L, H, d, k, c, g)
    assert lib.pivot_refine_host(None, h, h, L, H, d, k, c, g, 8, h, ws, 4096, None) == 1
    assert lib.pivot_refine_host(*args, 0, h, ws, 4096, None) == 1      # chunks outside 1..64
    assert lib.pivot_refine_host(*args, 65, h, ws, 4096, None) == 1
    mis = ctypes.c_void_p(ws.value + 16)
    assert lib.pivot_refine_host(*args, 8, h, mis, 4096, None) == 1     # ws not 256-byte aligned
    assert lib.pivot_refine_host(*args, 8, h, ws, 4096, None) == 3      # workspace too small
