"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Small cases are checked on every row/group; the long workloads on a seeded
sample of groups (always including the first and last group and the groups
whose prefix straddles c and k+g-1), at the sizes and launch configuration
the bench uses.  Refine is checked in two levels: the GPU candidate set C_i
against the oracle's proxy scores, then the member rows against the oracle
re-scoring over the GPU's own C_i.
"""
import numpy as np
import pytest
import torch

import top_token_selection_proxy_b200 as P
from parity import check_row, summarize
from top_token_selection_proxy_b200 import inputs
from top_token_selection_proxy_b200 import multigpu as MG

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from top_token_selection_proxy_b200 import build

    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    P.set_device_timeout_ns(2_000_000_000)
    P.set_debug_flags(0)


def dev(x):
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def host(t):
    return None if t is None else t.cpu().numpy()


def members(L, g, i):
    return list(range(i * g, min(i * g + g, L)))


def pooled(m, agg):
    """The member rows the proxy pools: all (mean), the first or the last one."""
    return {"mean": m, "first": m[:1], "last": m[-1:]}[agg]


# ---------------------------------------------------------------- checkers


def check_dense(orc, x, idx, sc, rows, topk, pos=None, block=512):
    """Dense rows `rows` of idx/sc (positions `pos`, default the row numbers) against
    the oracle's scores of those queries over their prefixes; oracle scores are
    computed `block` rows at a time."""
    q, w, k = x["q"], x["w"], x["k"]
    rows = list(rows)
    pos = rows if pos is None else list(pos)
    fails = []
    for b0 in range(0, len(rows), block):
        rb, pb = rows[b0:b0 + block], pos[b0:b0 + block]
        qv, wv = orc.query_rows(q, w, rb)
        F = orc.scores_batch(qv, wv, k, plen=np.array(pb) + 1)
        for i, (r, t) in enumerate(zip(rb, pb)):
            fails += check_row(idx[r], None if sc is None else sc[r], np.arange(t + 1), F[i, :t + 1],
                               min(topk, t + 1), orc, f"dense row {r}")
    return fails


def check_reuse(orc, x, idx, sc, groups, topk, g, agg="mean", block=256):
    q, w, k = x["q"], x["w"], x["k"]
    L = q.shape[0]
    groups = list(groups)
    fails = []
    for b0 in range(0, len(groups), block):
        mem = [members(L, g, i) for i in groups[b0:b0 + block]]
        qv, wv = orc.proxies(q, w, [pooled(m, agg) for m in mem])
        F = orc.scores_batch(qv, wv, k, plen=np.array([m[-1] + 1 for m in mem]))
        for gi, m in enumerate(mem):
            for t in m:
                fails += check_row(idx[t], None if sc is None else sc[t], np.arange(t + 1), F[gi, :t + 1],
                                   min(topk, t + 1), orc, f"reuse g={g} t={t}")
    return fails


def check_refine(orc, x, idx, sc, cand, csc, groups, topk, c, g, agg="mean", block=64):
    """Two levels: each group's C_i against the oracle's proxy scores, then every member
    row against the oracle's re-scoring (Eq. 8) and top-k (Eq. 9) over that C_i."""
    q, w, k = x["q"], x["w"], x["k"]
    L = q.shape[0]
    groups = list(groups)
    fails = []
    for b0 in range(0, len(groups), block):
        gb = groups[b0:b0 + block]
        mem = [members(L, g, i) for i in gb]
        qv, wv = orc.proxies(q, w, [pooled(m, agg) for m in mem])
        F = orc.scores_batch(qv, wv, k, plen=np.array([m[-1] + 1 for m in mem]))
        for gi, (i, m) in enumerate(zip(gb, mem)):
            e = m[-1]
            fails += check_row(cand[i], None if csc is None else csc[i], np.arange(e + 1), F[gi, :e + 1],
                               min(c, e + 1), orc, f"C_{i}")
        fails += check_refine_rows(orc, x, idx, sc, cand, gb, topk, g)
    return fails


def check_refine_rows(orc, x, idx, sc, cand, groups, topk, g):
    """Member rows of the given groups against the oracle's Eq. (8)-(9) over the
    candidate sets `cand` (the GPU's own C_i)."""
    q, w, k = x["q"], x["w"], x["k"]
    L = q.shape[0]
    mem = [members(L, g, i) for i in groups]
    rows = [t for m in mem for t in m]
    grp_of = [i for i, m in zip(groups, mem) for _ in m]
    qv, wv = orc.query_rows(q, w, rows)
    C = np.stack([cand[i] for i in grp_of]).astype(np.int64)
    M = orc.scores_batch(qv, wv, k, key_rows=C)
    fails = []
    for r, (t, i) in enumerate(zip(rows, grp_of)):
        ok = (C[r] >= 0) & (C[r] <= t)
        E, f = C[r][ok], M[r][ok]
        fails += check_row(idx[t], None if sc is None else sc[t], E, f, min(topk, E.size), orc,
                           f"refine g={g} t={t}")
    return fails


def run_all(x, topk, c, g, scores=True):
    q, w, k = dev(x["q"]), dev(x["w"]), dev(x["k"])
    d_idx, d_sc = P.indexer_dense(q, w, k, topk, scores=scores)
    u_idx, u_sc = P.reuse(q, w, k, topk, g, scores=scores)
    r_idx, r_sc, r_c, r_cs = P.refine(q, w, k, topk, c, g, scores=scores, cand=True)
    torch.cuda.synchronize()
    return {n: host(v) for n, v in dict(d_idx=d_idx, d_sc=d_sc, u_idx=u_idx, u_sc=u_sc, r_idx=r_idx,
                                        r_sc=r_sc, r_c=r_c, r_cs=r_cs).items()}


def full_check(orc, x, res, topk, c, g, groups=None, dense_rows=None):
    L = x["q"].shape[0]
    G = (L + g - 1) // g
    groups = list(range(G)) if groups is None else list(groups)
    dense_rows = list(range(L)) if dense_rows is None else list(dense_rows)
    fails = check_dense(orc, x, res["d_idx"], res["d_sc"], dense_rows, topk)
    fails += check_reuse(orc, x, res["u_idx"], res["u_sc"], groups, topk, g)
    fails += check_refine(orc, x, res["r_idx"], res["r_sc"], res["r_c"], res["r_cs"], groups, topk, c, g)
    return fails


# ---------------------------------------------------------------- small workloads, every row


@pytest.mark.parametrize("c_sel,topk", [(100, 37), (130, 64)])
def test_refine_unaligned_candidates_and_odd_c(orc, c_sel, topk):
    """C written to a 4-byte-offset buffer, c not a multiple of 4: the member
    top-k takes its scalar-load path; every group is checked."""
    x = inputs.random_prefill(1337, 64, 128, inputs.BF16, seed=777)
    q, w, k = dev(x["q"]), dev(x["w"]), dev(x["k"])
    g = 8
    G = (1337 + g - 1) // g
    backing = torch.empty(G * c_sel + 1, dtype=torch.int32, device=q.device)
    cand_buf = backing[1:].view(G, c_sel)
    assert cand_buf.data_ptr() % 16 != 0
    r_idx, r_sc, r_c, r_cs = P.refine(q, w, k, topk, c_sel, g, scores=True, cand=cand_buf)
    torch.cuda.synchronize()
    assert r_c.data_ptr() == cand_buf.data_ptr()
    fails = check_refine(orc, x, host(r_idx), host(r_sc), host(r_c), host(r_cs), range(G), topk, c_sel, g)
    assert not fails, summarize(fails)


def test_tiny_config_every_group(orc):
    s = inputs.TINY
    x = inputs.make_prefill(s)
    assert P.path(P.OP_REFINE, s.L, s.H, s.d, s.k, s.c, s.g, P.F32) == 0
    res = run_all(x, s.k, s.c, s.g)
    fails = full_check(orc, x, res, s.k, s.c, s.g)
    assert not fails, summarize(fails)


@pytest.mark.parametrize("g", [4, 8, 16])
def test_tensor_core_path_every_group(orc, g):
    # ragged: L is not a multiple of 128 keys, of g, nor of 4 groups per work item;
    # k and c small enough that the streaming selection cuts back several times
    L, H, d, topk, c = 1337, 64, 128, 64, 128
    x = inputs.random_prefill(L, H, d, inputs.BF16, seed=100 + g, rho=0.95, heavy=0.01)
    assert P.path(P.OP_REFINE, L, H, d, topk, c, g, P.BF16) == 1
    res = run_all(x, topk, c, g)
    fails = full_check(orc, x, res, topk, c, g)
    assert not fails, summarize(fails)


def test_tensor_core_d64(orc):
    L, H, d, topk, c, g = 700, 64, 64, 32, 64, 8
    x = inputs.random_prefill(L, H, d, inputs.BF16, seed=7, rho=0.9, heavy=0.02)
    assert P.path(P.OP_REFINE, L, H, d, topk, c, g, P.BF16) == 1
    res = run_all(x, topk, c, g)
    fails = full_check(orc, x, res, topk, c, g)
    assert not fails, summarize(fails)


def test_cuda_core_path_bf16_odd_heads(orc):
    L, H, d, topk, c, g = 300, 8, 40, 10, 20, 3
    x = inputs.random_prefill(L, H, d, inputs.BF16, seed=9)
    assert P.path(P.OP_REFINE, L, H, d, topk, c, g, P.BF16) == 0
    res = run_all(x, topk, c, g)
    fails = full_check(orc, x, res, topk, c, g)
    assert not fails, summarize(fails)


# ---------------------------------------------------------------- edge cases


@pytest.mark.parametrize("L", [1, 2, 127, 128, 129])
def test_short_sequences(orc, L):
    x = inputs.random_prefill(L, 64, 128, inputs.BF16, seed=L)
    topk, c, g = 8, 16, 4
    res = run_all(x, topk, c, g)
    fails = full_check(orc, x, res, topk, c, g)
    assert not fails, summarize(fails)


def test_k_larger_than_prefix_and_c_ge_L(orc):
    # c >= L: C_i is the whole prefix, so Refine rows equal dense rows (Eq. 7-9 reduce to Eq. 1)
    L, topk, c, g = 300, 256, 512, 8
    x = inputs.random_prefill(L, 64, 128, inputs.BF16, seed=11)
    res = run_all(x, topk, c, g)
    fails = full_check(orc, x, res, topk, c, g)
    assert not fails, summarize(fails)
    for t in range(L):
        a = set(res["r_idx"][t][res["r_idx"][t] >= 0].tolist())
        b = set(res["d_idx"][t][res["d_idx"][t] >= 0].tolist())
        assert a == b, t


def test_ties_zero_queries_lowest_index(orc):
    """All-zero queries: every score is +-0 -> each row is exactly 0..min(k,t+1)-1."""
    L, H, d, topk, c, g = 400, 64, 128, 32, 64, 8
    x = inputs.random_prefill(L, H, d, inputs.BF16, seed=12)
    x["q"][:] = 0
    x["w"][:] = -1.0
    res = run_all(x, topk, c, g)
    for name in ("d_idx", "u_idx", "r_idx"):
        for t in range(L):
            n = min(topk, t + 1)
            assert sorted(res[name][t][:n].tolist()) == list(range(n)), (name, t)
            assert (res[name][t][n:] == -1).all()


def test_duplicate_keys_lower_index(orc):
    L, H, d, topk, c, g = 512, 64, 128, 16, 32, 4
    x = inputs.random_prefill(L, H, d, inputs.BF16, seed=13)
    x["k"][100:200] = x["k"][50]  # many exact ties in every score
    res = run_all(x, topk, c, g)
    fails = full_check(orc, x, res, topk, c, g)
    assert not fails, summarize(fails)


def test_reuse_g1_equals_dense_on_gpu():
    L, topk = 1000, 32
    x = inputs.random_prefill(L, 64, 128, inputs.BF16, seed=14)
    q, w, k = dev(x["q"]), dev(x["w"]), dev(x["k"])
    a, _ = P.indexer_dense(q, w, k, topk)
    b, _ = P.reuse(q, w, k, topk, 1)
    assert torch.equal(a.sort(dim=1).values, b.sort(dim=1).values)


# ---------------------------------------------------------------- the workloads at full size


def test_prefill_8k_every_group(orc):
    """The 8K prefill workload: every one of its 1024 groups (Refine at both levels,
    Reuse on every member row) and every dense row, against the oracle."""
    s = inputs.PREFILL_8K
    x = inputs.make_prefill(s)
    res = run_all(x, s.k, s.c, s.g)
    fails = full_check(orc, x, res, s.k, s.c, s.g)
    assert not fails, summarize(fails)


@pytest.mark.parametrize("rho", inputs.SWEEP_RHO)
@pytest.mark.parametrize("g", inputs.SWEEP_G)
def test_sweep_32k_sampled(orc, g, rho):
    """Each point of the L = 32768 group-size sweep: Reuse and Refine on 256 seeded groups."""
    s = inputs.sweep_32k(g, rho)
    x = inputs.make_prefill(s)
    q, w, k = dev(x["q"]), dev(x["w"]), dev(x["k"])
    u_idx, u_sc = P.reuse(q, w, k, s.k, g, scores=True)
    r_idx, r_sc, r_c, r_cs = P.refine(q, w, k, s.k, s.c, g, scores=True, cand=True)
    torch.cuda.synchronize()
    G = (s.L + g - 1) // g
    groups = inputs.sample_groups(G, g, s.k, s.c, 256, s.seed + 1000 + g)
    fails = check_reuse(orc, x, host(u_idx), host(u_sc), groups, s.k, g)
    fails += check_refine(orc, x, host(r_idx), host(r_sc), host(r_c), host(r_cs), groups, s.k, s.c, g)
    assert not fails, summarize(fails)


@pytest.fixture(scope="module")
def long_inputs():
    return inputs.make_prefill(inputs.LONG_128K)


def test_long_128k_refine_reuse_dense_sampled(orc, long_inputs):
    """The L = 131072 headline workload on 256 seeded groups: Refine at both levels,
    Reuse and the dense indexer on every member row of those groups."""
    s = inputs.LONG_128K
    x = long_inputs
    q, w, k = dev(x["q"]), dev(x["w"]), dev(x["k"])
    r_idx, r_sc, r_c, r_cs = P.refine(q, w, k, s.k, s.c, s.g, scores=True, cand=True)
    u_idx, u_sc = P.reuse(q, w, k, s.k, s.g, scores=True)
    d_idx, d_sc = P.indexer_dense(q, w, k, s.k, scores=True)
    torch.cuda.synchronize()
    G = (s.L + s.g - 1) // s.g
    groups = inputs.sample_groups(G, s.g, s.k, s.c, 256, s.seed + 1000)
    fails = check_refine(orc, x, host(r_idx), host(r_sc), host(r_c), host(r_cs), groups, s.k, s.c, s.g)
    fails += check_reuse(orc, x, host(u_idx), host(u_sc), groups, s.k, s.g)
    rows = [t for i in groups for t in members(s.L, s.g, int(i))]
    fails += check_dense(orc, x, host(d_idx), host(d_sc), rows, s.k)
    assert not fails, summarize(fails)


def _decode_batch_fails(orc, s, x, run=None):
    """Every sequence's C row and Reuse rows, and every Refine row, against the oracle.  run(q, w,
    k_cache, offsets) -> (Reuse indices, scores, Refine indices, scores, C, C scores) on the device
    (default: the batch calls)."""
    off = x["offsets"]
    q, w, kc = dev(x["q"]), dev(x["w"]), dev(x["k"])
    if run is None:
        u_idx, u_sc = P.reuse_varlen(q, w, kc, off, s.k, s.g, scores=True)
        r_idx, r_sc, r_c, r_cs = P.refine_varlen(q, w, kc, off, s.k, s.c, s.g, scores=True, cand=True)
    else:
        u_idx, u_sc, r_idx, r_sc, r_c, r_cs = run(q, w, kc, off)
    torch.cuda.synchronize()
    u_idx, u_sc, r_idx, r_sc, r_c, r_cs = map(host, (u_idx, u_sc, r_idx, r_sc, r_c, r_cs))
    B, g = s.B, s.g
    mem = [list(range(b * g, b * g + g)) for b in range(B)]
    qv, wv = orc.proxies(x["q"], x["w"], mem)
    Pb = np.diff(off)
    F = orc.scores_batch(qv, wv, x["k"], plen=Pb, key_base=off[:-1])
    fails = []
    for b in range(B):
        fails += check_row(r_c[b], r_cs[b], np.arange(Pb[b]), F[b, :Pb[b]], min(s.c, Pb[b]), orc, f"C_{b}")
        for r in range(g):
            t = Pb[b] - g + r
            fails += check_row(u_idx[b * g + r], u_sc[b * g + r], np.arange(t + 1), F[b, :t + 1],
                               min(s.k, t + 1), orc, f"decode reuse b={b} r={r}")
    rows = list(range(B * g))
    qv, wv = orc.query_rows(x["q"], x["w"], rows)
    C = np.repeat(r_c.astype(np.int64), g, axis=0)
    M = orc.scores_batch(qv, wv, x["k"], key_rows=C, key_base=np.repeat(off[:-1], g))
    for row in rows:
        b, r = divmod(row, g)
        t = Pb[b] - g + r
        ok = (C[row] >= 0) & (C[row] <= t)
        fails += check_row(r_idx[row], r_sc[row], C[row][ok], M[row][ok], min(s.k, int(ok.sum())), orc,
                           f"decode refine b={b} r={r}")
    return fails, (u_idx, u_sc, r_idx, r_sc, r_c, r_cs)


def test_decode_batch_every_sequence(orc):
    s = inputs.DECODE
    fails, _ = _decode_batch_fails(orc, s, inputs.make_decode(s))
    assert not fails, summarize(fails)


def test_decode_many_short_sequences(orc):
    # about 5 scan sets per CTA over several sequences: the proxy ring turns over and the
    # per-CTA digit counts are flushed at every sequence change; many P_b <= c (keep all)
    s = inputs.DecodeSpec("short", B=600, p_lo=4, p_hi=700, H=64, d=128, k=64, c=128, g=4, seed=23)
    fails, _ = _decode_batch_fails(orc, s, inputs.make_decode(s))
    assert not fails, summarize(fails)


def test_decode_duplicate_keys_lowest_index_wins(orc):
    # every cached key is one of 40 vectors, so whole blocks of keys tie exactly and the
    # selection's final bin holds hundreds of equal scores: the lower index must win
    s = inputs.DecodeSpec("dup", B=3, p_lo=3000, p_hi=20000, H=64, d=128, k=256, c=512, g=4, seed=29)
    x = inputs.make_decode(s)
    vid = np.random.default_rng(31).integers(0, 40, size=x["k"].shape[0])
    x["k"] = np.ascontiguousarray(x["k"][vid])
    fails, (u_idx, u_sc, r_idx, r_sc, r_c, r_cs) = _decode_batch_fails(orc, s, x)
    assert not fails, summarize(fails)
    off = x["offsets"]

    def lowest_copies(row, sc, b, t, what):
        got = row[row >= 0].astype(np.int64)
        v = vid[off[b] + got]
        for u in np.unique(v):
            mine = got[v == u]
            assert np.unique(sc[row >= 0][v == u]).size == 1, f"{what}: copies of one key scored differently"
            pos = np.flatnonzero(vid[off[b]:off[b] + t + 1] == u)
            assert np.array_equal(np.sort(mine), pos[:mine.size]), f"{what}: vector {u} not its lowest copies"

    for b in range(s.B):
        Pb = int(off[b + 1] - off[b])
        lowest_copies(r_c[b], r_cs[b], b, Pb - 1, f"C_{b}")
        for r in range(s.g):
            lowest_copies(u_idx[b * s.g + r], u_sc[b * s.g + r], b, Pb - s.g + r, f"reuse b={b} r={r}")


def _split_run(s, world):
    """The decode step with every prefix split over `world` ranks, run rank after rank on this GPU."""
    def run(q, w, kc, off):
        u_idx, u_sc = MG.decode_split_emulated(P.OP_REUSE, q, w, kc, off, world, s.k, s.c, s.g, scores=True)
        r_idx, r_sc, r_c, r_cs = MG.decode_split_emulated(P.OP_REFINE, q, w, kc, off, world, s.k, s.c, s.g,
                                                         scores=True)
        return u_idx, u_sc, r_idx, r_sc, r_c, r_cs
    return run


@pytest.mark.parametrize("world", [2, 3])
def test_decode_prefix_split_small_ragged(orc, world):
    """One long prefix over ranks (C ABI pivot_decode_shard_select / _merge / _shard_rescore /
    _rowselect): prefixes of 4 to 3000 keys in 2 or 3 shards, some at or under c and k + g - 1;
    every C row, Reuse row and Refine row against the oracle."""
    s = inputs.DecodeSpec("small", B=5, p_lo=4, p_hi=3000, H=64, d=128, k=64, c=128, g=4, seed=21)
    fails, _ = _decode_batch_fails(orc, s, inputs.make_decode(s), run=_split_run(s, world))
    assert not fails, summarize(fails)


def test_decode_prefix_split_full_batch_matches_one_call(orc):
    """The full decode batch split over 3 ranks writes exactly the rows of the one-call decode
    (the same scores and the same exact selections), and its rows pass the oracle."""
    s = inputs.DECODE
    x = inputs.make_decode(s)
    fails, got = _decode_batch_fails(orc, s, x, run=_split_run(s, 3))
    assert not fails, summarize(fails)
    q, w, kc = dev(x["q"]), dev(x["w"]), dev(x["k"])
    off = x["offsets"]
    u_idx, _ = P.reuse_varlen(q, w, kc, off, s.k, s.g)
    r_idx, _, r_c, _ = P.refine_varlen(q, w, kc, off, s.k, s.c, s.g, cand=True)
    for a, b_ in ((got[0], u_idx), (got[2], r_idx), (got[4], r_c)):
        assert np.array_equal(np.sort(a, axis=1), np.sort(host(b_), axis=1))


def test_decode_small_ragged(orc):
    """Five sequences with prefixes from 4 to 3000 keys (several at or under c and k + g - 1):
    every C row, Reuse row and Refine row against the oracle."""
    s = inputs.DecodeSpec("small", B=5, p_lo=4, p_hi=3000, H=64, d=128, k=64, c=128, g=4, seed=21)
    fails, _ = _decode_batch_fails(orc, s, inputs.make_decode(s))
    assert not fails, summarize(fails)


# ---------------------------------------------------------------- scan visiting orders


def test_sampled_order_natural_order_and_fallback_agree(orc):
    """The scan's sampled threshold estimate (default), natural tile order (flag 2)
    and a too-high estimate that forces every long item to be scanned again
    (flag 4) select exactly the same sets; a few groups are also checked
    against the oracle."""
    L, topk, c, g = 16384, 256, 512, 8
    x = inputs.random_prefill(L, 64, 128, inputs.BF16, seed=61, rho=0.9, heavy=0.02)
    q, w, k = dev(x["q"]), dev(x["w"]), dev(x["k"])
    runs = {}
    try:
        for flags in (0, 2, 4):
            P.set_debug_flags(flags)
            d_idx, _ = P.indexer_dense(q, w, k, topk)
            u_idx, _ = P.reuse(q, w, k, topk, g)
            r_idx, _, r_c, _ = P.refine(q, w, k, topk, c, g, cand=True)
            torch.cuda.synchronize()
            runs[flags] = [host(t) for t in (d_idx, u_idx, r_idx, r_c)]
    finally:
        P.set_debug_flags(0)
    for flags in (2, 4):
        for name, a0, a1 in zip(("dense", "reuse", "refine", "cand"), runs[0], runs[flags]):
            assert np.array_equal(np.sort(a0, axis=1), np.sort(a1, axis=1)), \
                f"{name}: flags {flags} differ from the sampled order"
    G = (L + g - 1) // g
    groups = [0, 1, G // 3, G - 2, G - 1]
    fails = check_refine(orc, x, runs[0][2], None, runs[0][3], None, groups, topk, c, g)
    assert not fails, summarize(fails)


# ---------------------------------------------------------------- one sequence split into group ranges


def test_group_ranges_reproduce_the_whole_sequence(orc):
    """The zig-zag chunks of a 4-rank split, each run as a group-range call with only
    its rows and its key prefix, give exactly the rows of the whole-sequence call
    (dense, Reuse, Refine; tensor-core and CUDA-core paths), and the rows assembled
    from the chunks pass the oracle checks on every group."""
    from top_token_selection_proxy_b200 import multigpu as M

    for x, topk, c, g in ((inputs.random_prefill(4096, 64, 128, inputs.BF16, seed=73), 128, 256, 8),
                          (inputs.make_prefill(inputs.TINY), inputs.TINY.k, inputs.TINY.c, inputs.TINY.g)):
        q, w, k = dev(x["q"]), dev(x["w"]), dev(x["k"])
        L = x["q"].shape[0]
        G = (L + g - 1) // g
        full = {"dense": host(P.indexer_dense(q, w, k, topk)[0]), "reuse": host(P.reuse(q, w, k, topk, g)[0]),
                "refine": host(P.refine(q, w, k, topk, c, g)[0])}
        got = {n: np.full((L, topk), -2, np.int32) for n in ("dense", "reuse", "refine")}
        got_sc = {n: np.full((L, topk), np.nan, np.float32) for n in got}
        cand = np.full((G, c), -2, np.int32)
        world = 4
        for r in range(world):
            for t0, t1 in M.zigzag_chunks(L, g, world, r):
                qr, wr, kp = q[t0:t1].contiguous(), w[t0:t1].contiguous(), k[:t1].contiguous()
                d_i, d_s = P.indexer_dense_range(qr, wr, kp, L, topk, t0, t1, scores=True)
                u_i, u_s = P.reuse_range(qr, wr, kp, L, topk, g, t0 // g, t1 // g if t1 < L else G, scores=True)
                r_i, r_s, r_c, _ = P.refine_range(qr, wr, kp, L, topk, c, g, t0 // g, t1 // g if t1 < L else G,
                                                  scores=True, cand=True)
                torch.cuda.synchronize()
                for n, (i_, s_) in (("dense", (d_i, d_s)), ("reuse", (u_i, u_s)), ("refine", (r_i, r_s))):
                    got[n][t0:t1], got_sc[n][t0:t1] = host(i_), host(s_)
                cand[t0 // g:(t1 + g - 1) // g] = host(r_c)
        for name in full:
            assert (got[name] != -2).all(), f"{name}: rows not covered by the chunks"
            assert np.array_equal(np.sort(got[name], axis=1), np.sort(full[name], axis=1)), f"{name}, L = {L}"
        assert (cand != -2).all()
        fails = check_dense(orc, x, got["dense"], got_sc["dense"], range(L), topk)
        fails += check_reuse(orc, x, got["reuse"], got_sc["reuse"], range(G), topk, g)
        fails += check_refine(orc, x, got["refine"], got_sc["refine"], cand, None, range(G), topk, c, g)
        assert not fails, summarize(fails)


def test_streamed_refine_from_host_memory_matches_one_call(orc):
    """refine_host (pivot_refine_host: pinned host inputs, copies overlapped with group-range calls in
    chunks) writes exactly the rows of one device-resident refine call, for a ragged
    length and chunk counts that do and do not divide the groups; twice in a row
    (buffer reuse, earlier output overwritten).  Its rows also pass the oracle's
    re-scoring and top-k (Eq. 8-9) over the one call's candidate sets, every group."""
    x = inputs.random_prefill(6001, 64, 128, inputs.BF16, seed=79)
    topk, c, g = 128, 256, 8
    q, w, k = dev(x["q"]), dev(x["w"]), dev(x["k"])
    one_idx, _, one_c, one_cs = P.refine(q, w, k, topk, c, g, scores=True, cand=True)
    want = np.sort(host(one_idx), axis=1)
    cand, cand_sc = host(one_c), host(one_cs)
    qh = torch.from_numpy(x["q"].view(np.int16)).pin_memory().view(torch.bfloat16)
    wh = torch.from_numpy(x["w"]).pin_memory()
    kh = torch.from_numpy(x["k"].view(np.int16)).pin_memory().view(torch.bfloat16)
    oh = torch.empty((q.shape[0], topk), dtype=torch.int32).pin_memory()
    G = (6001 + g - 1) // g
    for chunks in (1, 3, 8, 8):
        oh.fill_(-7)
        P.refine_host(qh, wh, kh, topk, c, g, out_host=oh, chunks=chunks)
        torch.cuda.current_stream().synchronize()
        assert np.array_equal(np.sort(oh.numpy(), axis=1), want), f"chunks = {chunks}"
    fails = check_refine(orc, x, oh.numpy().copy(), None, cand, cand_sc, range(G), topk, c, g)
    assert not fails, summarize(fails)


# ---------------------------------------------------------------- proxy aggregation variants


@pytest.mark.parametrize("agg", ["first", "last"])
def test_aggregation_variants_every_group(orc, agg):
    """First- / last-query proxies (the ablation's aggregation variants) on both
    kernel paths, every group against the oracle."""
    for x, topk, c, g in ((inputs.random_prefill(1337, 64, 128, inputs.BF16, seed=71), 64, 128, 8),
                          (inputs.make_prefill(inputs.TINY), inputs.TINY.k, inputs.TINY.c, inputs.TINY.g)):
        q, w, k = dev(x["q"]), dev(x["w"]), dev(x["k"])
        L = x["q"].shape[0]
        G = (L + g - 1) // g
        u_idx, u_sc = P.reuse(q, w, k, topk, g, scores=True, aggregation=agg)
        r_idx, r_sc, r_c, r_cs = P.refine(q, w, k, topk, c, g, scores=True, cand=True, aggregation=agg)
        torch.cuda.synchronize()
        fails = check_reuse(orc, x, host(u_idx), host(u_sc), range(G), topk, g, agg)
        fails += check_refine(orc, x, host(r_idx), host(r_sc), host(r_c), host(r_cs), range(G), topk, c, g, agg)
        assert not fails, summarize(fails)


# ---------------------------------------------------------------- guardrail


def test_guardrail_runs_the_chosen_path_exactly(orc):
    """Behind the guardrail the call returns exactly the rows of the path it picks:
    dense at short context (c >= L), Refine / Reuse otherwise; the guarded rows also
    pass the oracle checks of that path on every row."""
    g, c, topk = 8, 512, 256
    for L, want_dense in ((400, True), (4096, False)):
        x = inputs.random_prefill(L, 64, 128, inputs.BF16, seed=40 + L)
        q, w, k = dev(x["q"]), dev(x["w"]), dev(x["k"])
        G = (L + g - 1) // g
        assert P.guardrail_dense(P.OP_REFINE, L, c, g) == want_dense
        gi, gs, ran_dense = P.refine_guarded(q, w, k, topk, c, g, scores=True)
        assert ran_dense == want_dense
        if want_dense:
            ri, rs = P.indexer_dense(q, w, k, topk, scores=True)
            rc = None
        else:
            ri, rs, rc, _ = P.refine(q, w, k, topk, c, g, scores=True, cand=True)
        torch.cuda.synchronize()
        assert np.array_equal(np.sort(host(gi), axis=1), np.sort(host(ri), axis=1))
        if want_dense:
            fails = check_dense(orc, x, host(gi), host(gs), range(L), topk)
        else:  # the guarded call's rows against the oracle over the Refine path's C_i
            fails = check_refine_rows(orc, x, host(gi), host(gs), host(rc), range(G), topk, g)
        ui, us, ran_dense_u = P.reuse_guarded(q, w, k, topk, g, scores=True)
        assert not ran_dense_u
        torch.cuda.synchronize()
        assert np.array_equal(np.sort(host(ui), axis=1), np.sort(host(P.reuse(q, w, k, topk, g)[0]), axis=1))
        fails += check_reuse(orc, x, host(ui), host(us), range(G), topk, g)
        assert not fails, summarize(fails)
    # g = 1: Reuse and dense do the same work, the guardrail runs dense
    x = inputs.random_prefill(300, 64, 128, inputs.BF16, seed=41)
    q, w, k = dev(x["q"]), dev(x["w"]), dev(x["k"])
    ui, us, ran_dense_u = P.reuse_guarded(q, w, k, 64, 1, scores=True)
    assert ran_dense_u
    assert np.array_equal(np.sort(host(ui), axis=1), np.sort(host(P.indexer_dense(q, w, k, 64)[0]), axis=1))
    fails = check_dense(orc, x, host(ui), host(us), range(300), 64)
    assert not fails, summarize(fails)


# ---------------------------------------------------------------- failure paths (no GPU fault)


def test_forced_device_timeout_is_reported_and_context_survives(orc):
    L, topk, g = 600, 16, 4
    x = inputs.random_prefill(L, 64, 128, inputs.BF16, seed=15)
    q, w, k = dev(x["q"]), dev(x["w"]), dev(x["k"])
    ws = P.Workspace()
    try:
        P.set_device_timeout_ns(50_000_000)
        P.set_debug_flags(1)
        P.reuse(q, w, k, topk, g, ws=ws)
        assert P.last_device_status(ws) == 5  # PIVOT_ERR_DEVICE_TIMEOUT
    finally:
        P.set_debug_flags(0)
        P.set_device_timeout_ns(2_000_000_000)
    idx, sc = P.reuse(q, w, k, topk, g, ws=ws, scores=True)
    assert P.last_device_status(ws) == 0
    fails = check_reuse(orc, x, host(idx), host(sc), range((L + g - 1) // g), topk, g)
    assert not fails, summarize(fails)


def test_invalid_calls_raise():
    x = inputs.random_prefill(64, 64, 128, inputs.BF16, seed=16)
    q, w, k = dev(x["q"]), dev(x["w"]), dev(x["k"])
    with pytest.raises(P.PivotError):
        P.refine(q, w, k, 32, 16, 4)  # c < k
    with pytest.raises(P.PivotError):
        P.reuse(q, w, k, 8, 17)  # g > 16
