"""World-size-2 CPU (gloo) test of the multi-rank host logic the bench runs under
torchrun: per-rank sequences, barriers with rank-0-only work between them, the
max-over-ranks time and the whole-job throughput."""
from __future__ import annotations

import dataclasses
import hashlib
import json
import os
import socket
import time

import pytest
import torch
import torch.multiprocessing as mp

from top_token_selection_proxy_b200 import inputs
from top_token_selection_proxy_b200 import multigpu as M


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, outdir: str) -> None:
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    w, r, lr = M.env()
    assert (w, r, lr) == (world, rank, rank)
    M.init("gloo", w, timeout_s=60.0)
    # each rank's own sequence, from its own seed (rank 0 keeps the workload's seed)
    spec = dataclasses.replace(inputs.TINY, seed=M.rank_seed(inputs.TINY.seed, r))
    x = inputs.make_prefill(spec)
    digest = hashlib.sha256(x["q"].tobytes() + x["k"].tobytes() + x["w"].tobytes()).hexdigest()
    # rank-0-only work between barriers (the bench's side measurements) must not strand the others
    M.barrier(w)
    if r == 0:
        time.sleep(0.3)
    M.barrier(w)
    mx = M.max_over_ranks(3.0 + 4.0 * r, w)
    ms, value = M.weak_scaling(10.0 + 5.0 * r, 2, 1000, w)
    with open(os.path.join(outdir, f"rank{r}.json"), "w") as f:
        json.dump({"seed": spec.seed, "digest": digest, "max": mx, "ms": ms, "value": value}, f)
    M.finish(w)


@pytest.mark.timeout(300)
def test_two_ranks_gloo(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert res[0]["seed"] == inputs.TINY.seed
    assert res[1]["seed"] == inputs.TINY.seed + M.SEED_STRIDE
    assert res[0]["digest"] != res[1]["digest"], "ranks must index different sequences"
    for r in res:
        assert r["max"] == 7.0
        assert r["ms"] == pytest.approx(15.0 / 2)                      # slowest rank's total / steps
        assert r["value"] == pytest.approx(world * 1000 / (7.5e-3))     # all ranks' units / that time


def test_single_rank_needs_no_process_group():
    assert not torch.distributed.is_initialized()
    assert M.max_over_ranks(2.5, 1) == 2.5
    assert M.weak_scaling(30.0, 3, 10, 1) == (10.0, pytest.approx(1000.0))
    M.barrier(1)
    M.finish(1)


# ---------------------------------------------------------------- one sequence over several ranks


def _zigzag_case(world: int):
    """(L, g, k, c) of the zig-zag test: L a multiple of 2 * world * g."""
    return 48 * world, 4, 8, 16


def _zigzag_rank(rank: int, world: int, port: int, outdir: str) -> None:
    import numpy as np

    from oracle import oracle as orc

    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    M.init("gloo", world, timeout_s=60.0)
    L, g, k, c = _zigzag_case(world)
    x = inputs.random_prefill(L, 4, 16, inputs.F32, seed=97)   # every rank draws the same sequence
    chunks = M.zigzag_chunks(L, g, world, rank)
    # the rank holds only its chunks' rows; split_step gathers the keys and indexes each chunk
    q_loc, w_loc = M.local_rows(x["q"], chunks), M.local_rows(x["w"], chunks)
    k_loc = M.local_rows(torch.from_numpy(x["k"]), chunks)
    seen = {}

    def index_fn(q_rows, w_rows, k_prefix, t0, t1):
        kp = k_prefix.numpy()
        seen[t0] = bool(np.array_equal(kp, x["k"][:t1]))
        # the chunk's groups from its own rows: a sequence whose rows before t0 are never read
        # except as keys (their queries are zero-filled here)
        qq = np.zeros((t1,) + x["q"].shape[1:], x["q"].dtype)
        ww = np.zeros((t1,) + x["w"].shape[1:], x["w"].dtype)
        qq[t0:t1], ww[t0:t1] = q_rows, w_rows
        idx, val, _, _ = orc.refine(qq, ww, kp, k, c, g, g0=t0 // g, g1=t1 // g)
        return idx, val

    rows = {}
    for t0, t1, (idx, val) in M.split_step(index_fn, q_loc, w_loc, k_loc, L, g, world, rank):
        rows[t0] = (idx.tolist(), np.nan_to_num(val, nan=7.0).tolist())
    work = [M.chunk_work(L, g, c, t0, t1) for t0, t1 in chunks]
    with open(os.path.join(outdir, f"zz{rank}.json"), "w") as f:
        json.dump({"keys_equal": all(seen.values()) and len(seen) == 2, "rows": rows, "work": sum(work)}, f)
    M.finish(world)


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world", [2, 3])
def test_one_sequence_zigzag_over_ranks(tmp_path, orc, world):
    import numpy as np

    mp.spawn(_zigzag_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"zz{r}.json")) for r in range(world)]
    assert all(r["keys_equal"] for r in res), "gathered keys differ from the sequence's keys"
    L, g, k, c = _zigzag_case(world)
    x = inputs.random_prefill(L, 4, 16, inputs.F32, seed=97)
    ref_idx, ref_val, _, _ = orc.refine(x["q"], x["w"], x["k"], k, c, g)
    covered = np.zeros(L, bool)
    for r in res:
        for t0, (idx, val) in r["rows"].items():
            t0 = int(t0)
            n = len(idx)
            assert np.array_equal(np.array(idx), ref_idx[t0:t0 + n])
            assert np.array_equal(np.array(val), np.nan_to_num(ref_val[t0:t0 + n], nan=7.0))
            assert not covered[t0:t0 + n].any()
            covered[t0:t0 + n] = True
    assert covered.all(), "every row is computed by exactly one rank"
    works = [r["work"] for r in res]
    assert max(works) - min(works) <= 0.1 * max(works), "zig-zag chunks balance the causal triangle"


def test_zigzag_layout():
    g = 8
    for world in (1, 2, 4, 8):
        L = 2 * world * g * 16
        seen = []
        for r in range(world):
            for t0, t1 in M.zigzag_chunks(L, g, world, r):
                assert t0 % g == 0 and t1 % g == 0 and t1 - t0 == L // (2 * world)
                seen.append((t0, t1))
        assert sorted(seen) == [(i * L // (2 * world), (i + 1) * L // (2 * world)) for i in range(2 * world)]
        works = [sum(M.chunk_work(L, g, 4096, t0, t1) for t0, t1 in M.zigzag_chunks(L, g, world, r))
                 for r in range(world)]
        assert max(works) <= 1.12 * min(works)
    with pytest.raises(ValueError):
        M.zigzag_chunks(100, 8, 2, 0)


# ---------------------------------------------------------------- one long decode prefix over ranks


def _split_case():
    """A small decode batch whose prefixes are split over the ranks (P_b >= 3 for world 3)."""
    return inputs.DecodeSpec("split", B=3, p_lo=40, p_hi=300, H=4, d=16, k=8, c=24, g=4, seed=83, dtype=inputs.F32)


def _oracle_split_fns(x, rank, world, variant, orc):
    """The split step's four functions on the CPU: the oracle's scores (Eq. 5 for the proxies,
    Eq. 8 for the members) with the selections written out in numpy.  Entries travel as
    (score, position) tensors; a candidate's member scores are 0 on the ranks that do not hold it."""
    import numpy as np

    s = _split_case()
    off = x["offsets"]
    B, g, k, c = s.B, s.g, s.k, s.c
    plen = np.diff(off)
    mem = [list(range(b * g, b * g + g)) for b in range(B)]
    qv, wv = orc.proxies(x["q"], x["w"], mem)
    F = orc.scores_batch(qv, wv, x["k"], plen=plen, key_base=off[:-1])
    cuts = M.decode_shards(plen, world, rank)
    n = k + g - 1 if variant == 0 else c

    def top(sc, ix, m):  # the m best by (score desc, position asc)
        keep = ix >= 0
        sc, ix = sc[keep], ix[keep]
        o = np.lexsort((ix, -sc))[:m]
        return sc[o], ix[o]

    def select_fn():  # this rank's shard of every prefix: its exact top-n
        sc = np.full((B, n), -np.inf)
        ix = np.full((B, n), -1, np.int64)
        for b, (lo, hi) in enumerate(cuts):
            f, p = top(F[b, lo:hi], np.arange(lo, hi), n)
            sc[b, :f.size], ix[b, :p.size] = f, p
        return torch.from_numpy(sc), torch.from_numpy(ix)

    def merge_fn(gathered):
        sc, ix = gathered[0].numpy(), gathered[1].numpy()  # [R, B, n]
        if variant == 0:  # Reuse rows: member t keeps the k best of the selection's entries <= t
            rows = []
            for b in range(B):
                f, p = top(sc[:, b].ravel(), ix[:, b].ravel(), min(n, plen[b]))
                for r in range(g):
                    e = p <= plen[b] - g + r
                    rows.append(sorted(top(f[e], p[e], k)[1].tolist()))
            return rows
        C = np.full((B, c), -1, np.int64)
        CL = np.full((B, c), -1, np.int64)
        for b in range(B):
            p = top(sc[:, b].ravel(), ix[:, b].ravel(), min(c, plen[b]))[1]
            C[b, :p.size] = p
            lo, hi = cuts[b]
            held = (p >= lo) & (p < hi)
            CL[b, :p.size][held] = p[held] - lo
        return C, CL

    def rescore_fn(merged):
        C, CL = merged
        qm, wm = orc.query_rows(x["q"], x["w"], list(range(B * g)))
        key_rows = np.full((B * g, c), -1, np.int64)
        for b in range(B):
            held = CL[b] >= 0
            for r in range(g):
                key_rows[b * g + r, held] = C[b, held]
        Ms = orc.scores_batch(qm, wm, x["k"], key_rows=key_rows, key_base=np.repeat(off[:-1], g))
        held = key_rows >= 0
        return torch.from_numpy(np.where(held, Ms, 0.0)), torch.from_numpy(held.astype(np.int64))

    def rowselect_fn(summed, merged):
        C = merged[0]
        Ms, cnt = summed[0].numpy(), summed[1].numpy()
        rows, once = [], True
        for b in range(B):
            valid = C[b] >= 0
            once &= bool((cnt[b * g:(b + 1) * g][:, valid] == 1).all())
            for r in range(g):
                e = valid & (C[b] <= plen[b] - g + r)
                rows.append(sorted(top(Ms[b * g + r][e], C[b][e], k)[1].tolist()))
        return rows, once

    if variant == 0:
        return select_fn, merge_fn, None, None
    return select_fn, merge_fn, rescore_fn, rowselect_fn


def _decode_split_rank(rank: int, world: int, port: int, outdir: str) -> None:
    from oracle import oracle as orc

    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    M.init("gloo", world, timeout_s=60.0)
    x = inputs.make_decode(_split_case())  # every rank draws the same batch and keeps its shards' keys
    out = {}
    for variant in (0, 1):
        sel, merge, rescore, rowsel = _oracle_split_fns(x, rank, world, variant, orc)
        res = M.decode_split_step(sel, merge, world, rescore, rowsel)
        out[variant] = {"rows": res} if variant == 0 else {"rows": res[0], "held_once": res[1]}
    with open(os.path.join(outdir, f"ds{rank}.json"), "w") as f:
        json.dump(out, f)
    M.finish(world)


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world", [2, 3])
def test_decode_prefix_split_over_ranks(tmp_path, orc, world):
    """One all-gather of the shards' exact top-n and a merge give every rank the Reuse rows of the
    whole prefixes; Refine's per-rank re-scoring of held candidates and one element-wise sum give
    its rows.  Both equal the oracle's decode on the unsplit batch."""
    import numpy as np

    mp.spawn(_decode_split_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"ds{r}.json")) for r in range(world)]
    s = _split_case()
    x = inputs.make_decode(s)
    for variant in (0, 1):
        idx = orc.decode(x["q"], x["w"], x["k"], x["offsets"], s.k, s.c, s.g, variant)[0]
        want = [sorted(int(v) for v in row if v >= 0) for row in idx]
        for r in res:
            assert r[str(variant)]["rows"] == want, f"variant {variant}: split rows differ from the whole prefix"
            if variant == 1:
                assert r["1"]["held_once"], "every candidate is held by exactly one rank"


def test_decode_shards_partition_every_prefix():
    import numpy as np

    plen = [3, 7, 100, 4097]
    for world in (1, 2, 3):
        cover = [np.zeros(P, int) for P in plen]
        for rank in range(world):
            for b, (lo, hi) in enumerate(M.decode_shards(plen, world, rank)):
                assert hi - lo >= 1
                cover[b][lo:hi] += 1
        assert all((cv == 1).all() for cv in cover)
    with pytest.raises(ValueError):
        M.decode_shards([2], 3, 0)
    k = np.arange(20 * 2).reshape(20, 2)
    off = np.array([0, 8, 20])
    ks, so, pb = M.shard_of(k, off, 2, 1)
    assert so.tolist() == [0, 4, 10] and pb.tolist() == [4, 6]
    assert np.array_equal(ks, np.concatenate([k[4:8], k[14:20]]))


def test_decode_split_step_single_rank_passes_through():
    """With one rank the exchanges are a leading axis of 1 and the identity, and the step runs
    select -> merge (Reuse), or select -> merge -> rescore -> row select (Refine), in that order."""
    calls = []

    def select_fn():
        calls.append("select")
        return torch.arange(6).reshape(2, 3), torch.zeros(2, 3)

    def merge_fn(g_):
        calls.append("merge")
        assert g_[0].shape == (1, 2, 3) and g_[1].shape == (1, 2, 3)
        return "C", "C_local", None

    def rescore_fn(merged):
        calls.append("rescore")
        assert merged[1] == "C_local"
        return torch.ones(4, 5, dtype=torch.int32)

    def rowselect_fn(keys, merged):
        calls.append("rowselect")
        assert torch.equal(keys, torch.ones(4, 5, dtype=torch.int32)) and merged[0] == "C"
        return "rows"

    assert M.decode_split_step(select_fn, merge_fn, 1) == ("C", "C_local", None)
    assert calls == ["select", "merge"]
    calls.clear()
    assert M.decode_split_step(select_fn, merge_fn, 1, rescore_fn, rowselect_fn) == "rows"
    assert calls == ["select", "merge", "rescore", "rowselect"]
    k = torch.arange(20 * 2).reshape(20, 2)
    ks, so, pb = M.shard_of(k, [0, 8, 20], 2, 0)
    assert torch.equal(ks, torch.cat([k[0:4], k[8:14]])) and so.tolist() == [0, 4, 10] and pb.tolist() == [0, 0]
