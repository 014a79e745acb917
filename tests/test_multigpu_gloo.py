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
