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
