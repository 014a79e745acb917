"""One process per GPU.

Independent sequences per rank (weak scaling): PIVOT indexes each sequence's
groups independently of every other sequence, so N GPUs index N sequences with
no collective on the data path; the only collectives are the barriers around a
timed region and one max-reduction of the per-rank time.  The whole-job
throughput is the queries of all ranks over the slowest rank's time.

One sequence over N GPUs: zig-zag chunks of its groups per rank and one
all-gather of the key chunks (below).  One long decode prefix over N GPUs: a key
shard per rank, one all-gather of the shards' selections and a merge (Refine adds
one element-wise sum of the member scores).
"""
from __future__ import annotations

import datetime
import os
from typing import Tuple

import torch
import torch.distributed as dist

SEED_STRIDE = 7919  # rank r draws its sequence from seed + SEED_STRIDE * r


def env() -> Tuple[int, int, int]:
    """(world size, rank, local rank) from the launcher's environment (1, 0, 0 when absent)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, world: int, timeout_s: float = 300.0) -> None:
    """Join the process group when world > 1 (env:// rendezvous; MASTER_ADDR must be set)."""
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s sequence: rank 0 keeps the workload's own seed."""
    return seed + SEED_STRIDE * rank


def barrier(world: int) -> None:
    if world > 1:
        dist.barrier()


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The maximum of x over all ranks (x itself when world == 1)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling(total_ms_local: float, steps: int, units_per_rank: int, world: int, device=None):
    """(ms per step, whole-job units/s): every rank processed units_per_rank per step;
    the job takes as long as its slowest rank."""
    total_ms = max_over_ranks(total_ms_local, world, device)
    ms = total_ms / steps
    return ms, world * units_per_rank / (ms / 1000.0)


# ---------------------------------------------------------------- one sequence over several GPUs
# The groups of one prefill sequence are independent given its keys.  A zig-zag
# layout (the sequence cut into 2W equal chunks of whole groups; rank r holds
# chunks r and 2W-1-r) gives every rank an early and a late part of the causal
# triangle, so the per-rank work sum_i (P_i + |G_i| min(c, P_i)) is nearly equal.
# Each rank holds the queries, weights and keys of its own chunks; one
# all-gather of the key chunks gives every rank the keys its groups read.


def zigzag_chunks(L: int, g: int, world: int, rank: int):
    """Token ranges [(t0, t1), (t0', t1')] of rank `rank`: chunks rank and 2W-1-rank of
    2W chunks of equal size (a multiple of g; L must be a multiple of 2W*g)."""
    n = 2 * world
    if L % (n * g) != 0:
        raise ValueError(f"L = {L} must be a multiple of 2 * world * g = {n * g}")
    cs = L // n
    return [(rank * cs, (rank + 1) * cs), ((n - 1 - rank) * cs, (n - rank) * cs)]


def chunk_work(L: int, g: int, c: int, t0: int, t1: int) -> int:
    """sum over the groups of rows [t0, t1) of P_i + |G_i| * min(c, P_i) (Refine's key-row products)."""
    w = 0
    for i0 in range(t0, t1, g):
        P = min(i0 + g, L)
        w += P + (P - i0) * min(c, P)
    return w


def gather_keys(k_local: torch.Tensor, L: int, g: int, world: int) -> torch.Tensor:
    """All-gather of the zig-zag key chunks: k_local [2 * L / (2W), d] holds this rank's two
    chunks (in zigzag_chunks order); returns all L key rows in position order."""
    n = 2 * world
    cs = L // n
    if world <= 1:
        return k_local
    parts = [torch.empty_like(k_local) for _ in range(world)]
    dist.all_gather(parts, k_local.contiguous())
    full = torch.empty((L,) + tuple(k_local.shape[1:]), dtype=k_local.dtype, device=k_local.device)
    for r in range(world):
        for j, (t0, t1) in enumerate(zigzag_chunks(L, g, world, r)):
            full[t0:t1] = parts[r][j * cs:(j + 1) * cs]
    return full


def local_rows(a, chunks):
    """This rank's rows of a per-position array (numpy or torch): its chunks, concatenated
    in zigzag_chunks order."""
    parts = [a[t0:t1] for t0, t1 in chunks]
    if isinstance(a, torch.Tensor):
        return torch.cat(parts).contiguous()
    import numpy as np

    return np.ascontiguousarray(np.concatenate(parts))


def split_step(index_fn, q_local, w_local, k_local, L: int, g: int, world: int, rank: int):
    """One step of one sequence indexed by `world` ranks: the all-gather of the key chunks
    (the one exchange), then index_fn(q_rows, w_rows, k_prefix, t0, t1) on each of this
    rank's zig-zag chunks, with that chunk's query / weight rows and the key prefix
    [0, t1) it reads.  q_local / w_local / k_local hold the rank's chunks (local_rows).
    Returns [(t0, t1, index_fn's result)]."""
    k_full = gather_keys(k_local, L, g, world)
    out, off = [], 0
    for t0, t1 in zigzag_chunks(L, g, world, rank):
        n = t1 - t0
        out.append((t0, t1, index_fn(q_local[off:off + n], w_local[off:off + n], k_full[:t1], t0, t1)))
        off += n
    return out


# ---------------------------------------------------------------- one long decode prefix over ranks
# The groups' selections (Eq. 5-7) run over a whole prefix, and the exact top-n of a set lies in
# the union of the exact top-n of its parts.  So each rank holds one contiguous shard of every
# sequence's cached keys, selects its shard's top-n, and one all-gather plus a merge give the
# exact top-n of the whole prefix.  Refine then re-scores each candidate on the rank that holds
# its key (Eq. 8) and one element-wise sum gathers the member scores (every candidate is held by
# exactly one rank) before the member top-k (Eq. 9).


def decode_shards(plen, world: int, rank: int):
    """[(lo, hi)] per sequence: rank `rank`'s contiguous shard of each prefix of plen[b] keys
    (equal cuts; every shard holds at least one key, so plen[b] >= world)."""
    out = []
    for P in plen:
        P = int(P)
        if P < world:
            raise ValueError(f"a prefix of {P} keys cannot give {world} ranks a key each")
        out.append((P * rank // world, P * (rank + 1) // world))
    return out


def shard_of(k_cache, offsets, world: int, rank: int):
    """This rank's key rows (numpy or torch, in sequence order), their shard offsets [B+1] and
    the prefix position of each shard's first key [B]."""
    import numpy as np

    plen = np.diff(np.asarray(offsets, dtype=np.int64))
    cuts = decode_shards(plen, world, rank)
    rows = [k_cache[int(offsets[b]) + lo:int(offsets[b]) + hi] for b, (lo, hi) in enumerate(cuts)]
    if isinstance(k_cache, torch.Tensor):
        k_shard = torch.cat(rows).contiguous()
    else:
        k_shard = np.ascontiguousarray(np.concatenate(rows))
    shard_off = np.concatenate([[0], np.cumsum([hi - lo for lo, hi in cuts])]).astype(np.int64)
    pos_base = np.array([lo for lo, _ in cuts], dtype=np.int64)
    return k_shard, shard_off, pos_base


def gather_ranks(t, world: int):
    """All-gather of this rank's tensor (or tuple of tensors): [world, ...] each."""
    if isinstance(t, tuple):
        return tuple(gather_ranks(x, world) for x in t)
    if world <= 1:
        return t.unsqueeze(0)
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous())
    return torch.stack(parts)


def sum_ranks(t, world: int):
    """Element-wise sum over the ranks (in place; tuples element by element)."""
    if isinstance(t, tuple):
        return tuple(sum_ranks(x, world) for x in t)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t


def decode_split_step(select_fn, merge_fn, world: int, rescore_fn=None, rowselect_fn=None):
    """One decode step with every prefix split over `world` ranks: select_fn() -> this rank's
    shard selection; one all-gather; merged = merge_fn(gathered) -> the Reuse rows, or for
    Refine the candidate sets, which then go through rescore_fn(merged) -> this rank's held
    candidates' member scores, one element-wise sum, and rowselect_fn(summed, merged)."""
    merged = merge_fn(gather_ranks(select_fn(), world))
    if rescore_fn is None:
        return merged
    return rowselect_fn(sum_ranks(rescore_fn(merged), world), merged)


def device_split_fns(op: int, q, w, k_shard, shard_off, pos_base, plen_off, topk: int, c: int, g: int,
                     scores: bool = False):
    """The four steps on this rank's GPU through the library (the C ABI's pivot_decode_* calls).
    Reuse's merge returns (indices, scores|None); Refine's returns (C, C scores|None, C in this
    rank's shard rows) and its row select (indices, scores|None).  The offsets and shard positions
    go to the device once, here."""
    import top_token_selection_proxy_b200 as P

    shard_off = P.DeviceOffsets(shard_off, q.device)
    pos_base = P.DeviceOffsets(pos_base, q.device)
    plen_off = P.DeviceOffsets(plen_off, q.device)

    def select_fn():
        return P.decode_shard_select(op, q, w, k_shard, shard_off, pos_base, topk, c, g)

    def merge_fn(ent):
        if op == P.OP_REUSE:
            return P.decode_merge(op, ent, plen_off, topk, c, g, scores=scores)
        return P.decode_merge(op, ent, plen_off, topk, c, g, shard_offsets=shard_off, pos_base=pos_base,
                              scores=scores)

    def rescore_fn(merged):
        return P.decode_shard_rescore(q, w, k_shard, shard_off, pos_base, plen_off, merged[2], topk, c, g)

    def rowselect_fn(keys, merged):
        return P.decode_rowselect(keys, merged[0], plen_off, topk, c, g, scores=scores)

    if op == P.OP_REUSE:
        return select_fn, merge_fn, None, None
    return select_fn, merge_fn, rescore_fn, rowselect_fn


def decode_split_emulated(op: int, q, w, k_cache, offsets, world: int, topk: int, c: int, g: int,
                          scores: bool = False):
    """The split decode step of `world` ranks run one rank after another on this GPU (the
    exchanges become a stack and a sum; no kernel waits for another).  Reuse: (indices [B*g, k],
    scores|None); Refine: (indices, scores|None, C [B, c], C scores|None)."""
    import numpy as np

    plen_off = np.asarray(offsets, dtype=np.int64)
    shards = [shard_of(k_cache, plen_off, world, r) for r in range(world)]
    fns = [device_split_fns(op, q, w, ks, so, pb, plen_off, topk, c, g, scores) for ks, so, pb in shards]
    ent = torch.stack([f[0]() for f in fns])
    if fns[0][2] is None:
        return fns[0][1](ent)
    merged = [f[1](ent) for f in fns]  # every rank merges the same entries; each keeps its own local C
    keys = torch.stack([f[2](m) for f, m in zip(fns, merged)]).sum(0, dtype=torch.int64)
    keys = keys.to(torch.int32)  # every candidate is held by exactly one rank: no carry
    idx, sc = fns[0][3](keys, merged[0])
    return idx, sc, merged[0][0], merged[0][1]


def finish(world: int) -> None:
    """Every rank calls this last: a final barrier, then leave the process group."""
    if world > 1 and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()


__all__ = ["SEED_STRIDE", "env", "init", "rank_seed", "barrier", "max_over_ranks", "weak_scaling", "finish",
           "zigzag_chunks", "chunk_work", "gather_keys", "local_rows", "split_step",
           "decode_shards", "shard_of", "gather_ranks", "sum_ranks", "decode_split_step", "device_split_fns",
           "decode_split_emulated"]
