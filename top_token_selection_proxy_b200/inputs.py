"""Seeded synthetic inputs for the PIVOT indexer workloads.

This module only draws random numbers and lays them out; it holds none of
the indexer's arithmetic (no scores, no pooling, no selection).  Both the
CUDA path's tests/bench and the CPU oracle are fed from here.

The workloads stand in for the activations of a DSA indexer (PIVOT, picx.dev
summary, "Key observations", O1 and O3): keys with a long-tailed score
profile, and queries that change slowly along the sequence so that
neighbouring queries pick overlapping keys.

Recipe (numpy ``PCG64`` generators seeded from ``SeedSequence(seed).spawn``,
one child stream per item below, so that chunks can be drawn in parallel
threads and the result does not depend on the thread count):

* ``u``: one random unit vector in R^d shared by all heavy keys.
* keys ``k_s ~ N(0, I/d)``; a subset of ``round(heavy * L)`` positions, drawn
  without replacement, gets ``k_s += 3 u`` (a shift of norm 3).
* queries, per head, AR(1) along t: ``q_0 = e_0``,
  ``q_t = rho q_{t-1} + e_t`` with innovations ``e_t ~ N(0, I/d)`` (float32),
  drawn in t-chunks of 8192 rows; each chunk is filtered from a zero state and
  then carried: ``q_t += rho^(t - t0 + 1) q_{t0 - 1}``.
* ``w ~ N(0, 1/H)`` i.i.d. per (t, head).
* bf16 tensors are rounded to nearest-even from float32 (torch CPU cast) and
  handed around as uint16 bit patterns.

Decode batches (one MTP group per sequence): prefix lengths
``P_b ~ U[p_lo, p_hi]``; each sequence's keys follow the key recipe; the
current query row is drawn from the AR(1) stationary law
``N(0, I/(d (1 - rho^2)))`` per head, the g-1 draft rows are the current row
plus ``N(0, 0.1^2/d)`` noise, and every draft row repeats the current row's w.
"""
from __future__ import annotations

import dataclasses
import os

import numpy as np

BF16 = "bf16"
F32 = "f32"


@dataclasses.dataclass(frozen=True)
class PrefillSpec:
    name: str
    L: int
    H: int
    d: int
    k: int
    c: int
    g: int
    dtype: str = BF16
    rho: float = 0.95
    heavy: float = 0.01
    seed: int = 0


@dataclasses.dataclass(frozen=True)
class DecodeSpec:
    name: str
    B: int
    p_lo: int
    p_hi: int
    H: int
    d: int
    k: int
    c: int
    g: int
    dtype: str = BF16
    rho: float = 0.95
    heavy: float = 0.01
    draft_sigma: float = 0.1
    seed: int = 0


SEED_BASE = 20261200

# The five workloads, with their sizes.  The seed of workload n is SEED_BASE + n.
TINY = PrefillSpec("tiny_L512_H4_d32_g4_f32", L=512, H=4, d=32, k=16, c=32, g=4,
                   dtype=F32, rho=0.95, heavy=0.02, seed=SEED_BASE + 1)
PREFILL_8K = PrefillSpec("prefill_L8192_g8", L=8192, H=64, d=128, k=2048, c=4096, g=8,
                         seed=SEED_BASE + 2)
LONG_128K = PrefillSpec("prefill_L131072_g8", L=131072, H=64, d=128, k=2048, c=4096, g=8,
                        seed=SEED_BASE + 4)
DECODE = DecodeSpec("decode_B32_P16k-200k_g4", B=32, p_lo=16384, p_hi=200000, H=64, d=128,
                    k=2048, c=4096, g=4, seed=SEED_BASE + 5)


def sweep_32k(g: int, rho: float) -> PrefillSpec:
    """Group-size sweep at L=32768; one seed per rho so the g axis sees the same inputs."""
    seed = SEED_BASE + 3 + (0 if rho == 0.9 else 100)
    return PrefillSpec(f"sweep_L32768_g{g}_rho{rho}", L=32768, H=64, d=128, k=2048, c=4096,
                       g=g, rho=rho, seed=seed)


SWEEP_G = (1, 4, 8, 16)
SWEEP_RHO = (0.9, 0.98)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float array -> bf16 bit patterns (uint16), round to nearest even."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact float32 values."""
    return (b.astype(np.uint32) << 16).view(np.float32)


def _cast(x: np.ndarray, dtype: str) -> np.ndarray:
    return to_bf16_bits(x) if dtype == BF16 else np.ascontiguousarray(x, dtype=np.float32)


def _keys(rng: np.random.Generator, n: int, d: int, heavy: float, u: np.ndarray) -> np.ndarray:
    k = rng.standard_normal((n, d), dtype=np.float32) * np.float32(1.0 / np.sqrt(d))
    nh = int(round(heavy * n))
    if nh > 0:
        pos = rng.choice(n, size=nh, replace=False)
        k[pos] += (3.0 * u).astype(np.float32)
    return k


def _unit(rng: np.random.Generator, d: int) -> np.ndarray:
    u = rng.standard_normal(d)
    return u / np.linalg.norm(u)


def _threads() -> int:
    try:
        return max(1, min(16, len(os.sched_getaffinity(0))))
    except AttributeError:  # pragma: no cover
        return 4


def _ar1_chunk(seed: np.random.SeedSequence, n: int, H: int, d: int, rho: float) -> np.ndarray:
    """Zero-state AR(1) of n rows of N(0, I/d) innovations (float32)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    e = rng.standard_normal((n, H, d), dtype=np.float32) * np.float32(1.0 / np.sqrt(d))
    r = np.float32(rho)
    for t in range(1, n):
        e[t] += r * e[t - 1]
    return e


def make_prefill(spec: PrefillSpec, chunk: int = 8192) -> dict:
    """q [L,H,d], w [L,H] float32, k [L,d]; q/k as bf16 bits or float32."""
    from concurrent.futures import ThreadPoolExecutor

    L, H, d = spec.L, spec.H, spec.d
    n_chunks = (L + chunk - 1) // chunk
    ss = np.random.SeedSequence(spec.seed).spawn(3 + n_chunks)
    u = _unit(np.random.Generator(np.random.PCG64(ss[0])), d)
    k = _cast(_keys(np.random.Generator(np.random.PCG64(ss[1])), L, d, spec.heavy, u), spec.dtype)
    w = (np.random.Generator(np.random.PCG64(ss[2])).standard_normal((L, H), dtype=np.float32)
         * np.float32(1.0 / np.sqrt(H)))
    qdt = np.uint16 if spec.dtype == BF16 else np.float32
    q = np.empty((L, H, d), dtype=qdt)
    bounds = [(c * chunk, min(L, c * chunk + chunk)) for c in range(n_chunks)]
    with ThreadPoolExecutor(_threads()) as ex:
        parts = list(ex.map(lambda c: _ar1_chunk(ss[3 + c], bounds[c][1] - bounds[c][0], H, d, spec.rho),
                            range(n_chunks)))
    prev = None
    r = np.float32(spec.rho)
    for c, (t0, t1) in enumerate(bounds):
        z = parts[c]
        if prev is not None:  # carry the state of the previous chunk: + rho^(i+1) * q_{t0-1}
            powers = r ** np.arange(1, t1 - t0 + 1, dtype=np.float32)
            z += powers[:, None, None] * prev[None]
        prev = z[-1].copy()
        q[t0:t1] = _cast(z, spec.dtype)
        parts[c] = None
    return {"q": q, "w": w, "k": k, "spec": spec}


def make_decode(spec: DecodeSpec) -> dict:
    """q [B*g,H,d], w [B*g,H], k_cache [sum P_b, d], offsets [B+1] int64."""
    from concurrent.futures import ThreadPoolExecutor

    B, H, d, g = spec.B, spec.H, spec.d, spec.g
    ss = np.random.SeedSequence(spec.seed).spawn(5 + B)
    u = _unit(np.random.Generator(np.random.PCG64(ss[0])), d)
    P = np.random.Generator(np.random.PCG64(ss[1])).integers(spec.p_lo, spec.p_hi, size=B,
                                                              endpoint=True).astype(np.int64)
    off = np.zeros(B + 1, dtype=np.int64)
    off[1:] = np.cumsum(P)
    kdt = np.uint16 if spec.dtype == BF16 else np.float32
    kc = np.empty((int(off[-1]), d), dtype=kdt)

    def fill(b):
        rng = np.random.Generator(np.random.PCG64(ss[5 + b]))
        kc[off[b]:off[b + 1]] = _cast(_keys(rng, int(P[b]), d, spec.heavy, u), spec.dtype)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(fill, range(B)))
    rq = np.random.Generator(np.random.PCG64(ss[2]))
    scale = 1.0 / np.sqrt(d * (1.0 - spec.rho ** 2))
    cur = rq.standard_normal((B, 1, H, d)) * scale
    drafts = cur + np.random.Generator(np.random.PCG64(ss[3])).standard_normal((B, g - 1, H, d)) * (
        spec.draft_sigma / np.sqrt(d))
    q = _cast(np.concatenate([cur, drafts], axis=1).reshape(B * g, H, d), spec.dtype)
    wc = (np.random.Generator(np.random.PCG64(ss[4])).standard_normal((B, 1, H)) / np.sqrt(H)).astype(np.float32)
    w = np.ascontiguousarray(np.repeat(wc, g, axis=1).reshape(B * g, H))
    return {"q": q, "w": w, "k": kc, "offsets": off, "spec": spec}


def sample_groups(n_groups: int, g: int, k: int, c: int, n: int, seed: int) -> np.ndarray:
    """Seeded sample of prefill group ids for the long-sequence checks.

    Always contains the first and last group and the groups whose prefix
    length P_i = min(i*g+g, L) straddles c and k+g-1; the rest are uniform
    without replacement."""
    must = {0, n_groups - 1}
    for edge in (c, k + g - 1):
        i = max(0, (edge - 1) // g)
        for j in (i - 1, i, i + 1):
            if 0 <= j < n_groups:
                must.add(j)
    rng = np.random.Generator(np.random.PCG64(seed))
    rest = np.setdiff1d(np.arange(n_groups), np.array(sorted(must)))
    take = max(0, min(n - len(must), rest.size))
    extra = rng.choice(rest, size=take, replace=False) if take else np.array([], dtype=np.int64)
    return np.sort(np.concatenate([np.array(sorted(must), dtype=np.int64), extra.astype(np.int64)]))


def random_prefill(L: int, H: int, d: int, dtype: str, seed: int, rho: float = 0.95,
                   heavy: float = 0.02, k: int = 8, c: int = 16, g: int = 4) -> dict:
    """Small ad-hoc prefill case (tests)."""
    return make_prefill(PrefillSpec(f"adhoc_{L}_{H}_{d}", L=L, H=H, d=d, k=k, c=c, g=g,
                                    dtype=dtype, rho=rho, heavy=heavy, seed=seed))


def host_bytes(x: dict) -> int:
    return sum(v.nbytes for v in x.values() if isinstance(v, np.ndarray))


__all__ = [
    "BF16", "F32", "PrefillSpec", "DecodeSpec", "TINY", "PREFILL_8K", "LONG_128K", "DECODE",
    "sweep_32k", "SWEEP_G", "SWEEP_RHO", "make_prefill", "make_decode", "sample_groups",
    "random_prefill", "to_bf16_bits", "bf16_bits_to_f32", "host_bytes",
]
