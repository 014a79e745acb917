#!/usr/bin/env python
"""Throughput of the PIVOT indexer library on B200.

One step = one PIVOT-Refine call (proxy pooling, proxy scan, streaming
candidate selection, candidate re-scoring and member top-k) over the
L = 131072, H_I = 64, d = 128, k = 2048, c = 4096, g = 8 prefill sequence
with inputs resident in HBM.  The metric is indexed queries per second.
The same run also times the dense indexer (g = 1) and PIVOT-Reuse on the
same inputs, the MTP decode batch, the CPU oracle on a bounded sample
(a baseline, not the target), and the call end to end through host buffers.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs its own sequence (independent
problems, no collective on the data path: weak scaling); rank 0 prints one
JSON line with the max-over-ranks time.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "indexer queries/sec at L=128K g=8 Refine (1×B200); % of roofline; × vs dense"
UNIT = "queries/s"
L2_FLUSH_BYTES = 256 << 20
E2E_CHUNKS = 8  # runs of groups the end-to-end call pipelines its copies over

# DRAM bytes (read + write) of one scan launch on this workload, from a 1-pass
# ncu capture (dram__bytes_read.sum + dram__bytes_write.sum); valid only while
# the sources the scan kernel is built from hash to `sources_sha256`.
SCAN_TRAFFIC = {
    "bytes": 2500000000 + 949310000,  # 2.50 GB + 949.31 MB, as ncu printed them
    "sources": ("scan.cu", "select.cuh", "ptx.cuh", "kernels.cuh", "headsum.cuh"),
    "sources_sha256": "09345fcff2aee30e9689cf7e53448ce1ce41b74bdae9b8721d517af192714fca",
    "profile": "profiles/kernels_prefill_L131072_g8_refine_1pass.md",
}


def scan_sources_sha256():
    import hashlib

    h = hashlib.sha256()
    for f in SCAN_TRAFFIC["sources"]:
        with open(os.path.join(ROOT, "top_token_selection_proxy_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def scan_traffic():
    """Measured DRAM bytes per scan launch, or None once the kernel changed since the capture."""
    try:
        return SCAN_TRAFFIC["bytes"] if scan_sources_sha256() == SCAN_TRAFFIC["sources_sha256"] else None
    except OSError:
        return None


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--no-extras", action="store_true", help="skip dense/Reuse/decode side measurements")
    p.add_argument("--no-configs", action="store_true", help="skip the per-workload lines (tiny, 8K, 32K sweep, "
                                                             "decode)")
    p.add_argument("--split", action="store_true",
                   help="one L=131072 sequence over all ranks (zig-zag group ranges + key all-gather; strong "
                        "scaling) instead of one sequence per rank")
    p.add_argument("--split-decode", action="store_true",
                   help="the MTP decode batch with every prefix split over all ranks (key shards, all-gather of "
                        "the shards' selections, merge; Refine re-scores held candidates and sums; strong "
                        "scaling)")
    p.add_argument("--profile-case", type=int, default=0, metavar="L",
                   help="profiling run: two PIVOT-Refine calls at sequence length L (H_I=64, d=128, k=2048, "
                        "c=4096, g=8) and exit; no timing, no JSON")
    p.add_argument("--profile-decode", action="store_true",
                   help="profiling run: the MTP decode batch (B=32, P_b in [16384, 200000], g=4), two PIVOT-Refine "
                        "then two PIVOT-Reuse calls, and exit; no timing, no JSON")
    return p.parse_args()


def run_profile_case(L):
    """Small case for ncu captures: a warm-up call, then the captured call."""
    import numpy as np
    import torch

    import top_token_selection_proxy_b200 as P
    from top_token_selection_proxy_b200 import build, inputs

    build.build()
    spec = inputs.PrefillSpec(f"profile_L{L}", L=L, H=64, d=128, k=2048, c=4096, g=8, seed=5)
    x = inputs.make_prefill(spec)
    dev = torch.device("cuda", 0)
    q, w, k = to_dev(x["q"], dev), to_dev(x["w"], dev), to_dev(x["k"], dev)
    ws = P.Workspace(dev)
    for _ in range(2):
        P.refine(q, w, k, spec.k, spec.c, spec.g, ws=ws)
    torch.cuda.synchronize()
    st = P.last_device_status(ws)
    print(f"profile case L={L}: status {P.STATUS.get(st, st)}")
    if st != 0:
        raise SystemExit(1)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return m["hbm_gbs"], m["bf16_tflops"], m["bf16_tflops_sustained"], "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def workload_flops_bytes(spec):
    """Algorithmic work of one PIVOT-Refine pass (FLOPs = 2*H*d per query-row/key pair)."""
    L, H, d, g, c, k = spec.L, spec.H, spec.d, spec.g, spec.c, spec.k
    G = (L + g - 1) // g
    f_scan = f_ref = 0
    for i in range(G):
        P = min(i * g + g, L)
        m = P - i * g
        f_scan += 2 * H * d * P
        f_ref += 2 * m * min(c, P) * H * d
    f_dense = 2 * H * d * L * (L + 1) // 2
    # q read twice (pooling, member re-scoring), w twice, keys once, C written + read, indices written
    b_alg = 2 * L * H * d * 2 + 2 * L * H * 4 + L * d * 2 + 2 * G * c * 4 + L * k * 4
    return f_scan, f_ref, f_dense, b_alg


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                       "-lms", "200", "-i", str(gpu_index)], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        time.sleep(0.3)
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = max(mx, float(r[2]))
                for n, v in zip(names, r[5:9]):
                    if "Active" in v and "Not" not in v:
                        reasons.add(n)
            except (ValueError, IndexError):
                pass
        if not sm:
            return None
        load = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_env():
    from top_token_selection_proxy_b200 import multigpu

    return multigpu.env()


def to_dev(a, dev):
    import numpy as np
    import torch

    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    return torch.from_numpy(a).to(dev)


def cpu_oracle_sample(x, spec, runs=24):
    """Oracle PIVOT-Refine on `runs` contiguous runs of groups spread over the
    sequence (one group per host thread each), so the sampled prefix lengths
    average those of the full workload.  Returns (rows/s, cores, description)."""
    from oracle import oracle as orc

    cores = len(os.sched_getaffinity(0))
    orc.set_threads(cores)
    G = (spec.L + spec.g - 1) // spec.g
    per = max(1, cores)
    rows = 0
    units_sampled = 0
    t0 = time.perf_counter()
    for j in range(runs):
        g0 = min(G - per, int((2 * j + 1) * G / (2 * runs)))
        orc.refine(x["q"], x["w"], x["k"], spec.k, spec.c, spec.g, g0=g0, g1=g0 + per)
        rows += per * spec.g
        units_sampled += refine_units(spec, g0, g0 + per)
    dt = time.perf_counter() - t0
    desc = (f"oracle PIVOT-Refine (double precision, OpenMP over groups) on {runs} runs of {per} consecutive "
            f"groups ({rows} query rows) centred at {runs} evenly spaced positions of the L={spec.L} sequence")
    return rows / dt, orc.threads(), desc, dt, units_sampled


def refine_units(spec, g0, g1):
    """Key-row products sum_i (P_i + |G_i| min(c, P_i)) of groups [g0, g1)."""
    u = 0
    for i in range(g0, g1):
        P = min(i * spec.g + spec.g, spec.L)
        u += P + (P - i * spec.g) * min(spec.c, P)
    return u


def prefill_work(spec, g=None):
    """(scan FLOPs, refine FLOPs, Refine key-row products sum_i (P_i + |G_i| min(c, P_i))) of one
    prefill sequence; FLOPs are 2*H*d per (query-or-proxy row, key) pair."""
    L, H, d, c = spec.L, spec.H, spec.d, spec.c
    g = spec.g if g is None else g
    f_scan = f_ref = units = 0
    for t0 in range(0, L, g):
        P = min(t0 + g, L)
        m = P - t0
        f_scan += 2 * H * d * P
        f_ref += 2 * m * min(c, P) * H * d
        units += P + m * min(c, P)
    return f_scan, f_ref, units


def oracle_refine_timed(x, spec, groups):
    """Wall time of the oracle's PIVOT-Refine over the given runs [(g0, g1)] of groups and the
    key-row products they cover."""
    from oracle import oracle as orc

    L, g, c = spec.L, spec.g, spec.c
    units = 0
    t0 = time.perf_counter()
    for g0, g1 in groups:
        orc.refine(x["q"], x["w"], x["k"], spec.k, c, g, g0=g0, g1=g1)
        for i in range(g0, g1):
            P = min(i * g + g, L)
            units += P + (P - i * g) * min(c, P)
    return time.perf_counter() - t0, units


def per_config_lines(to_dev_fn, dev, ws, flush, timed, tf_burst, hbm, cpu):
    """Every workload of the build: GPU times of its paths with queries/s, us per group, roofline
    fraction (scan [+ refine] FLOPs at the burst bf16 peak over the time) and x vs the dense
    indexer on the same inputs; the CPU oracle timed whole on the tiny and 8K workloads, and on a
    sample of groups, extrapolated to the whole sequence by key-row products, on the others."""
    import numpy as np

    import top_token_selection_proxy_b200 as P
    from top_token_selection_proxy_b200 import inputs
    from oracle import oracle as orc

    out = []

    def entry(spec, x, paths, cpu_mode):
        q, w, k = to_dev_fn(x["q"], dev), to_dev_fn(x["w"], dev), to_dev_fn(x["k"], dev)
        G = (spec.L + spec.g - 1) // spec.g
        f_scan, f_ref, units = prefill_work(spec)
        f_dense = 2 * spec.H * spec.d * spec.L * (spec.L + 1) // 2
        ms = {}
        if "dense" in paths:
            ms["dense"] = timed(lambda: P.indexer_dense(q, w, k, spec.k, ws=ws), n=2)
        if "reuse" in paths:
            ms["reuse"] = timed(lambda: P.reuse(q, w, k, spec.k, spec.g, ws=ws))
        if "refine" in paths:
            ms["refine"] = timed(lambda: P.refine(q, w, k, spec.k, spec.c, spec.g, ws=ws))
        flops = {"dense": f_dense, "reuse": f_scan, "refine": f_scan + f_ref}
        e = {"workload": spec.name, "L": spec.L, "g": spec.g, "k": spec.k, "c": spec.c, "rho": spec.rho,
             "dtype": "f32" if spec.dtype == inputs.F32 else "bf16"}
        for name, t in ms.items():
            e[name] = {"ms": t, "queries_per_s": spec.L / (t * 1e-3), "us_per_group": 1000.0 * t / G,
                       "roofline_frac": (flops[name] / (tf_burst * 1e12)) / (t * 1e-3)}
            if "dense" in ms and name != "dense":
                e[name]["x_vs_dense"] = ms["dense"] / t
        if cpu_mode == "whole" and cpu:
            secs, u = oracle_refine_timed(x, spec, [(0, G)])
            e["cpu_oracle_refine"] = {"seconds": secs, "queries_per_s": spec.L / secs, "cores": orc.threads(),
                                      "kind": "oracle, timed whole"}
        elif cpu_mode == "sample" and cpu:
            runs = [(int(i), int(i) + 1) for i in inputs.sample_groups(G, spec.g, spec.k, spec.c, 16,
                                                                       spec.seed + 2000)]
            secs, u = oracle_refine_timed(x, spec, runs)
            est = secs * units / u
            e["cpu_oracle_refine"] = {"sample_seconds": secs, "sample_groups": len(runs),
                                      "extrapolated_seconds": est, "queries_per_s": spec.L / est,
                                      "cores": orc.threads(),
                                      "kind": "oracle on 16 seeded groups, EXTRAPOLATED to the whole sequence "
                                              "by key-row products sum_i (P_i + |G_i| min(c, P_i))"}
        del q, w, k
        return e

    out.append(entry(inputs.TINY, inputs.make_prefill(inputs.TINY), ("dense", "reuse", "refine"), "whole"))
    out.append(entry(inputs.PREFILL_8K, inputs.make_prefill(inputs.PREFILL_8K), ("dense", "reuse", "refine"),
                     "whole"))
    for rho in inputs.SWEEP_RHO:
        x = inputs.make_prefill(inputs.sweep_32k(1, rho))  # one sequence per rho; the g axis sees the same inputs
        dense_ms = None
        for g in inputs.SWEEP_G:
            spec = inputs.sweep_32k(g, rho)
            e = entry(spec, x, ("dense", "reuse", "refine") if g == 1 else ("reuse", "refine"), "sample")
            if g == 1:
                dense_ms = e["dense"]["ms"]
            else:
                for name in ("reuse", "refine"):
                    e[name]["x_vs_dense"] = dense_ms / e[name]["ms"]
            out.append(e)
        del x
    ds = inputs.DECODE
    xd = inputs.make_decode(ds)
    dq, dw, dk = to_dev_fn(xd["q"], dev), to_dev_fn(xd["w"], dev), to_dev_fn(xd["k"], dev)
    off = xd["offsets"]
    key_bytes = int(off[-1]) * ds.d * 2
    offd = P.DeviceOffsets(off, dev)  # the batch's offsets stay on the device, like its keys
    d_ms = {"refine": timed(lambda: P.refine_varlen(dq, dw, dk, offd, ds.k, ds.c, ds.g, ws=ws)),
            "reuse": timed(lambda: P.reuse_varlen(dq, dw, dk, offd, ds.k, ds.g, ws=ws))}
    rows = ds.B * ds.g
    e = {"workload": ds.name, "B": ds.B, "g": ds.g, "k": ds.k, "c": ds.c, "key_bytes": key_bytes,
         **{n: {"ms": t, "queries_per_s": rows / (t * 1e-3), "us_per_group": 1000.0 * t / ds.B,
                "roofline_frac": (key_bytes / (hbm * 1e9)) / (t * 1e-3), "bound": "hbm"}
            for n, t in d_ms.items()}}
    if cpu:
        t0 = time.perf_counter()
        orc.decode(xd["q"], xd["w"], xd["k"], off, ds.k, ds.c, ds.g, 1)
        secs = time.perf_counter() - t0
        e["cpu_oracle_refine"] = {"seconds": secs, "queries_per_s": rows / secs, "cores": orc.threads(),
                                  "kind": "oracle, timed whole (all 32 sequences)"}
    out.append(e)
    del dq, dw, dk
    return out


def run_split(args):
    """One L=131072 sequence indexed by all ranks (PIVOT-Refine): each rank holds the rows of
    its zig-zag chunks, the key chunks are all-gathered (NCCL; the one exchange), then every
    rank runs the group-range call on its two chunks.  value = L / max-over-ranks step time."""
    import numpy as np
    import torch

    import top_token_selection_proxy_b200 as P
    from top_token_selection_proxy_b200 import build, inputs
    from top_token_selection_proxy_b200 import multigpu as M

    world, rank, local = M.env()
    M.init("nccl", world)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        build.build()
    M.barrier(world)
    P.lib()
    spec = inputs.LONG_128K
    x = inputs.make_prefill(spec)  # every rank draws the same sequence and keeps its chunks
    chunks = M.zigzag_chunks(spec.L, spec.g, world, rank)
    q_loc = to_dev(M.local_rows(x["q"], chunks), dev)
    w_loc = to_dev(M.local_rows(x["w"], chunks), dev)
    k_loc = to_dev(M.local_rows(x["k"], chunks), dev)
    del x
    ws = P.Workspace(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def index_fn(q_rows, w_rows, k_prefix, t0, t1):
        return P.refine_range(q_rows, w_rows, k_prefix, spec.L, spec.k, spec.c, spec.g, t0 // spec.g,
                              t1 // spec.g, ws=ws)[0]

    def step():
        return M.split_step(index_fn, q_loc, w_loc, k_loc, spec.L, spec.g, world, rank)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    M.barrier(world)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    tot = 0.0
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record()
        step()
        ev[i][1].record()
        torch.cuda.synchronize()
        tot += ev[i][0].elapsed_time(ev[i][1])
    M.barrier(world)
    ms = M.max_over_ranks(tot, world, dev) / args.steps
    status = M.max_over_ranks(float(P.last_device_status(ws)), world, dev)
    if rank == 0:
        print(json.dumps({"metric": METRIC, "value": spec.L / (ms / 1000.0), "unit": UNIT, "n_gpus": world,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                          "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                          "config": {"workload": spec.name + "_refine_split", "L": spec.L, "H_I": spec.H,
                                     "d": spec.d, "k": spec.k, "c": spec.c, "g": spec.g,
                                     "parallelism": f"one sequence over {world} GPU(s): zig-zag group ranges, "
                                                    "key all-gather",
                                     "l2": "flushed before every step (256 MiB write)"},
                          "gpu_launches": 3 * 2 * args.steps, "device_status": int(status)}), flush=True)
    M.finish(world)


def run_split_decode(args):
    """The MTP decode batch with every sequence's prefix split over the ranks (PIVOT-Refine): each
    rank holds one contiguous key shard per sequence; a step is the shard selections, one
    all-gather of them (NCCL), the merge, the re-scoring of the candidates each rank holds, one
    element-wise sum of the member scores (NCCL) and the member top-k.  value = the batch's
    queries / max-over-ranks step time."""
    import torch

    import top_token_selection_proxy_b200 as P
    from top_token_selection_proxy_b200 import build, inputs
    from top_token_selection_proxy_b200 import multigpu as M

    world, rank, local = M.env()
    M.init("nccl", world)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        build.build()
    M.barrier(world)
    P.lib()
    ds = inputs.DECODE
    x = inputs.make_decode(ds)  # every rank draws the same batch and keeps its shards' keys
    k_shard, shard_off, pos_base = M.shard_of(x["k"], x["offsets"], world, rank)
    q, w, ks = to_dev(x["q"], dev), to_dev(x["w"], dev), to_dev(k_shard, dev)
    fns = M.device_split_fns(P.OP_REFINE, q, w, ks, shard_off, pos_base, x["offsets"], ds.k, ds.c, ds.g)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        return M.decode_split_step(fns[0], fns[1], world, fns[2], fns[3])

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    M.barrier(world)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    tot = 0.0
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record()
        step()
        ev[i][1].record()
        torch.cuda.synchronize()
        tot += ev[i][0].elapsed_time(ev[i][1])
    M.barrier(world)
    ms = M.max_over_ranks(tot, world, dev) / args.steps
    if rank == 0:
        print(json.dumps({"metric": "decode queries/s, prefixes split over GPUs", "value": ds.B * ds.g / (ms / 1e3),
                          "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                          "ms_per_step": ms, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
                          "dtype": "bf16", "data": "synthetic",
                          "config": {"workload": ds.name + "_refine_prefix_split", "B": ds.B, "g": ds.g,
                                     "k": ds.k, "c": ds.c,
                                     "parallelism": f"every prefix over {world} GPU(s): key shards, all-gather of "
                                                    "the shard selections, sum of the member scores",
                                     "l2": "flushed before every step (256 MiB write)"},
                          "gpu_launches": 6 * args.steps}), flush=True)
    M.finish(world)


def run_reference(args):
    """Reference arm: the CPU oracle as it stands, on bounded samples of the workload."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    from top_token_selection_proxy_b200 import inputs
    from oracle import oracle as orc

    orc.build()
    spec = inputs.LONG_128K
    x = inputs.make_prefill(spec)
    cores = len(os.sched_getaffinity(0))
    orc.set_threads(cores)
    G = (spec.L + spec.g - 1) // spec.g
    per = max(1, cores)
    R = 4

    def step(j):
        g0 = min(G - per, int((2 * (j % R) + 1) * G / (2 * R)))
        orc.refine(x["q"], x["w"], x["k"], spec.k, spec.c, spec.g, g0=g0, g1=g0 + per)
        return per * spec.g

    for j in range(args.warmup):
        step(j)
    rows = 0
    t0 = time.perf_counter()
    for j in range(args.steps):
        rows += step(j)
    dt = time.perf_counter() - t0
    v = rows / dt
    out = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": spec.name + "_refine", "L": spec.L, "H_I": spec.H, "d": spec.d, "k": spec.k,
                   "c": spec.c, "g": spec.g},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": orc.threads(), "kind": "oracle",
                         "sample": f"each step: {per} consecutive groups ({per * spec.g} query rows) at one of "
                                   f"{R} evenly spaced positions of the L={spec.L} sequence"},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def run_profile_decode():
    """The decode batch for ncu launch lists: per variant a warm-up call, then the captured call."""
    import torch

    import top_token_selection_proxy_b200 as P
    from top_token_selection_proxy_b200 import build, inputs

    build.build()
    ds = inputs.DECODE
    x = inputs.make_decode(ds)
    dev = torch.device("cuda", 0)
    q, w, kc = to_dev(x["q"], dev), to_dev(x["w"], dev), to_dev(x["k"], dev)
    ws = P.Workspace(dev)
    for _ in range(2):
        P.refine_varlen(q, w, kc, x["offsets"], ds.k, ds.c, ds.g, ws=ws)
    for _ in range(2):
        P.reuse_varlen(q, w, kc, x["offsets"], ds.k, ds.g, ws=ws)
    torch.cuda.synchronize()
    st = P.last_device_status(ws)
    print(f"profile decode {ds.name}: status {P.STATUS.get(st, st)}")
    if st != 0:
        raise SystemExit(1)


def main():
    args = parse()
    if args.profile_case:
        run_profile_case(args.profile_case)
        return
    if args.profile_decode:
        run_profile_decode()
        return
    if args.impl == "reference":
        run_reference(args)
        return
    if args.split:
        run_split(args)
        return
    if args.split_decode:
        run_split_decode(args)
        return
    import numpy as np
    import torch

    import top_token_selection_proxy_b200 as P
    from top_token_selection_proxy_b200 import build, inputs
    from top_token_selection_proxy_b200 import multigpu as M

    world, rank, local = M.env()
    M.init("nccl", world)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        build.build()
    M.barrier(world)
    P.lib()

    spec = inputs.LONG_128K
    # each rank indexes its own sequence (independent problems)
    spec_r = dataclasses.replace(spec, seed=M.rank_seed(spec.seed, rank))
    x = inputs.make_prefill(spec_r)
    q, w, k = to_dev(x["q"], dev), to_dev(x["w"], dev), to_dev(x["k"], dev)
    ws = P.Workspace(dev)
    out_idx = torch.empty((spec.L, spec.k), dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    timer = P.KernelTimer()

    def step():
        P.refine(q, w, k, spec.k, spec.c, spec.g, out=out_idx, ws=ws)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    # every rank takes the same decision (a rank that left alone would strand the others at a barrier)
    if M.max_over_ranks(1.0 if P.last_device_status(ws) != 0 else 0.0, world, dev) > 0:
        M.finish(world)
        raise SystemExit("device status not OK after warm-up")

    clocks = Clocks(local)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    k_scan, k_ref, k_sel = [], [], []
    M.barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)  # write 256 MiB > L2 so each step starts cold
        starts[i].record()
        with timer:
            step()
        ends[i].record()
        torch.cuda.synchronize()
        a, b, c = timer.ms()
        k_scan.append(a)
        k_ref.append(b)
        k_sel.append(c)
    torch.cuda.synchronize()
    M.barrier(world)
    clk = clocks.stop()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms, value = M.weak_scaling(sum(step_ms), args.steps, spec.L, world, dev)
    status = P.last_device_status(ws)

    extras = {}
    if not args.no_extras and rank == 0:
        def timed(f, n=3):
            f()
            torch.cuda.synchronize()
            ts = []
            for _ in range(n):
                flush.fill_(1)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                f()
                e1.record()
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1))
            return statistics.median(ts)

        agg_ms = {a_: timed(lambda a_=a_: P.refine(q, w, k, spec.k, spec.c, spec.g, out=out_idx, ws=ws,
                                                    aggregation=a_)) for a_ in ("first", "last")}
        extras["aggregation_refine_ms"] = agg_ms
        dense_ms = timed(lambda: P.indexer_dense(q, w, k, spec.k, out=out_idx, ws=ws), n=2)
        reuse_ms = timed(lambda: P.reuse(q, w, k, spec.k, spec.g, out=out_idx, ws=ws))
        extras.update(dense_ms=dense_ms, reuse_ms=reuse_ms, x_vs_dense=dense_ms / ms, reuse_x_vs_dense=dense_ms / reuse_ms)
        ds = inputs.DECODE
        xd = inputs.make_decode(ds)
        dq, dw, dk = to_dev(xd["q"], dev), to_dev(xd["w"], dev), to_dev(xd["k"], dev)
        off = xd["offsets"]
        offd = P.DeviceOffsets(off, dev)  # the batch's offsets stay on the device, like its keys
        dref = timed(lambda: P.refine_varlen(dq, dw, dk, offd, ds.k, ds.c, ds.g, ws=ws))
        dreu = timed(lambda: P.reuse_varlen(dq, dw, dk, offd, ds.k, ds.g, ws=ws))

        def decode_phases(f, n=3):
            """Median (proxies + scan, selection + emit, re-scoring + row select) of n calls."""
            ph = []
            for _ in range(n):
                flush.fill_(1)
                with timer:
                    f()
                torch.cuda.synchronize()
                ph.append(timer.ms())
            return {name: statistics.median(x[i] for x in ph)
                    for i, name in enumerate(("scan", "select_emit", "refine_rowselect"))}

        dph = decode_phases(lambda: P.refine_varlen(dq, dw, dk, offd, ds.k, ds.c, ds.g, ws=ws))
        key_bytes = int(off[-1]) * ds.d * 2
        hbm, _, _, _ = peaks()
        extras["decode"] = {"workload": ds.name, "refine_ms": dref, "reuse_ms": dreu, "refine_kernels_ms": dph,
                            "key_bytes": key_bytes, "refine_hbm_frac": key_bytes / (dref * 1e-3) / (hbm * 1e9)}
        del dq, dw, dk
        # guardrail: the guarded Refine call against both of its paths on short prefills
        guard = []
        for gs in (inputs.PREFILL_8K, dataclasses.replace(inputs.PREFILL_8K, name="prefill_L3072_g8", L=3072)):
            xg = inputs.make_prefill(gs)
            gq, gw, gk = to_dev(xg["q"], dev), to_dev(xg["w"], dev), to_dev(xg["k"], dev)
            g_ref = timed(lambda: P.refine(gq, gw, gk, gs.k, gs.c, gs.g, ws=ws))
            g_den = timed(lambda: P.indexer_dense(gq, gw, gk, gs.k, ws=ws))
            g_grd = timed(lambda: P.refine_guarded(gq, gw, gk, gs.k, gs.c, gs.g, ws=ws))
            guard.append({"workload": gs.name, "path": "dense" if P.guardrail_dense(P.OP_REFINE, gs.L, gs.c, gs.g)
                          else "refine", "guarded_ms": g_grd, "refine_ms": g_ref, "dense_ms": g_den})
            del gq, gw, gk
        extras["guardrail"] = guard
        # the pages' observations O1-O3 on the seeded 8K workload, from the dense indexer's rows
        from top_token_selection_proxy_b200 import diagnostics

        xg = inputs.make_prefill(inputs.PREFILL_8K)
        gq, gw, gk = to_dev(xg["q"], dev), to_dev(xg["w"], dev), to_dev(xg["k"], dev)
        Lg, kg = inputs.PREFILL_8K.L, inputs.PREFILL_8K.k
        di, _ = P.indexer_dense(gq, gw, gk, kg, ws=ws)
        _, dfull = P.indexer_dense(gq, gw, gk, Lg, scores=True, ws=ws)  # every prefix score
        extras["workload_diagnostics"] = {"workload": inputs.PREFILL_8K.name,
                                          **diagnostics.summary(di.cpu().numpy(), kg, dfull.cpu().numpy())}
        del gq, gw, gk, di, dfull
        if not args.no_configs:
            hbm_, tfb_, _, _ = peaks()
            extras["configs"] = per_config_lines(to_dev, dev, ws, flush, timed, tfb_, hbm_, not args.no_cpu)

    e2e = None
    M.barrier(world)  # every rank measures end to end (rank 0 arrives after its side measurements)
    if not args.no_e2e:
        qh = torch.from_numpy(x["q"].view(np.int16)).pin_memory()
        wh = torch.from_numpy(x["w"]).pin_memory()
        kh = torch.from_numpy(x["k"].view(np.int16)).pin_memory()
        oh = torch.empty((spec.L, spec.k), dtype=torch.int32).pin_memory()

        def e2e_step():  # the public host-memory call: copies in, kernels and copies out overlap by chunks
            P.refine_host(qh.view(torch.bfloat16), wh, kh.view(torch.bfloat16), spec.k, spec.c, spec.g,
                              out_host=oh, chunks=E2E_CHUNKS, ws=ws, device=dev)

        e2e_step()
        torch.cuda.synchronize()
        n = max(3, min(args.steps, 5))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            e2e_step()
        e1.record()
        torch.cuda.synchronize()
        e_ms = M.max_over_ranks(e0.elapsed_time(e1) / n, world, dev)
        e2e = {"value": world * spec.L / (e_ms / 1000.0), "unit": UNIT, "ms_per_step": e_ms,
               "h2d_bytes_per_step": int(qh.numel() * 2 + wh.numel() * 4 + kh.numel() * 2),
               "d2h_bytes_per_step": int(oh.numel() * 4), "host_buffers": "pinned",
               "api": f"C ABI pivot_refine_host, {E2E_CHUNKS} runs of whole groups, copies overlapped with the kernels"}

    if rank != 0:
        M.finish(world)
        return

    hbm, tf_burst, tf_sust, src = peaks()
    f_scan, f_ref, f_dense, b_alg = workload_flops_bytes(spec)
    scan_ms = statistics.median(k_scan)
    achieved = f_scan / (scan_ms * 1e-3) / 1e12
    t_roof_lit = max(f_scan / (tf_burst * 1e12), b_alg / (hbm * 1e9)) * 1e3
    t_roof_alg = max((f_scan + f_ref) / (tf_burst * 1e12), b_alg / (hbm * 1e9)) * 1e3
    G = (spec.L + spec.g - 1) // spec.g
    cpu = None
    if not args.no_cpu:
        v, cores, desc, secs, u_s = cpu_oracle_sample(x, spec)
        full = secs * refine_units(spec, 0, G) / u_s
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc, "seconds": secs,
               "extrapolated_full_sequence_seconds": full,
               "extrapolated_queries_per_s": spec.L / full,
               "extrapolation": "EXTRAPOLATED from the sample by key-row products sum_i (P_i + |G_i| min(c, P_i))"}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": spec.name + "_refine", "L": spec.L, "H_I": spec.H, "d": spec.d, "k": spec.k,
                   "c": spec.c, "g": spec.g, "inputs": "q/k bf16, w fp32, resident in HBM",
                   "l2": "flushed before every step (256 MiB write)",
                   "parallelism": "independent sequence per GPU" if world > 1 else "single GPU"},
        "us_per_group": 1000.0 * ms / G,
        "kernels_ms": {"scan": scan_ms, "refine": statistics.median(k_ref), "rowselect": statistics.median(k_sel)},
        "roofline": {"bound": "tensor", "kernel": "scan (proxy pooling + tcgen05 proxy scan + streaming select)",
                     "achieved": achieved, "peak": tf_burst, "unit": "TFLOP/s", "frac": achieved / tf_burst,
                     "peak_kind": f"{src} bf16 dense, burst", "frac_of_sustained": achieved / tf_sust,
                     "flops_per_launch": f_scan, "traffic": scan_traffic(),
                     "traffic_source": SCAN_TRAFFIC["profile"]},
        "roofline_path": {"t_roof_ms_scan_only": t_roof_lit, "frac_scan_only": t_roof_lit / ms,
                          "t_roof_ms_scan_plus_refine": t_roof_alg, "frac_scan_plus_refine": t_roof_alg / ms,
                          "peak": f"{src} burst bf16 {tf_burst} TFLOP/s, HBM {hbm} GB/s",
                          "flops_scan": f_scan, "flops_refine": f_ref, "flops_dense": f_dense, "bytes_alg": b_alg},
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 3 * args.steps, "clocks": clk,
        "device_status": P.STATUS.get(status, status),
    }
    line.update(extras)
    print(json.dumps(line), flush=True)
    M.finish(world)


if __name__ == "__main__":
    main()
