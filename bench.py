#!/usr/bin/env python
"""Benchmark of the on-device MoE dispatch/combine path on B200.

One step = one pass of the whole path over one batch of synthetic tokens:
route_topk -> demand_hist -> replica_assign -> build_layout -> pack ->
combine (identity experts: the packed rows are the expert outputs), all in
libmoe.so's kernels on one stream.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config c4] [--impl ours|reference]

Prints one JSON line (rank 0).  ``value`` is dispatched token-rows per second
over the whole job (all ranks' rows / the slowest rank's device time), with
inputs resident in HBM; ``e2e`` is the same metric through the public API
with pinned host buffers and the host<->device copies inside the timed region.
With N > 1 (torchrun, one process per GPU) every rank runs an independent
replica on its own seeded batch: the path has no exchange between GPUs, so
there is no collective on the data path ("scaling": "weak").

``--impl reference`` times the CPU oracle instead, on the host cores, on a
bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "dispatch+combine token-rows/s and achieved HBM GB/s vs peak on 1 B200"
PEAK_FALLBACK_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
KERNEL_SOURCES = {  # kernel -> source file whose hash the ncu traffic figure is tied to
    "pack": "combine_router_softmax_02_b200/csrc/pack.cu",
    "combine": "combine_router_softmax_02_b200/csrc/combine.cu",
}


# ------------------------------------------------------------------ helpers
def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return PEAK_FALLBACK_GBS, "fallback"


def src_hash(rel: str) -> str:
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel on
    this workload, or None when there is none or the kernel changed since."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    h = re.search(r"source_sha256_16:\s*([0-9a-f]{16})", text)
    t = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", text)
    if not h or not t or h.group(1) != src_hash(KERNEL_SOURCES[kernel]):
        return None
    return int(t.group(1))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the GPU works."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.dev), "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ---------------------------------------------------------- byte accounting
def step_bytes(cfg: W.Config, rows: int, rows_hop1: int, S: int) -> dict:
    """Algorithmic HBM bytes of each call of one step (each array read or
    written once at its minimum size)."""
    T, E, k, R, H, b = cfg.T, cfg.E, cfg.k, cfg.R, cfg.H, cfg.elem_bytes
    d = {
        "route_topk": T * E * 4 + T * k * 8,
        "demand_hist": T * k * 4 + E * 4,
        "replica_assign": E * 4 * 4 + S * 8 + R * 4,
        "build_layout": T * k * 4 + (T * k * 8 + E * 4) + rows * 8 + T * k * 4 + R * R * 4,
    }
    if cfg.mode == W.TWO_HOP:
        d["build_layout"] += rows_hop1 * (4 + k * 4) + T * k * 4 + rows * 4
        # one read of each token, both hops' rows written
        d["pack"] = (T + rows_hop1 + rows) * H * b + 2 * T * k * 4
        # rank rows read once; group partials and tokens written
        d["combine"] = (rows + rows_hop1 + T) * H * b + rows * 8 + T * k * 4
    else:
        d["pack"] = (T + rows) * H * b + T * k * 4
        d["combine"] = (rows + T) * H * b + rows * 4 + T * k * 4
    # the fused front end reads the picks once less (no separate count pass)
    d["route_layout"] = d["route_topk"] + d["build_layout"] - T * k * 4
    return d


def make_trace(cfg: W.Config, counts, expert_slot, expert_rank, rank_active, rank_offsets,
               send_counts, group_offsets=None, calls=None) -> dict:
    """One step's routing decisions and buffer sizes, from host arrays: the
    replica chosen for every active expert, each rank's group, activated experts
    and received rows, and the two all-to-all-v exchanges the layout stands for
    (bytes per source -> destination rank), plus per-call start and duration
    (us) when `calls` gives [(name, start_us, dur_us)]."""
    b = cfg.H * cfg.elem_bytes
    rpg = max(cfg.ranks_per_group, 1)
    counts, expert_slot, expert_rank = (np.asarray(a) for a in (counts, expert_slot, expert_rank))
    rows = np.diff(np.asarray(rank_offsets))
    S = np.asarray(send_counts).reshape(cfg.R, cfg.R)
    tr = {
        "workload": cfg.name,
        "ranks": cfg.R,
        "replicas": [{"expert": int(e), "demand": int(counts[e]), "slot": int(expert_slot[e]),
                      "rank": int(expert_rank[e])} for e in np.flatnonzero(counts > 0)],
        "rank_detail": [{"rank": r, "group": r // rpg if cfg.mode == W.TWO_HOP else 0,
                         "active_experts": int(rank_active[r]), "rows": int(rows[r]),
                         "recv_bytes": int(rows[r]) * b} for r in range(cfg.R)],
        "collectives": [
            {"name": "dispatch all-to-all-v (pack: token rows to their destination ranks)",
             "bytes": int(S.sum()) * b, "bytes_src_dst": (S * b).tolist()},
            {"name": "combine all-to-all-v (expert outputs back to the token's rank)",
             "bytes": int(S.sum()) * b, "bytes_src_dst": (S.T * b).tolist()},
        ],
    }
    if cfg.mode == W.TWO_HOP and group_offsets is not None:
        g_rows = np.diff(np.asarray(group_offsets))
        tr["collectives"].insert(0, {"name": "dispatch hop 1 (token rows to their groups)",
                                     "bytes": int(g_rows.sum()) * b,
                                     "group_bytes": [int(x) * b for x in g_rows]})
    if calls is not None:
        tr["calls_us"] = [{"call": n, "start": round(t, 3), "duration": round(d, 3)} for n, t, d in calls]
    return tr


# ------------------------------------------------------------------- ours
def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import combine_router_softmax_02_b200 as moe

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    cfg = config_of(args)
    seed = args.seed + rank
    logits_h = torch.from_numpy(W.make_logits(cfg, seed)).pin_memory()
    x_h = W.make_activations(cfg, seed).pin_memory()
    rm = W.make_replica_map(cfg, seed)
    tdt = x_h.dtype
    dc = moe.DispatchCombine(cfg.T, cfg.H, cfg.E, cfg.k, cfg.R, torch.from_numpy(rm.replica_offsets),
                             torch.from_numpy(rm.replica_slots), torch.from_numpy(rm.slot_rank),
                             cfg.mode, cfg.tokens_per_rank, max(cfg.ranks_per_group, 1),
                             cfg.n_groups, cfg.groups_per_token, dtype=tdt, device=dev)
    logits = logits_h.to(dev)
    x = x_h.to(dev)
    stream = torch.cuda.current_stream(dev)
    names = ["route_topk", "demand_hist", "replica_assign", "build_layout", "pack", "combine"]
    single = bool(np.all(np.diff(rm.replica_offsets) == 1))
    if args.fused:
        names = ["route_layout", "pack", "combine"]
        if single:
            static_rank = torch.from_numpy(rm.slot_rank[rm.replica_slots]).to(dev, torch.int32)

    def one_step(ev=None):
        marks = iter(ev) if ev is not None else None

        def mark():
            if marks is not None:
                next(marks).record(stream)

        mark()
        if args.fused and single:
            dc.route_single_replica(logits, static_rank)
            mark()
        elif args.fused:
            dc.route_one_launch(logits)
            mark()
        else:
            moe.route_topk(logits, cfg.k, cfg.n_groups, cfg.groups_per_token, False, dc.topk_idx, dc.topk_w)
            mark()
            moe.demand_hist(dc.topk_idx, cfg.E, dc.counts)
            mark()
            moe.replica_assign(dc.counts, dc.replica_offsets, dc.replica_slots, dc.slot_rank, cfg.R,
                               dc.expert_slot, dc.expert_rank, dc.rank_active)
            mark()
            moe.build_layout(dc.topk_idx, dc.topk_w, dc.expert_rank, dc.layout)
            mark()
        moe.pack(x, dc.layout, dc.packed, dc.packed_hop1)
        mark()
        dc.combine()
        mark()

    def barrier():
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]))
    sampler.start()
    for _ in range(args.warmup):
        one_step()
    st = moe.get_status()
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {moe.status_string(st)}")
    rows = int(dc.layout.num_rows.item())
    rows1 = int(dc.layout.num_rows_hop1.item()) if cfg.mode == W.TWO_HOP else 0

    # device-resident timed region: CUDA events on the launching stream
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    barrier()
    launches0 = moe.kernel_launches()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        one_step(evs[i])
    t_end.record(stream)
    barrier()
    launches = moe.kernel_launches() - launches0
    clocks = sampler.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    per = {n: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs) for j, n in enumerate(names)}
    st = moe.get_status()
    if st != 0:
        raise RuntimeError(f"device status after timing: {moe.status_string(st)}")
    eager_ms = elapsed_ms
    if args.graph:
        # the same step captured once in a CUDA graph and replayed: no host
        # launch latency between the kernels (the decode workloads' regime)
        g = torch.cuda.CUDAGraph()
        n0 = moe.kernel_launches()
        with torch.cuda.graph(g):
            one_step()
        kernels_per_step = moe.kernel_launches() - n0
        for _ in range(args.warmup):
            g.replay()
        barrier()
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(args.steps):
            g.replay()
        g1.record(stream)
        barrier()
        elapsed_ms = g0.elapsed_time(g1)
        launches = kernels_per_step * args.steps
        st = moe.get_status()
        if st != 0:
            raise RuntimeError(f"device status after graph replays: {moe.status_string(st)}")
        del g

    # end to end through the public API: pinned host inputs in, result out,
    # every step (HostPipeline overlaps the copies with the kernels)
    out_h = torch.empty((cfg.T, cfg.H), dtype=tdt).pin_memory()
    pipe = moe.HostPipeline(dc, chunks=args.e2e_chunks)
    for _ in range(max(1, min(args.warmup, 2))):
        pipe.step(logits_h, x_h, out_h)
    pipe.join(stream)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_steps = max(1, min(args.steps, 10))
    e0.record(stream)
    pipe.wait(e0)
    for _ in range(e2e_steps):
        pipe.step(logits_h, x_h, out_h)
    pipe.join(stream)
    e1.record(stream)
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    st = moe.get_status()
    if st != 0:
        raise RuntimeError(f"device status after e2e: {moe.status_string(st)}")

    # workload statistics of the last pass (device kernels, outside the timed regions)
    stats = moe.dispatch_stats(dc.counts, dc.layout.send_counts).cpu().tolist()
    _, tb_active = moe.token_balanced_assign(dc.counts, dc.replica_offsets, dc.replica_slots,
                                             dc.slot_rank, cfg.R)
    workload_stats = dict(zip(moe.STAT_NAMES, stats))
    workload_stats.update(
        max_active_metro=int(dc.rank_active.max().item()),
        max_active_token_balanced=int(tb_active.max().item()),
        active_experts=int((dc.counts > 0).sum().item()))
    st = moe.get_status()
    if st != 0:
        raise RuntimeError(f"device status after statistics: {moe.status_string(st)}")
    if args.trace:
        last = evs[-1]
        calls = [(n, last[0].elapsed_time(last[j]) * 1e3, last[j].elapsed_time(last[j + 1]) * 1e3)
                 for j, n in enumerate(names)]
        L = dc.layout
        if args.fused and single:  # the single-replica kernel takes the ranks as given
            e_slot = rm.replica_slots[rm.replica_offsets[:-1]]
            e_rank = rm.slot_rank[e_slot]
        else:
            e_slot, e_rank = dc.expert_slot.cpu().numpy(), dc.expert_rank.cpu().numpy()
        tr = make_trace(cfg, dc.counts.cpu().numpy(), e_slot, e_rank, dc.rank_active.cpu().numpy(),
                        L.rank_offsets.cpu().numpy(), L.send_counts.cpu().numpy(),
                        L.group_offsets.cpu().numpy() if cfg.mode == W.TWO_HOP else None, calls)
        path = args.trace if world == 1 else f"{args.trace}.rank{rank}"
        with open(path, "w") as f:
            json.dump(tr, f)

    # whole-job aggregation: max time over ranks, rows summed over ranks
    agg = aggregate(dist, dev, [elapsed_ms, e2e_ms], [rows * args.steps, rows * e2e_steps])
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return None
    (elapsed_max, e2e_max), (rows_all, rows_e2e_all) = agg
    peak, peak_kind = measured_peak()
    bytes_ = step_bytes(cfg, rows, rows1, rm.S)
    step_total = sum(bytes_[n] for n in names)
    ms_step = elapsed_max / args.steps
    dom = max(("pack", "combine"), key=lambda n: per[n])
    achieved = bytes_[dom] / (per[dom] * 1e-3) / 1e9
    traffic = ncu_traffic(dom, cfg.name)
    workload = f"{cfg.name}: {cfg.desc}" + (" (two-hop)" if cfg.mode == W.TWO_HOP else
                                           (" (dedup)" if cfg.mode == W.DEDUP else " (per-pick)"))
    line = {
        "metric": METRIC,
        "value": rows_all / (elapsed_max * 1e-3),
        "unit": "token-rows/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg.dtype,
        "data": "synthetic, seeded (rank seed = base + rank); mock-token routing, which the DODOCO "
                "study finds overstates imbalance relative to real text",
        "config": {
            "workload": workload, "tokens": cfg.T, "hidden": cfg.H, "experts": cfg.E, "top_k": cfg.k,
            "ranks": cfg.R, "rows_per_step": rows, "rows_hop1_per_step": rows1 or None,
            "layout": {0: "per_pick", 1: "dedup", 2: "two_hop"}[cfg.mode],
            "l2": "inputs larger than L2 (activations %.2f GB, packed rows %.2f GB per step; L2 126 MB)"
                  % (cfg.T * cfg.H * cfg.elem_bytes / 1e9, rows * cfg.H * cfg.elem_bytes / 1e9),
            "parallelism": f"independent replica per GPU x{world}",
            "launch": "cuda_graph" if args.graph else "eager",
            "front_end": ("separate calls" if not args.fused else
                          "one launch: route+layout, single-replica" if single else
                          "one launch: route+histogram+METRO assignment+layout"),
        },
        "eager_ms_per_step": eager_ms / args.steps,
        "hbm_GBps": step_total / (ms_step * 1e-3) / 1e9,
        "hbm_frac_of_measured": step_total / (ms_step * 1e-3) / 1e9 / peak,
        "hbm_frac_of_8TBps": step_total / (ms_step * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
        "kernels_us": {n: per[n] * 1e3 for n in names},
        "kernels_GBps": {n: bytes_[n] / (per[n] * 1e-3) / 1e9 for n in names},
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                     "algorithmic_bytes": bytes_[dom],
                     "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"},
        "e2e": {"value": rows_e2e_all / (e2e_max * 1e-3), "unit": "token-rows/s",
                "h2d_bytes_per_step": int(logits_h.numel() * 4 + x_h.numel() * x_h.element_size()),
                "d2h_bytes_per_step": int(out_h.numel() * out_h.element_size()),
                "steps": e2e_steps, "ms_per_step": e2e_max / e2e_steps,
                "pipeline": f"HostPipeline: 3 streams, {len(pipe.ranges)} token ranges per step, "
                            "double-buffered device inputs/outputs"},
        "gpu_launches": int(launches),
        "clocks": clocks,
        "workload_stats": workload_stats,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, args)
    return line


def aggregate(dist, dev, times_ms, rows):
    """Max of each time over ranks and sum of each row count over ranks."""
    if dist is None:
        return list(times_ms), list(rows)
    import torch
    t = torch.tensor(times_ms, dtype=torch.float64, device=dev)
    r = torch.tensor(rows, dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(r, op=dist.ReduceOp.SUM)
    return t.tolist(), r.tolist()


# --------------------------------------------------------------- the oracle
def oracle_step(cfg: W.Config, logits, x32, rm):
    """One pass of the CPU oracle over a sample; returns the rows processed."""
    import oracle
    idx, w = oracle.route_topk(logits, cfg.k, cfg.n_groups, cfg.groups_per_token)
    counts = oracle.demand_hist(idx, cfg.E)
    _, er, _ = oracle.replica_assign(counts, rm.replica_offsets, rm.replica_slots, rm.slot_rank, cfg.R)
    tpr = -(-logits.shape[0] // cfg.R)
    L = oracle.build_layout(idx, w, er, tpr, cfg.R, cfg.mode, max(cfg.ranks_per_group, 1))
    if cfg.mode == W.TWO_HOP:
        p1 = oracle.pack(x32, L["hop1_row_token"])
        p2 = oracle.pack(p1, L["hop2_src_row"])            # hop-2 row reads its hop-1 row
        oracle.combine_two_hop(p2, L, L["row_coef"], cfg.dtype)
    else:
        p = oracle.pack(x32, L["row_token"])
        oracle.combine(p, L["token_rows"], L["row_coef"])
    return int(L["num_rows"])


def oracle_sample(cfg: W.Config, tokens: int, seed: int):
    sub = cfg.with_(T=tokens)
    logits = W.make_logits(sub, seed)
    x32 = W.make_activations(sub, seed).float().numpy()
    return sub, logits, x32, W.make_replica_map(cfg, seed)


def cpu_baseline(cfg: W.Config, args):
    tokens = min(cfg.T, args.cpu_sample_tokens)
    sub, logits, x32, rm = oracle_sample(cfg, tokens, args.seed)
    t0 = time.perf_counter()
    rows = oracle_step(sub, logits, x32, rm)
    dt = time.perf_counter() - t0
    return {"value": rows / dt, "unit": "token-rows/s", "cores": 1, "kind": "oracle",
            "sample": f"first {tokens} of {cfg.T} tokens of the same workload, one full pass of the "
                      f"float64 numpy oracle ({rows} rows, {dt:.2f} s), single thread",
            "host_cpus": os.cpu_count()}


def config_of(args) -> W.Config:
    cfg = W.CONFIGS[args.config]
    if args.tokens:
        cfg = cfg.with_(T=args.tokens, name=f"{cfg.name}_T{args.tokens}")
    return cfg


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return None
    cfg = config_of(args)
    tokens = min(cfg.T, args.ref_sample_tokens)
    sub, logits, x32, rm = oracle_sample(cfg, tokens, args.seed)
    for _ in range(args.warmup):
        oracle_step(sub, logits, x32, rm)
    t0 = time.perf_counter()
    rows = 0
    for _ in range(args.steps):
        rows += oracle_step(sub, logits, x32, rm)
    dt = time.perf_counter() - t0
    value = rows / dt
    sample = (f"each step: the first {tokens} of {cfg.T} tokens of the same workload through the "
              f"float64 numpy oracle, single thread")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "token-rows/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / max(args.steps, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic, seeded",
        "config": {"workload": f"{cfg.name}: {cfg.desc}", "tokens": cfg.T, "hidden": cfg.H,
                   "experts": cfg.E, "top_k": cfg.k, "ranks": cfg.R,
                   "parallelism": "CPU oracle on rank 0"},
        "cpu_baseline": {"value": value, "unit": "token-rows/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "token-rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="c4", choices=sorted(W.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--tokens", type=int, default=0,
                    help="run the workload with this many tokens instead (profiling captures)")
    ap.add_argument("--cpu-sample-tokens", type=int, default=8192)
    ap.add_argument("--ref-sample-tokens", type=int, default=1024)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=8,
                    help="token ranges per step in the end-to-end pipeline (copies overlap the kernels)")
    ap.add_argument("--fused", action="store_true",
                    help="route, histogram, assignment and layout in one launch "
                         "(the single-replica kernel when every expert has one replica)")
    ap.add_argument("--trace", default="",
                    help="write the last timed step's routing decisions, buffer sizes and call "
                         "times as JSON to this path (outside the timed region)")
    ap.add_argument("--graph", action="store_true",
                    help="time replays of the step captured in a CUDA graph")
    args = ap.parse_args(argv)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and not (world == 1 and args.gpus == 1):
        if world == 1 and args.impl == "ours":
            raise SystemExit(f"--gpus {args.gpus} needs torchrun with {args.gpus} processes")
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        line = run_ours(args, rank, world, local_rank)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
