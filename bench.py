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
import math
import os
import re
import statistics
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


_SAMPLER = r"""
import sys, time, pynvml
pynvml.nvmlInit()
uuid, period = sys.argv[1], float(sys.argv[2])
try:
    h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
except pynvml.NVMLError:
    h = pynvml.nvmlDeviceGetHandleByIndex(int(sys.argv[3]))
print("max", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM), flush=True)
while True:
    t = time.perf_counter()
    print(t, pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
          pynvml.nvmlDeviceGetCurrentClocksEventReasons(h), pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0,
          flush=True)
    time.sleep(period)
"""


class ClockRecord:
    """A clock record to fill in once the sampler has stopped: the host-time
    windows of one timed region (or several)."""

    def __init__(self, regions):
        self.regions = regions


def fill_clock_records(obj, sampler):
    """Replaces every ClockRecord in a nested dict/list by its statistics."""
    if isinstance(obj, ClockRecord):
        return sampler.stats(obj.regions)
    if isinstance(obj, dict):
        return {k: fill_clock_records(v, sampler) for k, v in obj.items()}
    if isinstance(obj, list):
        return [fill_clock_records(v, sampler) for v in obj]
    return obj


class ClockSampler:
    """SM clock, power and clock-event reasons of the GPU, read through NVML
    every 10 ms by a separate process (reading only; no setting is touched),
    so that sampling takes no time from the process that launches the
    kernels.  Samples carry time.perf_counter() stamps (CLOCK_MONOTONIC, the
    same clock in both processes); ``stats(regions)`` summarises the samples
    taken inside the given host-time windows, so each timed region gets its
    own record."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, dev, period_s: float = 0.01):
        self.dev, self.period = dev, period_s
        self.proc = None
        self.samples = None        # (host time, sm MHz, reasons bitmask, power W), filled by stop()
        self.sm_max = None
        self.error = None

    def start(self):
        import torch
        uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        index = self.dev.index if self.dev.index is not None else 0
        if "CUDA_VISIBLE_DEVICES" in os.environ:
            vis = os.environ["CUDA_VISIBLE_DEVICES"].split(",")
            index = int(vis[index]) if index < len(vis) and vis[index].strip().isdigit() else index
        import subprocess
        try:
            self.proc = subprocess.Popen([sys.executable, "-c", _SAMPLER, uuid, str(self.period), str(index)],
                                         stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
        except Exception as e:  # no sampler: the record says so
            self.error = f"clock sampler unavailable: {e}"
        time.sleep(0.5)  # the sampler is running before the first timed region

    def stop(self):
        if self.samples is not None:
            return
        self.samples = []
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, err = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out, err = self.proc.communicate()
        for line in out.splitlines():
            parts = line.split()
            try:
                if parts[0] == "max":
                    self.sm_max = float(parts[1])
                else:
                    self.samples.append((float(parts[0]), float(parts[1]), int(parts[2]), float(parts[3])))
            except (ValueError, IndexError):
                continue
        if not self.samples and self.error is None:
            self.error = "NVML sampler gave no samples: " + " ".join(err.split())[:200]

    def stats(self, regions):
        self.stop()
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.sm_max, "reasons": [self.error or "no samples"],
                    "samples": 0}
        sel = [x for x in self.samples if any(a <= x[0] <= b for a, b in regions)]
        reasons = sorted({n for x in sel for n, bit in self.REASONS if x[2] & bit})
        sm = [x[1] for x in sel]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_mhz_min": min(sm) if sm else None,
                "sm_max_mhz": self.sm_max, "reasons": reasons, "samples": len(sel),
                "power_w_max": max(x[3] for x in sel) if sel else None,
                "seconds": round(sum(b - a for a, b in regions), 3), "source": "NVML, 10 ms, sampler process"}


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
# Workloads measured beside the headline in the default run (label, config,
# config overrides, one-launch front end, CUDA graph, end-to-end leg).
EXTRA_RUNS = (
    ("c5 two-hop", "c5", {}, False, False, True),
    ("c3 training, correlated placement", "c3", {}, False, False, False),
    ("c3 training, round-robin placement", "c3", {"placement": "roundrobin"}, False, False, False),
    ("c3 training, correlated placement, one-launch front end", "c3", {}, True, False, False),
    ("c1 METRO toy decode", "c1", {}, False, False, False),
    ("c1 METRO toy decode, one-launch front end, CUDA graph", "c1", {}, True, True, False),
    ("c2 MoE decode", "c2", {}, False, False, False),
    ("c2 MoE decode, one-launch front end, CUDA graph", "c2", {}, True, True, False),
)


class Workload:
    """One seeded workload resident on the device, with the buffers of one pass."""

    def __init__(self, moe, cfg: W.Config, seed: int, dev, fused: bool):
        import torch
        self.moe, self.cfg, self.dev = moe, cfg, dev
        self.logits_h = torch.from_numpy(W.make_logits(cfg, seed)).pin_memory()
        self.x_h = W.make_activations(cfg, seed).pin_memory()
        self.rm = rm = W.make_replica_map(cfg, seed)
        self.dc = moe.DispatchCombine(cfg.T, cfg.H, cfg.E, cfg.k, cfg.R, torch.from_numpy(rm.replica_offsets),
                                      torch.from_numpy(rm.replica_slots), torch.from_numpy(rm.slot_rank),
                                      cfg.mode, cfg.tokens_per_rank, max(cfg.ranks_per_group, 1),
                                      cfg.n_groups, cfg.groups_per_token, dtype=self.x_h.dtype, device=dev)
        self.logits = self.logits_h.to(dev)
        self.x = self.x_h.to(dev)
        self.single = bool(np.all(np.diff(rm.replica_offsets) == 1))
        self.fused = fused
        self.names = ["route_topk", "demand_hist", "replica_assign", "build_layout", "pack", "combine"]
        if fused:
            self.names = ["route_layout", "pack", "combine"]
            if self.single:
                self.static_rank = torch.from_numpy(rm.slot_rank[rm.replica_slots]).to(dev, torch.int32)

    def front_end(self) -> str:
        if not self.fused:
            return "separate calls"
        return ("one launch: route+layout, single-replica" if self.single else
                "one launch: route+histogram+METRO assignment+layout")

    def step(self, stream, ev=None):
        """One pass; with `ev`, records an event before and after each call."""
        moe, dc, cfg = self.moe, self.dc, self.cfg
        marks = iter(ev) if ev is not None else None

        def mark():
            if marks is not None:
                next(marks).record(stream)

        mark()
        if self.fused and self.single:
            dc.route_single_replica(self.logits, self.static_rank)
            mark()
        elif self.fused:
            dc.route_one_launch(self.logits)
            mark()
        else:
            moe.route_topk(self.logits, cfg.k, cfg.n_groups, cfg.groups_per_token, False, dc.topk_idx, dc.topk_w)
            mark()
            moe.demand_hist(dc.topk_idx, cfg.E, dc.counts)
            mark()
            moe.replica_assign(dc.counts, dc.replica_offsets, dc.replica_slots, dc.slot_rank, cfg.R,
                               dc.expert_slot, dc.expert_rank, dc.rank_active)
            mark()
            moe.build_layout(dc.topk_idx, dc.topk_w, dc.expert_rank, dc.layout)
            mark()
        moe.pack(self.x, dc.layout, dc.packed, dc.packed_hop1)
        mark()
        dc.combine()
        mark()

    def rows(self):
        L = self.dc.layout
        return (int(L.num_rows.item()),
                int(L.num_rows_hop1.item()) if self.cfg.mode == W.TWO_HOP else 0)


def check_status(moe, when: str):
    st = moe.get_status()
    if st != 0:
        raise RuntimeError(f"device status {when}: {moe.status_string(st)}")


def timed_steps(wl: Workload, stream, steps: int, barrier, regions: list, per_kernel=True):
    """Times exactly `steps` eager passes between a barrier and a synchronize
    on both sides (CUDA events on the launching stream).  Per-call events are
    recorded on every `stride`-th pass (all of them up to 500 passes).
    Returns (elapsed ms, mean us per call, kernels launched)."""
    import torch
    n = len(wl.names)
    stride = max(1, -(-steps // 500)) if per_kernel else 0
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
           for _ in range(len(range(0, steps, stride)) if stride else 0)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier()
    launches0 = wl.moe.kernel_launches()
    h0 = time.perf_counter()
    t0.record(stream)
    j = 0
    for i in range(steps):
        if stride and i % stride == 0:
            wl.step(stream, evs[j])
            j += 1
        else:
            wl.step(stream)
    t1.record(stream)
    barrier()
    regions.append((h0, time.perf_counter()))
    launches = wl.moe.kernel_launches() - launches0
    per = {nm: statistics.mean(e[q].elapsed_time(e[q + 1]) for e in evs) * 1e3
           for q, nm in enumerate(wl.names)} if evs else {}
    return t0.elapsed_time(t1), per, launches


def timed_graph(wl: Workload, stream, steps, warmup: int, barrier, regions: list):
    """The pass captured once in a CUDA graph, replayed `steps` times (no host
    launch latency between the kernels); `steps` may be a function of the
    measured ms per replay (timed over the warm-up replays).  Returns (elapsed
    ms, kernels per pass, replays)."""
    import torch
    g = torch.cuda.CUDAGraph()
    n0 = wl.moe.kernel_launches()
    with torch.cuda.graph(g):
        wl.step(torch.cuda.current_stream(wl.dev))
    per_pass = wl.moe.kernel_launches() - n0
    w0 = torch.cuda.Event(enable_timing=True)
    w1 = torch.cuda.Event(enable_timing=True)
    g.replay()
    w0.record(stream)
    for _ in range(max(1, warmup - 1)):
        g.replay()
    w1.record(stream)
    barrier()
    if callable(steps):
        steps = steps(w0.elapsed_time(w1) / max(1, warmup - 1))
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    h0 = time.perf_counter()
    g0.record(stream)
    for _ in range(steps):
        g.replay()
    g1.record(stream)
    barrier()
    regions.append((h0, time.perf_counter()))
    ms = g0.elapsed_time(g1)
    del g
    return ms, per_pass, steps


def timed_e2e(wl: Workload, stream, steps: int, warmup: int, chunks: int, barrier, regions: list):
    """The same pass through the public API from pinned host memory: every
    step copies its logits and activations in and its output out
    (HostPipeline overlaps the copies with the kernels)."""
    import torch
    dc, cfg = wl.dc, wl.cfg
    out_h = torch.empty((cfg.T, cfg.H), dtype=wl.x_h.dtype).pin_memory()
    pipe = wl.moe.HostPipeline(dc, chunks=chunks)
    for _ in range(max(1, warmup)):
        pipe.step(wl.logits_h, wl.x_h, out_h)
    pipe.join(stream)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    h0 = time.perf_counter()
    e0.record(stream)
    pipe.wait(e0)
    for _ in range(steps):
        pipe.step(wl.logits_h, wl.x_h, out_h)
    pipe.join(stream)
    e1.record(stream)
    barrier()
    regions.append((h0, time.perf_counter()))
    info = {"h2d_bytes_per_step": int(wl.logits_h.numel() * 4 + wl.x_h.numel() * wl.x_h.element_size()),
            "d2h_bytes_per_step": int(out_h.numel() * out_h.element_size()),
            "steps": steps,
            "pipeline": f"HostPipeline: 3 streams, {len(pipe.ranges)} token ranges per step, "
                        "double-buffered device inputs/outputs"}
    return e0.elapsed_time(e1), info


def kernel_rooflines(cfg, per_us, bytes_, peak):
    """achieved GB/s and fraction of the peak for pack and combine."""
    out = {}
    for n in ("pack", "combine"):
        if n in per_us:
            a = bytes_[n] / (per_us[n] * 1e-6) / 1e9
            out[n] = {"us": per_us[n], "algorithmic_bytes": bytes_[n], "achieved_GBps": a, "frac": a / peak}
    return out


def steps_for(probe_ms: float, min_s: float, floor: int, cap: int = 100000) -> int:
    """Passes that fill at least `min_s` seconds at `probe_ms` per pass."""
    if probe_ms <= 0:
        return floor
    return int(min(cap, max(floor, math.ceil(min_s * 1e3 / probe_ms))))


def probe_ms(wl: Workload, stream, warmup: int) -> float:
    """Warm-up passes, timed together; ms per pass."""
    import torch
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    wl.step(stream)
    a.record(stream)
    for _ in range(max(1, warmup - 1)):
        wl.step(stream)
    b.record(stream)
    b.synchronize()
    return a.elapsed_time(b) / max(1, warmup - 1)


def measure_extra(moe, label, cfg, fused, graph, e2e, args, dev, stream, barrier, sampler, peak):
    """One workload beside the headline: eager passes for at least
    `--min-region-s` seconds (per-call times), then the CUDA-graph replays or the
    end-to-end leg when asked, each region with its own clock record."""
    wl = Workload(moe, cfg, args.seed, dev, fused)
    ms_probe = probe_ms(wl, stream, args.warmup)
    check_status(moe, f"after warm-up of {label}")
    rows, rows1 = wl.rows()
    bytes_ = step_bytes(cfg, rows, rows1, wl.rm.S)
    regions = []
    steps = steps_for(ms_probe, args.min_region_s, args.steps)
    ms, per, launches = timed_steps(wl, stream, steps, barrier, regions)
    check_status(moe, f"after {label}")
    step_total = sum(bytes_[n] for n in wl.names)
    entry = {
        "workload": f"{cfg.name}: {cfg.desc}" + mode_suffix(cfg),
        "tokens": cfg.T, "rows_per_step": rows, "rows_hop1_per_step": rows1 or None,
        "front_end": wl.front_end(),
        "eager": {"steps": steps, "ms_per_step": ms / steps, "value": rows * steps / (ms * 1e-3),
                  "unit": "token-rows/s", "kernels_us": per,
                  "kernels_GBps": {n: bytes_[n] / (per[n] * 1e-6) / 1e9 for n in per},
                  "hbm_GBps": step_total / (ms / steps * 1e-3) / 1e9,
                  "gpu_launches": int(launches), "clocks": ClockRecord(regions[-1:])},
        "roofline": kernel_rooflines(cfg, per, bytes_, peak),
        "l2": l2_note(cfg, rows),
    }
    if graph:
        gms, per_pass, gsteps = timed_graph(wl, stream, lambda ms: steps_for(ms, args.min_region_s, args.steps),
                                            args.warmup, barrier, regions)
        check_status(moe, f"after graph replays of {label}")
        entry["cuda_graph"] = {"steps": gsteps, "ms_per_step": gms / gsteps, "us_per_step": gms / gsteps * 1e3,
                               "value": rows * gsteps / (gms * 1e-3), "unit": "token-rows/s",
                               "kernels_per_step": per_pass, "clocks": ClockRecord(regions[-1:])}
    if e2e:
        esteps = max(1, min(args.steps, 10))
        ems, info = timed_e2e(wl, stream, esteps, min(args.warmup, 2), args.e2e_chunks, barrier, regions)
        check_status(moe, f"after the end-to-end leg of {label}")
        entry["e2e"] = {"value": rows * esteps / (ems * 1e-3), "unit": "token-rows/s",
                        "ms_per_step": ems / esteps, **info}
    entry["clocks"] = ClockRecord(list(regions))
    del wl
    return entry, regions


def mode_suffix(cfg):
    return {W.TWO_HOP: " (two-hop)", W.DEDUP: " (dedup)", W.PER_PICK: " (per-pick)"}[cfg.mode]


def l2_note(cfg, rows):
    act = cfg.T * cfg.H * cfg.elem_bytes
    pk = rows * cfg.H * cfg.elem_bytes
    big = act + pk > 126e6
    return (("inputs larger than L2" if big else "inputs fit in L2 (decode regime; no roofline claim)") +
            " (activations %.3f GB, packed rows %.3f GB per step; L2 126 MB)" % (act / 1e9, pk / 1e9))


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
    stream = torch.cuda.current_stream(dev)

    def barrier():
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    sampler = ClockSampler(dev)
    sampler.start()
    wl = Workload(moe, cfg, args.seed + rank, dev, args.fused)
    names = wl.names
    for _ in range(args.warmup):
        wl.step(stream)
    check_status(moe, "after warm-up")
    rows, rows1 = wl.rows()

    # the headline: exactly --steps passes, device-resident inputs
    regions = []
    elapsed_ms, per_us, launches = timed_steps(wl, stream, args.steps, barrier, regions)
    check_status(moe, "after timing")
    head_regions = list(regions)
    eager_ms = elapsed_ms
    if args.graph:
        elapsed_ms, per_pass, _ = timed_graph(wl, stream, args.steps, args.warmup, barrier, regions)
        launches = per_pass * args.steps
        head_regions = regions[-1:]
        check_status(moe, "after graph replays")

    e2e_steps = max(1, min(args.steps, 10))
    e2e_ms, e2e_info = timed_e2e(wl, stream, e2e_steps, min(args.warmup, 2), args.e2e_chunks, barrier, regions)
    check_status(moe, "after e2e")

    # workload statistics of the last pass (device kernels, outside the timed regions)
    dc = wl.dc
    stats = moe.dispatch_stats(dc.counts, dc.layout.send_counts).cpu().tolist()
    _, tb_active = moe.token_balanced_assign(dc.counts, dc.replica_offsets, dc.replica_slots,
                                             dc.slot_rank, cfg.R)
    workload_stats = dict(zip(moe.STAT_NAMES, stats))
    workload_stats.update(
        max_active_metro=int(dc.rank_active.max().item()),
        max_active_token_balanced=int(tb_active.max().item()),
        active_experts=int((dc.counts > 0).sum().item()))
    check_status(moe, "after statistics")
    if args.trace:
        write_trace(args, wl, rank, world)
    del wl, dc

    # the other workloads (rank 0's replica only, outside the headline)
    extra = {}
    peak, peak_kind = measured_peak()
    if not args.headline_only:
        for label, name, over, fused, graph, e2e in EXTRA_RUNS:
            if name == cfg.name and not over and fused == args.fused and graph == args.graph:
                continue
            c = W.CONFIGS[name].with_(**over) if over else W.CONFIGS[name]
            entry, reg = measure_extra(moe, label, c, fused, graph, e2e, args, dev, stream, barrier,
                                       sampler, peak)
            extra[label] = entry
            regions += reg
            torch.cuda.empty_cache()
    sampler.stop()
    clocks_all = sampler.stats(regions)
    clocks_head = sampler.stats(head_regions)
    extra = fill_clock_records(extra, sampler)

    # whole-job aggregation: max time over ranks, rows summed over ranks
    agg = aggregate(dist, dev, [elapsed_ms, e2e_ms], [rows * args.steps, rows * e2e_steps])
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return None
    (elapsed_max, e2e_max), (rows_all, rows_e2e_all) = agg
    bytes_ = step_bytes(cfg, rows, rows1, wl_S(cfg, args.seed))
    step_total = sum(bytes_[n] for n in names)
    ms_step = elapsed_max / args.steps
    dom = max(("pack", "combine"), key=lambda n: per_us[n])
    achieved = bytes_[dom] / (per_us[dom] * 1e-6) / 1e9
    traffic = ncu_traffic(dom, cfg.name)
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
            "workload": f"{cfg.name}: {cfg.desc}" + mode_suffix(cfg), "tokens": cfg.T, "hidden": cfg.H,
            "experts": cfg.E, "top_k": cfg.k, "ranks": cfg.R, "rows_per_step": rows,
            "rows_hop1_per_step": rows1 or None,
            "layout": {0: "per_pick", 1: "dedup", 2: "two_hop"}[cfg.mode],
            "l2": l2_note(cfg, rows),
            "parallelism": f"independent replica per GPU x{world}",
            "launch": "cuda_graph" if args.graph else "eager",
            "front_end": ("separate calls" if not args.fused else
                          "one launch (fused front end)"),
        },
        "eager_ms_per_step": eager_ms / args.steps,
        "hbm_GBps": step_total / (ms_step * 1e-3) / 1e9,
        "hbm_frac_of_measured": step_total / (ms_step * 1e-3) / 1e9 / peak,
        "hbm_frac_of_8TBps": step_total / (ms_step * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
        "kernels_us": per_us,
        "kernels_GBps": {n: bytes_[n] / (per_us[n] * 1e-6) / 1e9 for n in names},
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                     "algorithmic_bytes": bytes_[dom],
                     "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"},
        "roofline_kernels": kernel_rooflines(cfg, per_us, bytes_, peak),
        "e2e": {"value": rows_e2e_all / (e2e_max * 1e-3), "unit": "token-rows/s",
                "ms_per_step": e2e_max / e2e_steps, **e2e_info},
        "gpu_launches": int(launches),
        "clocks": dict(clocks_all, window="every timed region of this run: the headline passes, its "
                                          "end-to-end leg and each workload under 'configs'"),
        "clocks_headline": clocks_head,
        "workload_stats": workload_stats,
    }
    if extra:
        line["configs"] = extra
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, args)
    return line


def wl_S(cfg, seed):
    return W.make_replica_map(cfg, seed).S


def write_trace(args, wl: Workload, rank: int, world: int):
    """The last pass's routing decisions and buffer sizes, with per-call times
    of one more pass (outside the timed regions)."""
    import torch
    cfg, dc, rm = wl.cfg, wl.dc, wl.rm
    stream = torch.cuda.current_stream(wl.dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(wl.names) + 1)]
    wl.step(stream, ev)
    ev[-1].synchronize()
    calls = [(n, ev[0].elapsed_time(ev[j]) * 1e3, ev[j].elapsed_time(ev[j + 1]) * 1e3)
             for j, n in enumerate(wl.names)]
    L = dc.layout
    if wl.fused and wl.single:  # the single-replica kernel takes the ranks as given
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


# The all-cores oracle: the same oracle functions over disjoint chunks in a
# pool of spawned processes, arrays shared through named shared memory.
_SHM = {}


def _shm_array(name, shape, dtype):
    from multiprocessing import shared_memory
    if name not in _SHM:
        _SHM[name] = shared_memory.SharedMemory(name=name)
    return np.ndarray(shape, dtype=dtype, buffer=_SHM[name].buf)


def _par_route(job):
    import oracle
    (lg, idx, w), (t0, t1), k, ng, gpt = job
    i, wt = oracle.route_topk(_shm_array(*lg)[t0:t1], k, ng, gpt)
    _shm_array(*idx)[t0:t1] = i
    _shm_array(*w)[t0:t1] = wt


def _par_pack(job):
    import oracle
    (src, dst), rt, r0 = job
    _shm_array(*dst)[r0:r0 + len(rt)] = oracle.pack(_shm_array(*src), rt)


def _par_combine(job):
    import oracle
    (p, out), lay, coef, (t0, t1), two_hop, fmt = job
    toks = np.arange(t0, t1)
    if two_hop:
        o, _ = oracle.combine_two_hop(_shm_array(*p), lay, coef, fmt, tokens=toks)
    else:
        o = oracle.combine(_shm_array(*p), lay["token_rows"], coef, tokens=toks)
    _shm_array(*out)[t0:t1] = o


class ParallelOracle:
    """route, pack and combine of the oracle over disjoint token (or row)
    chunks in `procs` spawned processes; the histogram, the assignment and the
    layout are global and run single-threaded in this process."""

    def __init__(self, cfg: W.Config, logits, x32, procs: int):
        import multiprocessing as mp
        from multiprocessing import shared_memory
        self.cfg, self.procs = cfg, procs
        T, E, H, k = cfg.T, cfg.E, cfg.H, cfg.k
        self.blocks = []

        def alloc(shape, dtype):
            n = int(np.prod(shape)) * np.dtype(dtype).itemsize
            b = shared_memory.SharedMemory(create=True, size=max(n, 1))
            self.blocks.append(b)
            return (b.name, shape, np.dtype(dtype).str), np.ndarray(shape, dtype, buffer=b.buf)

        self.lg, lg = alloc((T, E), np.float32)
        lg[:] = logits
        self.x, xv = alloc((T, H), np.float32)
        xv[:] = x32
        self.idx, self.idx_v = alloc((T, k), np.int32)
        self.w, self.w_v = alloc((T, k), np.float64)
        self.p1 = alloc((T * k, H), np.float32)[0] if cfg.mode == W.TWO_HOP else None
        self.p, _ = alloc((T * k, H), np.float32)
        self.out, _ = alloc((T, H), np.float64)
        self.pool = mp.get_context("spawn").Pool(procs)
        self.pool.map(_par_route, self._route_jobs())   # workers import numpy and the oracle

    def _chunks(self, n):
        c = -(-n // (self.procs * 2)) if n else 1
        return [(a, min(n, a + c)) for a in range(0, n, c)]

    def _route_jobs(self):
        cfg = self.cfg
        return [((self.lg, self.idx, self.w), ch, cfg.k, cfg.n_groups, cfg.groups_per_token)
                for ch in self._chunks(cfg.T)]

    def step(self, rm) -> int:
        import oracle
        cfg = self.cfg
        self.pool.map(_par_route, self._route_jobs())
        idx, w = self.idx_v.copy(), self.w_v.copy()
        counts = oracle.demand_hist(idx, cfg.E)
        _, er, _ = oracle.replica_assign(counts, rm.replica_offsets, rm.replica_slots, rm.slot_rank, cfg.R)
        L = oracle.build_layout(idx, w, er, -(-cfg.T // cfg.R), cfg.R, cfg.mode, max(cfg.ranks_per_group, 1))
        two_hop = cfg.mode == W.TWO_HOP
        if two_hop:
            rt1 = L["hop1_row_token"]
            self.pool.map(_par_pack, [((self.x, self.p1), rt1[a:b], a) for a, b in self._chunks(len(rt1))])
            rt = L["hop2_src_row"]
            self.pool.map(_par_pack, [((self.p1, self.p), rt[a:b], a) for a, b in self._chunks(len(rt))])
            lay = {key: L[key] for key in ("token_rows", "token_groups", "hop2_src_row")}
        else:
            rt = L["row_token"]
            self.pool.map(_par_pack, [((self.x, self.p), rt[a:b], a) for a, b in self._chunks(len(rt))])
            lay = {"token_rows": L["token_rows"]}
        self.pool.map(_par_combine, [((self.p, self.out), lay, L["row_coef"], ch, two_hop, cfg.dtype)
                                     for ch in self._chunks(cfg.T)])
        return int(L["num_rows"])

    def close(self):
        self.pool.close()
        self.pool.join()
        for b in self.blocks:
            b.close()
            b.unlink()


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(cfg: W.Config, args):
    """The float64 oracle on a bounded sample of the same workload: one
    thread, best of 3 passes (the reported baseline), and across all host
    cores (route, pack and combine over disjoint chunks in a process pool; the
    global histogram, assignment and layout single-threaded), best of 3."""
    tokens = min(cfg.T, args.cpu_sample_tokens)
    sub, logits, x32, rm = oracle_sample(cfg, tokens, args.seed)
    times, rows = [], 0
    for _ in range(3):
        t0 = time.perf_counter()
        rows = oracle_step(sub, logits, x32, rm)
        times.append(time.perf_counter() - t0)
    best = min(times)
    cores = host_cores()
    out = {"value": rows / best, "unit": "token-rows/s", "cores": 1, "kind": "oracle",
           "sample": f"first {tokens} of {cfg.T} tokens of the same workload, one full pass of the "
                     f"float64 numpy oracle ({rows} rows), best of 3 ({', '.join('%.2f' % t for t in times)} s), "
                     f"single thread",
           "host_cpus": cores, "cpu_model": cpu_model()}
    if cores > 1 and not args.no_cpu_all_cores:
        par = ParallelOracle(sub, logits, x32, cores)
        try:
            ptimes = []
            for _ in range(3):
                t0 = time.perf_counter()
                prow = par.step(rm)
                ptimes.append(time.perf_counter() - t0)
        finally:
            par.close()
        assert prow == rows
        out["all_cores"] = {
            "value": rows / min(ptimes), "unit": "token-rows/s", "cores": cores, "kind": "oracle",
            "sample": f"the same {tokens} tokens; route, pack and combine over disjoint chunks in "
                      f"{cores} spawned processes, histogram, assignment and layout single-threaded; "
                      f"best of 3 ({', '.join('%.2f' % t for t in ptimes)} s)"}
    return out


def config_of(args) -> W.Config:
    cfg = W.CONFIGS[args.config]
    if args.tokens:
        cfg = cfg.with_(T=args.tokens, name=f"{cfg.name}_T{args.tokens}")
    return cfg


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return None
    cfg = config_of(args)
    tokens = min(cfg.T, args.cpu_sample_tokens)
    sub, logits, x32, rm = oracle_sample(cfg, tokens, args.seed)
    for _ in range(args.warmup):
        oracle_step(sub, logits, x32, rm)
    rows, times = 0, []
    t_all = time.perf_counter()
    for _ in range(args.steps):
        t0 = time.perf_counter()
        rows += oracle_step(sub, logits, x32, rm)
        times.append(time.perf_counter() - t0)
    dt = time.perf_counter() - t_all
    value = rows / dt
    best = rows / max(args.steps, 1) / min(times) if times else None
    sample = (f"each step: the first {tokens} of {cfg.T} tokens of the same workload through the "
              f"float64 numpy oracle, single thread (the sample of bench.py's cpu_baseline); "
              f"best step {best:.1f} token-rows/s" if best else "no steps")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "token-rows/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / max(args.steps, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic, seeded",
        "config": {"workload": f"{cfg.name}: {cfg.desc}" + mode_suffix(cfg), "tokens": cfg.T, "hidden": cfg.H,
                   "experts": cfg.E, "top_k": cfg.k, "ranks": cfg.R,
                   "parallelism": "CPU oracle on rank 0"},
        "cpu_baseline": {"value": value, "unit": "token-rows/s", "cores": 1, "kind": "oracle",
                         "sample": sample, "cpu_model": cpu_model(), "host_cpus": host_cores()},
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
    ap.add_argument("--cpu-sample-tokens", type=int, default=4096,
                    help="token sample of the CPU oracle (cpu_baseline and --impl reference)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-cpu-all-cores", action="store_true",
                    help="skip the all-cores figure of the CPU baseline")
    ap.add_argument("--headline-only", action="store_true",
                    help="time only the --config workload (no 'configs' entries)")
    ap.add_argument("--min-region-s", type=float, default=1.0,
                    help="length of each timed region of the 'configs' entries, in seconds")
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
