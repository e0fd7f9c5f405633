"""One full pass of the dispatch/combine path with preallocated buffers.

route_topk -> demand_hist -> replica_assign -> build_layout -> pack ->
(experts) -> combine, all on one stream, all in libmoe.so's kernels.  The
expert computation between pack and combine is the caller's; ``step`` runs
the path with identity experts (the packed rows are the expert outputs).
"""
from __future__ import annotations

from typing import Callable, Optional

import torch

from . import _binding as B


class DispatchCombine:
    def __init__(self, T: int, H: int, E: int, k: int, R: int, replica_offsets: torch.Tensor,
                 replica_slots: torch.Tensor, slot_rank: torch.Tensor, mode: int = B.DEDUP,
                 tokens_per_rank: Optional[int] = None, ranks_per_group: int = 1,
                 n_groups: int = 0, groups_per_token: int = 0, renormalize: bool = False,
                 dtype=torch.bfloat16, out_dtype=None, device="cuda",
                 capacity: Optional[int] = None, capacity_hop1: Optional[int] = None):
        self.T, self.H, self.E, self.k, self.R, self.mode = T, H, E, k, R, mode
        self.n_groups, self.groups_per_token, self.renormalize = n_groups, groups_per_token, renormalize
        self.dtype = dtype
        self.out_dtype = dtype if out_dtype is None else out_dtype
        dev = torch.device(device)
        self.replica_offsets = replica_offsets.to(dev, torch.int32).contiguous()
        self.replica_slots = replica_slots.to(dev, torch.int32).contiguous()
        self.slot_rank = slot_rank.to(dev, torch.int32).contiguous()
        i32 = dict(dtype=torch.int32, device=dev)
        self.topk_idx = torch.empty((T, k), **i32)
        self.topk_w = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.counts = torch.empty(E, **i32)
        self.expert_slot = torch.empty(E, **i32)
        self.expert_rank = torch.empty(E, **i32)
        self.rank_active = torch.empty(R, **i32)
        tpr = -(-T // R) if tokens_per_rank is None else tokens_per_rank
        self.layout = B.Layout(T, k, E, R, mode, tpr, ranks_per_group, capacity, capacity_hop1, dev)
        self.packed = torch.empty((max(self.layout.capacity, 1), H), dtype=dtype, device=dev)
        self.packed_hop1 = self.hop1_buf = None
        if mode == B.TWO_HOP:
            self.packed_hop1 = torch.empty((max(self.layout.capacity_hop1, 1), H), dtype=dtype, device=dev)
            self.hop1_buf = torch.empty_like(self.packed_hop1)
        self.out = torch.empty((T, H), dtype=self.out_dtype, device=dev)

    def route(self, logits: torch.Tensor):
        B.route_topk(logits, self.k, self.n_groups, self.groups_per_token, self.renormalize,
                     self.topk_idx, self.topk_w)
        B.demand_hist(self.topk_idx, self.E, self.counts)
        B.replica_assign(self.counts, self.replica_offsets, self.replica_slots, self.slot_rank,
                         self.R, self.expert_slot, self.expert_rank, self.rank_active)
        B.build_layout(self.topk_idx, self.topk_w, self.expert_rank, self.layout)

    def route_single_replica(self, logits: torch.Tensor, expert_rank: torch.Tensor):
        """The same outputs as route() for a map with one replica per expert,
        in one fused pass (expert_rank: each expert's only rank)."""
        B.route_layout_single_replica(logits, self.k, expert_rank, self.layout, self.n_groups,
                                      self.groups_per_token, self.renormalize, self.topk_idx,
                                      self.topk_w, self.counts, self.rank_active)

    def route_one_launch(self, logits: torch.Tensor):
        """The same outputs as route(), from one launch (moe_route_assign_layout)."""
        B.route_assign_layout(logits, self.k, self.replica_offsets, self.replica_slots, self.slot_rank,
                              self.layout, self.n_groups, self.groups_per_token, self.renormalize,
                              self.topk_idx, self.topk_w, self.counts, self.expert_slot,
                              self.expert_rank, self.rank_active)

    def dispatch(self, logits: torch.Tensor, x: torch.Tensor) -> torch.Tensor:
        self.route(logits)
        B.pack(x, self.layout, self.packed, self.packed_hop1)
        return self.packed

    def combine(self, y: Optional[torch.Tensor] = None) -> torch.Tensor:
        y = self.packed if y is None else y
        return B.combine(y, self.layout, self.out, self.out_dtype, None, self.hop1_buf)

    def step(self, logits: torch.Tensor, x: torch.Tensor) -> torch.Tensor:
        self.dispatch(logits, x)
        return self.combine()


def token_ranges(T: int, chunks: int):
    """`chunks` contiguous, non-empty token ranges [a, b) covering [0, T) in
    order, of sizes that differ by at most one (fewer when T < chunks)."""
    n = max(1, min(chunks, T))
    edges = [T * i // n for i in range(n + 1)]
    return [(a, b) for a, b in zip(edges, edges[1:]) if b > a]


class HostPipeline:
    """Steps of a DispatchCombine whose inputs and outputs are pinned host
    buffers, with the host<->device copies overlapped with the kernels.

    Three streams: copies in, kernels, copies out.  A step's logits are copied
    first (the router needs nothing else); its activations follow in `chunks`
    token ranges, and pack runs on each range as soon as it has arrived.  After
    the experts (``experts(dc) -> y``, identity by default: y = the packed
    rows), combine runs range by range and each finished range of the output
    is copied back at once.  Device logits, activations and outputs are
    double-buffered, so step s+1's copies in run while step s computes and
    copies out; in steady state a step costs about the larger of its two copy
    directions.  Every kernel is the DispatchCombine's (pack and combine on
    token ranges give the rows and outputs of whole-range calls).
    """

    def __init__(self, dc: DispatchCombine, chunks: int = 8):
        self.dc = dc
        dev = dc.out.device
        self.s_in = torch.cuda.Stream(dev)
        self.s_k = torch.cuda.Stream(dev)
        self.s_out = torch.cuda.Stream(dev)
        T, E, H = dc.T, dc.E, dc.H
        self.logits = [torch.empty((T, E), dtype=torch.float32, device=dev) for _ in range(2)]
        self.x = [torch.empty((T, H), dtype=dc.dtype, device=dev) for _ in range(2)]
        self.out = [torch.empty((T, H), dtype=dc.out_dtype, device=dev) for _ in range(2)]
        self.ranges = token_ranges(T, chunks)
        self.in_free = [None, None]   # kernels done with logits[b] and x[b]
        self.out_free = [None, None]  # copies out done with out[b]
        self.last = [None, None, None]  # last event of each stream
        self.i = 0

    def _record(self, stream) -> torch.cuda.Event:
        ev = torch.cuda.Event()
        ev.record(stream)
        return ev

    def wait(self, event: torch.cuda.Event):
        """Every pipeline stream waits for `event` (work enqueued later starts after it)."""
        for s in (self.s_in, self.s_k, self.s_out):
            s.wait_event(event)

    def join(self, stream=None):
        """`stream` (default: the current one) waits for all enqueued pipeline work."""
        stream = torch.cuda.current_stream() if stream is None else stream
        for s in (self.s_in, self.s_k, self.s_out):
            stream.wait_event(self._record(s))

    def step(self, logits_h: torch.Tensor, x_h: torch.Tensor, out_h: torch.Tensor,
             experts: Optional[Callable[[DispatchCombine], torch.Tensor]] = None):
        """Enqueues one step: logits_h [T][E] f32, x_h [T][H] and out_h [T][H]
        pinned host tensors.  out_h is complete once join() has been waited on."""
        dc, b = self.dc, self.i & 1
        self.i += 1
        with torch.cuda.stream(self.s_in):
            if self.in_free[b] is not None:
                self.s_in.wait_event(self.in_free[b])
            self.logits[b].copy_(logits_h, non_blocking=True)
            ev_lg = self._record(self.s_in)
            ev_x = []
            for a, e in self.ranges:
                self.x[b][a:e].copy_(x_h[a:e], non_blocking=True)
                ev_x.append(self._record(self.s_in))
        with torch.cuda.stream(self.s_k):
            self.s_k.wait_event(ev_lg)
            dc.route(self.logits[b])
            for (a, e), ev in zip(self.ranges, ev_x):
                self.s_k.wait_event(ev)
                B.pack(self.x[b], dc.layout, dc.packed, dc.packed_hop1, tokens=(a, e))
            self.in_free[b] = self._record(self.s_k)
            y = dc.packed if experts is None else experts(dc)
            if self.out_free[b] is not None:
                self.s_k.wait_event(self.out_free[b])
            ev_o = []
            for a, e in self.ranges:
                B.combine(y, dc.layout, self.out[b], dc.out_dtype, None, dc.hop1_buf, tokens=(a, e))
                ev_o.append(self._record(self.s_k))
        with torch.cuda.stream(self.s_out):
            for (a, e), ev in zip(self.ranges, ev_o):
                self.s_out.wait_event(ev)
                out_h[a:e].copy_(self.out[b][a:e], non_blocking=True)
            self.out_free[b] = self._record(self.s_out)

    def synchronize(self):
        for s in (self.s_in, self.s_k, self.s_out):
            s.synchronize()
