"""One full pass of the dispatch/combine path with preallocated buffers.

route_topk -> demand_hist -> replica_assign -> build_layout -> pack ->
(experts) -> combine, all on one stream, all in libmoe.so's kernels.  The
expert computation between pack and combine is the caller's; ``step`` runs
the path with identity experts (the packed rows are the expert outputs).
"""
from __future__ import annotations

from typing import Optional

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
