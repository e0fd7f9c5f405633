"""Seeded synthetic inputs for the MoE dispatch/combine path.

This module is shared by the CPU oracle tests, the CUDA parity tests and the
benchmark.  It draws random numbers and builds the replica placement maps that
the path takes as *inputs*; it computes none of the method itself (no softmax,
no top-k, no histogram, no assignment, no layout).

The five workloads follow the problem statements on the source pages:

* ``c1`` METRO toy decode -- "METRO AllGather vs AllToAll for MoE decode"
  (fanout.sh), section "Work the 8-GPU payload example": 8 ranks x 32 decode
  tokens, fp16 activations.  Hidden 4096, 64 experts top-2, one primary replica
  per expert plus 16 redundant replicas (80 slots, 10 per rank).
* ``c2`` MoE decode with METRO assignment -- same page, section "changes the
  routing information": 8 ranks x 128 tokens, hidden 7168 bf16, 256 experts
  top-8, 32 redundant replicas on the hottest experts, Zipf(1.1) expert bias.
* ``c3`` training dispatch with single-send dedup -- ainewsletter summary of
  arXiv:2610.09372, "Two locality techniques": 8192 tokens, hidden 4096 bf16,
  64 experts top-6, 32 ranks, 8 co-selection clusters; correlated (e // 2) vs
  round-robin (e % 32) placement.
* ``c4`` prefill-scale dispatch+combine: 65536 tokens, hidden 7168 bf16,
  256 experts top-8, 64 ranks, power-law (alpha 1.2) expert bias.
* ``c5`` two-hop hierarchical layout -- TerraceMoE editorial, "The core
  problem": 32768 tokens, hidden 4096 bf16, 128 experts top-8, 8 groups x 8
  ranks, at most 4 groups per token.

Recipes for the points the pages leave open:

* Zipf / power-law bias: ``bias[e] = -s * ln(1 + pi[e])`` where ``pi`` is a
  seeded permutation of the experts (so hot experts are spread over ranks).
* Clusters (c3): cluster ``c`` is experts ``[8c, 8c+8)``; each token draws a
  home cluster uniformly and gets ``logit = N(0,1) + beta`` on its home
  cluster's experts, ``beta = 1.0``.  The resulting in-cluster share of top-k
  picks is measured (about 0.4), not tuned per run.
* Redundant replicas: c1 draws its 16 replicated experts uniformly (its logits
  carry no bias, so no expert is hotter than another); c2 replicates the 32
  experts with the largest bias.  Each redundant replica goes to the rank with
  the fewest slots that does not already hold that expert (ties to the lower
  rank).  Slots are numbered rank-major.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

# Layout modes; the values match the C ABI enum ``moe_layout_mode``.
PER_PICK = 0
DEDUP = 1
TWO_HOP = 2

DTYPE_BYTES = {"f16": 2, "bf16": 2, "f32": 4}


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    desc: str
    T: int                 # gathered token set
    R: int                 # logical EP ranks
    H: int                 # hidden size
    dtype: str             # activation dtype: "f16" | "bf16"
    E: int                 # experts
    k: int                 # top-k
    n_redundant: int = 0   # redundant replicas on top of one primary per expert
    redundant_pick: str = "none"   # "uniform" | "hottest"
    bias: str = "none"     # "none" | "powerlaw"
    bias_s: float = 0.0
    clusters: int = 0      # co-selection clusters (c3)
    cluster_beta: float = 0.0
    placement: str = "block"   # "block" (e // (E/R)) | "roundrobin" (e % R)
    mode: int = DEDUP
    n_groups: int = 0      # router groups (two-hop / group-limited)
    groups_per_token: int = 0
    ranks_per_group: int = 0

    @property
    def tokens_per_rank(self) -> int:
        return self.T // self.R

    @property
    def elem_bytes(self) -> int:
        return DTYPE_BYTES[self.dtype]

    def with_(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "c1": Config("c1", "METRO toy decode: 8 ranks x 32 tokens, H4096 fp16, E64 top-2, 80 slots",
                 T=256, R=8, H=4096, dtype="f16", E=64, k=2,
                 n_redundant=16, redundant_pick="uniform"),
    "c2": Config("c2", "MoE decode METRO: 8 ranks x 128 tokens, H7168 bf16, E256 top-8, 288 slots, Zipf 1.1",
                 T=1024, R=8, H=7168, dtype="bf16", E=256, k=8,
                 n_redundant=32, redundant_pick="hottest", bias="powerlaw", bias_s=1.1),
    "c3": Config("c3", "training dedup: 8192 tokens, H4096 bf16, E64 top-6, EP32, 8 clusters, correlated placement",
                 T=8192, R=32, H=4096, dtype="bf16", E=64, k=6,
                 clusters=8, cluster_beta=1.0, placement="block"),
    "c4": Config("c4", "prefill dispatch+combine: 65536 tokens, H7168 bf16, E256 top-8, EP64, power-law 1.2",
                 T=65536, R=64, H=7168, dtype="bf16", E=256, k=8,
                 bias="powerlaw", bias_s=1.2),
    "c5": Config("c5", "two-hop: 32768 tokens, H4096 bf16, E128 top-8, 8 groups x 8 ranks, <=4 groups/token",
                 T=32768, R=64, H=4096, dtype="bf16", E=128, k=8,
                 mode=TWO_HOP, n_groups=8, groups_per_token=4, ranks_per_group=8),
}


@dataclasses.dataclass
class ReplicaMap:
    """CSR map expert -> replica slots, and slot -> hosting rank."""
    replica_offsets: np.ndarray   # int32 [E+1]
    replica_slots: np.ndarray     # int32 [S]
    slot_rank: np.ndarray         # int32 [S]

    @property
    def S(self) -> int:
        return int(self.slot_rank.shape[0])


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, stream]))


def expert_bias(cfg: Config, seed: int) -> np.ndarray:
    """Per-expert logit bias (float32 [E]); zeros when the config has none."""
    if cfg.bias == "none":
        return np.zeros(cfg.E, np.float32)
    perm = _rng(seed, 1).permutation(cfg.E)        # pi[e]: popularity rank of e
    return (-cfg.bias_s * np.log1p(perm.astype(np.float64))).astype(np.float32)


def make_logits(cfg: Config, seed: int = 0, T: Optional[int] = None) -> np.ndarray:
    """Router logits, float32 [T][E], row-major."""
    T = cfg.T if T is None else T
    rng = _rng(seed, 2)
    logits = rng.standard_normal((T, cfg.E), dtype=np.float32)
    logits += expert_bias(cfg, seed)[None, :]
    if cfg.clusters:
        per = cfg.E // cfg.clusters
        home = _rng(seed, 3).integers(0, cfg.clusters, size=T)
        cols = home[:, None] * per + np.arange(per)[None, :]
        logits[np.arange(T)[:, None], cols] += np.float32(cfg.cluster_beta)
    return logits


def make_activations_f32(cfg: Config, seed: int = 0, T: Optional[int] = None) -> np.ndarray:
    """Token activations ~N(0,1) as float32 [T][H] (cast to cfg.dtype by the caller)."""
    T = cfg.T if T is None else T
    return _rng(seed, 4).standard_normal((T, cfg.H), dtype=np.float32)


def make_activations(cfg: Config, seed: int = 0, T: Optional[int] = None):
    """Token activations as a CPU torch tensor of cfg.dtype (RNE from float32)."""
    import torch
    tdt = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[cfg.dtype]
    T = cfg.T if T is None else T
    out = torch.empty((T, cfg.H), dtype=tdt)
    chunk = max(1, (1 << 26) // cfg.H)
    rng = _rng(seed, 4)
    for s in range(0, T, chunk):
        n = min(chunk, T - s)
        out[s:s + n] = torch.from_numpy(rng.standard_normal((n, cfg.H), dtype=np.float32))
    return out


def expert_home_rank(cfg: Config) -> np.ndarray:
    """Rank of each expert's primary replica (int32 [E])."""
    e = np.arange(cfg.E)
    if cfg.placement == "roundrobin":
        return (e % cfg.R).astype(np.int32)
    per = cfg.E // cfg.R
    assert per * cfg.R == cfg.E, "block placement needs R | E"
    return (e // per).astype(np.int32)


def make_replica_map(cfg: Config, seed: int = 0) -> ReplicaMap:
    """Primary replica per expert plus cfg.n_redundant redundant replicas."""
    E, R = cfg.E, cfg.R
    home = expert_home_rank(cfg)
    held = [set() for _ in range(R)]           # experts held per rank
    per_rank = [[] for _ in range(R)]          # experts in slot order per rank
    for e in range(E):
        held[home[e]].add(e)
        per_rank[home[e]].append(e)
    if cfg.n_redundant:
        if cfg.redundant_pick == "uniform":
            extra = _rng(seed, 5).choice(E, size=cfg.n_redundant, replace=False)
        elif cfg.redundant_pick == "hottest":
            extra = np.argsort(-expert_bias(cfg, seed).astype(np.float64), kind="stable")[:cfg.n_redundant]
        else:
            raise ValueError(cfg.redundant_pick)
        for e in extra:
            e = int(e)
            cand = [r for r in range(R) if e not in held[r]]
            r = min(cand, key=lambda r: (len(per_rank[r]), r))
            held[r].add(e)
            per_rank[r].append(e)
    slot_expert, slot_rank = [], []
    for r in range(R):
        for e in per_rank[r]:
            slot_expert.append(e)
            slot_rank.append(r)
    slot_expert = np.asarray(slot_expert, np.int64)
    order = np.argsort(slot_expert, kind="stable")    # slots grouped by expert, ascending slot
    counts = np.bincount(slot_expert, minlength=E)
    offsets = np.zeros(E + 1, np.int32)
    offsets[1:] = np.cumsum(counts)
    return ReplicaMap(offsets, order.astype(np.int32), np.asarray(slot_rank, np.int32))


def identity_replica_map(E: int, expert_rank: np.ndarray) -> ReplicaMap:
    """One slot per expert: slot e on rank expert_rank[e]."""
    return ReplicaMap(np.arange(E + 1, dtype=np.int32), np.arange(E, dtype=np.int32),
                      np.asarray(expert_rank, np.int32))


def make_uniform_coefs(n: int, seed: int = 0) -> np.ndarray:
    """Random per-row combine coefficients in [0.05, 1) (float32 [n])."""
    return _rng(seed, 6).uniform(0.05, 1.0, size=n).astype(np.float32)


def sample_indices(n: int, count: int, seed: int = 0) -> np.ndarray:
    """Sorted sample of distinct indices in [0, n), always including 0 and n-1."""
    if n <= count:
        return np.arange(n)
    pick = _rng(seed, 7).choice(n, size=count - 2, replace=False)
    return np.unique(np.concatenate([[0, n - 1], pick]))


def algorithmic_pack_bytes(T: int, rows: int, H: int, elem_bytes: int) -> int:
    """Minimum HBM bytes of a read-once / write-each-row pack: (T + rows) * H * b."""
    return (T + rows) * H * elem_bytes


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = [n for n in dir() if not n.startswith("_") and n not in ("annotations", "dataclasses", "math", "Optional", "np")]
