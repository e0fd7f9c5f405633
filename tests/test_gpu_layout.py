"""GPU parity: the stable per-destination layout (one cooperative launch:
per-block counts, grid barrier, each block's prefix from the count table)
against the CPU oracle: every integer field bit-exact, the coefficients within
their float bound; plus the device-side error paths."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from gpu_util import assert_layout_equal, layout_fields, moe, to_dev  # noqa: F401

pytestmark = pytest.mark.gpu
U = 2.0 ** -24


def run_layout(moe, idx, w, er, T, tpr, k, E, R, mode, rpg=1, capacity=None):
    L = moe.Layout(T, k, E, R, mode, tpr, rpg, capacity=capacity)
    moe.build_layout(to_dev(idx.astype(np.int32)), to_dev(w.astype(np.float32)),
                     to_dev(er.astype(np.int32)), L)
    return L


def ref_layout(idx, w, er, tpr, R, mode, rpg=1):
    # the device gets float32 weights: the oracle sums the same values in float64
    return oracle.build_layout(idx, w.astype(np.float32).astype(np.float64), er, tpr, R, mode, rpg)


CONFIG_CASES = [("c1", W.DEDUP, "block"), ("c1", W.PER_PICK, "block"), ("c2", W.DEDUP, "block"),
                ("c3", W.DEDUP, "block"), ("c3", W.PER_PICK, "block"), ("c3", W.DEDUP, "roundrobin"),
                ("c3", W.PER_PICK, "roundrobin"), ("c4", W.DEDUP, "block"), ("c4", W.PER_PICK, "block"),
                ("c5", W.TWO_HOP, "block")]


@pytest.mark.parametrize("name,mode,placement", CONFIG_CASES)
def test_layout_full_size_configs(moe, name, mode, placement):
    cfg = W.CONFIGS[name].with_(placement=placement)
    rm = W.make_replica_map(cfg, 0)
    idx, w = oracle.route_topk(W.make_logits(cfg, 0), cfg.k, cfg.n_groups, cfg.groups_per_token)
    counts = oracle.demand_hist(idx, cfg.E)
    _, er, _ = oracle.replica_assign(counts, rm.replica_offsets, rm.replica_slots, rm.slot_rank, cfg.R)
    rpg = max(cfg.ranks_per_group, 1)
    L = run_layout(moe, idx, w, er, cfg.T, cfg.tokens_per_rank, cfg.k, cfg.E, cfg.R, mode, rpg)
    assert moe.get_status() == 0
    ref = ref_layout(idx, w, er, cfg.tokens_per_rank, cfg.R, mode, rpg)
    assert_layout_equal(layout_fields(L, mode), ref, mode, w_tol=cfg.k * U)


@pytest.mark.parametrize("mode,R,rpg", [(W.DEDUP, 32, 1), (W.PER_PICK, 32, 1), (W.TWO_HOP, 32, 4)])
def test_layout_multi_tile_chunks(moe, mode, R, rpg):
    """100000 tokens: each block's chunk spans two 256-token tiles, so phase 2
    reloads the picks tile by tile and carries every bin's base across tiles."""
    cfg = W.CONFIGS["c3"].with_(T=100000, R=R, mode=mode)
    idx, w = oracle.route_topk(W.make_logits(cfg, 3), cfg.k)
    er = np.random.default_rng(5).integers(0, R, size=cfg.E).astype(np.int32)
    tpr = -(-cfg.T // R)
    L = run_layout(moe, idx, w, er, cfg.T, tpr, cfg.k, cfg.E, R, mode, rpg)
    assert moe.get_status() == 0
    ref = ref_layout(idx, w, er, tpr, R, mode, rpg)
    assert_layout_equal(layout_fields(L, mode), ref, mode, w_tol=cfg.k * U)


@pytest.mark.parametrize("T,E,k,R,tpr,mode,rpg,skew", [
    (1, 8, 2, 4, 1, W.DEDUP, 1, False),
    (257, 16, 3, 8, 33, W.DEDUP, 1, False),        # ragged last tile
    (1000, 64, 6, 64, 16, W.DEDUP, 1, True),       # many source ranks per tile, skewed demand
    (64, 64, 8, 64, 1, W.DEDUP, 1, False),         # one token per source rank
    (3000, 32, 4, 1, 3000, W.DEDUP, 1, False),     # a single rank
    (600, 1024, 16, 64, 10, W.PER_PICK, 1, False),  # widest bins and picks
    (513, 12, 12, 5, 103, W.PER_PICK, 1, True),    # k = E
    (2049, 128, 8, 64, 33, W.TWO_HOP, 8, True),
    (999, 64, 5, 16, 63, W.TWO_HOP, 16, False),    # one group
    (700, 40, 7, 12, 59, W.TWO_HOP, 1, False),     # one rank per group
    (5000, 256, 8, 64, 79, W.TWO_HOP, 4, False),
    (512, 64, 4, 32, 16, W.DEDUP, 1, True),        # the largest set counted in one pass
    (513, 64, 4, 32, 17, W.DEDUP, 1, True),        # the smallest one with the count table
    (512, 128, 8, 64, 8, W.TWO_HOP, 8, False),
    (513, 128, 8, 64, 9, W.TWO_HOP, 8, False),
])
def test_layout_edges(moe, T, E, k, R, tpr, mode, rpg, skew):
    rng = np.random.default_rng(T + 31 * E + k)
    p = None
    if skew:
        p = 1.0 / (1.0 + np.arange(E)) ** 1.5
        p /= p.sum()
    idx = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0.01, 1.0, size=(T, k)).astype(np.float32)
    er = rng.integers(0, R, size=E).astype(np.int32)
    L = run_layout(moe, idx, w, er, T, tpr, k, E, R, mode, rpg)
    assert moe.get_status() == 0
    ref = ref_layout(idx, w, er, tpr, R, mode, rpg)
    assert_layout_equal(layout_fields(L, mode), ref, mode, w_tol=k * U)


def test_layout_zero_tokens(moe):
    L = moe.Layout(0, 2, 8, 4, W.DEDUP, 1)
    moe.build_layout(torch.empty((0, 2), dtype=torch.int32, device="cuda"),
                     torch.empty((0, 2), dtype=torch.float32, device="cuda"),
                     torch.zeros(8, dtype=torch.int32, device="cuda"), L)
    assert moe.get_status() == 0
    assert int(L.num_rows.item()) == 0 and L.rank_offsets.cpu().tolist() == [0] * 5


def test_layout_capacity_overflow(moe):
    rng = np.random.default_rng(5)
    T, E, k, R = 700, 32, 4, 8
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0.1, 1, size=(T, k)).astype(np.float32)
    er = (np.arange(E) % R).astype(np.int32)
    ref = ref_layout(idx, w, er, 88, R, W.DEDUP)
    n = int(ref["num_rows"])
    cap = n - 37
    L = run_layout(moe, idx, w, er, T, 88, k, E, R, W.DEDUP, capacity=cap)
    assert moe.get_status() == 7                      # MOE_ERR_CAPACITY
    assert int(L.num_rows.item()) == n                # the true count, to size a retry
    assert np.array_equal(L.row_token[:cap].cpu().numpy(), ref["row_token"][:cap])
    tr = ref["token_rows"].copy()
    tr[tr >= cap] = -1
    assert np.array_equal(L.token_rows.cpu().numpy(), tr)


def test_layout_bad_expert_id(moe):
    idx = np.tile(np.arange(4, dtype=np.int32), (300, 1))
    idx[100, 2] = 50
    w = np.ones((300, 4), np.float32)
    er = np.arange(8, dtype=np.int32) % 4
    run_layout(moe, idx, w, er, 300, 75, 4, 8, 4, W.DEDUP)
    assert moe.get_status() == 6


def test_layout_bounded_wait_reports_timeout(moe):
    """A block that never arrives at the grid barrier: the others' waits run
    out after the set limit and report MOE_ERR_TIMEOUT; the context stays
    usable.  6144 tokens: above the size that the layout counts in one pass
    without a barrier (512), so the barrier path runs."""
    rng = np.random.default_rng(9)
    T, E, k, R = 256 * 24, 16, 2, 4
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    w = np.ones((T, k), np.float32)
    er = (np.arange(E) % R).astype(np.int32)
    moe.debug_set_wait(20_000_000, 2)                  # 20 ms; tile 2 stays silent
    try:
        run_layout(moe, idx, w, er, T, T // R, k, E, R, W.DEDUP)
        assert moe.get_status() == 4                  # MOE_ERR_TIMEOUT
    finally:
        moe.debug_set_wait(0, -1)
    L = run_layout(moe, idx, w, er, T, T // R, k, E, R, W.DEDUP)
    assert moe.get_status() == 0
    ref = ref_layout(idx, w, er, T // R, R, W.DEDUP)
    assert np.array_equal(L.row_token[:int(ref["num_rows"])].cpu().numpy(), ref["row_token"])
