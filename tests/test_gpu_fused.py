"""GPU parity of the fused single-replica path (route + demand histogram +
assignment + layout in one pass) against the separate calls and the oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from gpu_util import layout_fields, moe, to_dev  # noqa: F401

pytestmark = pytest.mark.gpu


def run_both(moe, cfg, logits, er_static):
    rm = W.identity_replica_map(cfg.E, er_static)
    rpg = max(cfg.ranks_per_group, 1)
    tpr = -(-cfg.T // cfg.R)
    lg = to_dev(logits)
    sep = moe.DispatchCombine(cfg.T, cfg.H, cfg.E, cfg.k, cfg.R, to_dev(rm.replica_offsets),
                              to_dev(rm.replica_slots), to_dev(rm.slot_rank), cfg.mode, tpr, rpg,
                              cfg.n_groups, cfg.groups_per_token, dtype=torch.bfloat16)
    sep.route(lg)
    fus = moe.DispatchCombine(cfg.T, cfg.H, cfg.E, cfg.k, cfg.R, to_dev(rm.replica_offsets),
                              to_dev(rm.replica_slots), to_dev(rm.slot_rank), cfg.mode, tpr, rpg,
                              cfg.n_groups, cfg.groups_per_token, dtype=torch.bfloat16)
    fus.topk_idx.fill_(-7)
    fus.route_single_replica(lg, to_dev(er_static.astype(np.int32)))
    return sep, fus


def assert_same_route(moe, cfg, sep, fus):
    assert moe.get_status() == 0
    assert torch.equal(sep.topk_idx, fus.topk_idx)
    assert torch.equal(sep.topk_w.view(torch.int32), fus.topk_w.view(torch.int32))
    assert torch.equal(sep.counts, fus.counts)
    assert torch.equal(sep.rank_active, fus.rank_active)
    a, b = layout_fields(sep.layout, cfg.mode), layout_fields(fus.layout, cfg.mode)
    for key in a:
        assert np.array_equal(np.asarray(a[key]), np.asarray(b[key])), key


@pytest.mark.parametrize("name,mode,placement", [("c3", W.DEDUP, "block"), ("c3", W.PER_PICK, "roundrobin"),
                                                 ("c4", W.DEDUP, "block"), ("c5", W.TWO_HOP, "block")])
def test_fused_matches_separate_calls(moe, name, mode, placement):
    cfg = W.CONFIGS[name].with_(mode=mode, placement=placement)
    logits = W.make_logits(cfg, 0)
    er = W.expert_home_rank(cfg)
    sep, fus = run_both(moe, cfg, logits, er)
    assert_same_route(moe, cfg, sep, fus)
    # and the oracle
    idx, _ = oracle.route_topk(logits, cfg.k, cfg.n_groups, cfg.groups_per_token)
    assert np.array_equal(fus.topk_idx.cpu().numpy(), idx)
    assert np.array_equal(fus.counts.cpu().numpy(), oracle.demand_hist(idx, cfg.E))


@pytest.mark.parametrize("T,E,k,R,mode,rpg", [(1, 8, 2, 4, W.DEDUP, 1), (77, 40, 3, 8, W.DEDUP, 1),
                                              (300, 1024, 16, 64, W.PER_PICK, 1), (513, 96, 6, 12, W.TWO_HOP, 3),
                                              (2000, 64, 8, 1, W.DEDUP, 1)])
def test_fused_edges(moe, T, E, k, R, mode, rpg):
    cfg = W.Config("edge", "edge", T=T, R=R, H=64, dtype="bf16", E=E, k=k, mode=mode,
                   ranks_per_group=rpg if mode == W.TWO_HOP else 0)
    rng = np.random.default_rng(T + E)
    logits = (rng.integers(-3, 4, size=(T, E)) * 0.5).astype(np.float32)   # with ties
    er = rng.integers(0, R, size=E).astype(np.int32)
    sep, fus = run_both(moe, cfg, logits, er)
    assert_same_route(moe, cfg, sep, fus)


@pytest.mark.parametrize("mode,rpg", [(W.DEDUP, 1), (W.TWO_HOP, 2)])
def test_fused_multi_tile_chunks(moe, mode, rpg):
    """140000 tokens: the fused launch's chunks span two tiles each (phase 2
    reloads the picks its warps wrote in phase 1)."""
    cfg = W.Config("mt", "mt", T=140000, R=8, H=64, dtype="bf16", E=64, k=2, mode=mode,
                   ranks_per_group=rpg if mode == W.TWO_HOP else 0)
    rng = np.random.default_rng(11)
    logits = rng.standard_normal((cfg.T, cfg.E)).astype(np.float32)
    er = rng.integers(0, cfg.R, size=cfg.E).astype(np.int32)
    sep, fus = run_both(moe, cfg, logits, er)
    assert_same_route(moe, cfg, sep, fus)


def test_fused_full_path_two_hop_output(moe):
    """The whole two-hop path with the fused front end gives the same output bits."""
    cfg = W.CONFIGS["c5"].with_(T=4096)
    logits = W.make_logits(cfg, 1)
    er = W.expert_home_rank(cfg)
    sep, fus = run_both(moe, cfg, logits, er)
    x = W.make_activations(cfg, 1).cuda()
    for dc in (sep, fus):
        moe.pack(x, dc.layout, dc.packed, dc.packed_hop1)
        dc.combine()
    assert torch.equal(sep.out.view(torch.int16), fus.out.view(torch.int16))
    assert moe.get_status() == 0


# ---- the one-launch front end for any replica map (moe_route_assign_layout) ----
def run_one_launch(moe, cfg, logits, rm):
    rpg = max(cfg.ranks_per_group, 1)
    tpr = -(-cfg.T // cfg.R) if cfg.T else 1
    lg = to_dev(logits)
    mk = lambda: moe.DispatchCombine(cfg.T, cfg.H, cfg.E, cfg.k, cfg.R, to_dev(rm.replica_offsets),
                                     to_dev(rm.replica_slots), to_dev(rm.slot_rank), cfg.mode, tpr, rpg,
                                     cfg.n_groups, cfg.groups_per_token, dtype=torch.bfloat16)
    sep, one = mk(), mk()
    sep.route(lg)
    one.topk_idx.fill_(-7)
    one.expert_slot.fill_(-7)
    one.route_one_launch(lg)
    return sep, one


def assert_same_front(moe, cfg, sep, one):
    assert_same_route(moe, cfg, sep, one)
    assert torch.equal(sep.expert_slot, one.expert_slot)
    assert torch.equal(sep.expert_rank, one.expert_rank)


@pytest.mark.parametrize("name,mode", [("c1", W.DEDUP), ("c1", W.PER_PICK), ("c2", W.DEDUP),
                                       ("c3", W.DEDUP), ("c3", W.PER_PICK), ("c5", W.TWO_HOP),
                                       ("c4", W.DEDUP)])
def test_one_launch_front_matches_separate_calls(moe, name, mode):
    cfg = W.CONFIGS[name].with_(mode=mode)
    logits = W.make_logits(cfg, 2)
    rm = W.make_replica_map(cfg, 0)
    sep, one = run_one_launch(moe, cfg, logits, rm)
    assert_same_front(moe, cfg, sep, one)
    idx, _ = oracle.route_topk(logits, cfg.k, cfg.n_groups, cfg.groups_per_token)
    counts = oracle.demand_hist(idx, cfg.E)
    slot, er, act = oracle.replica_assign(counts, rm.replica_offsets, rm.replica_slots, rm.slot_rank, cfg.R)
    assert np.array_equal(one.expert_slot.cpu().numpy(), slot)
    assert np.array_equal(one.rank_active.cpu().numpy(), act)


@pytest.mark.parametrize("T,E,k,R,mode,rpg,extra", [(1, 8, 2, 4, W.DEDUP, 1, 4), (77, 40, 3, 8, W.DEDUP, 1, 13),
                                                    (300, 1024, 16, 64, W.PER_PICK, 1, 200),
                                                    (513, 96, 6, 12, W.TWO_HOP, 3, 30),
                                                    (2000, 64, 8, 1, W.DEDUP, 1, 0),
                                                    (140000, 64, 2, 8, W.DEDUP, 1, 16)])
def test_one_launch_front_edges(moe, T, E, k, R, mode, rpg, extra):
    """Ties in the logits, redundant replicas on random ranks, a single rank,
    the widest experts and picks, and chunks of two tiles."""
    cfg = W.Config("edge", "edge", T=T, R=R, H=64, dtype="bf16", E=E, k=k, mode=mode,
                   ranks_per_group=rpg if mode == W.TWO_HOP else 0)
    rng = np.random.default_rng(T + E + k)
    logits = (rng.integers(-3, 4, size=(T, E)) * 0.5).astype(np.float32)
    # one replica per expert plus `extra` redundant ones, slots spread over the ranks
    homes = rng.integers(0, R, size=E)
    more = rng.integers(0, E, size=extra)
    slots_of = [[e] for e in range(E)]
    slot_rank = list(homes)
    for i, e in enumerate(more):
        slots_of[e].append(E + i)
        slot_rank.append(int(rng.integers(0, R)))
    off = np.cumsum([0] + [len(s) for s in slots_of]).astype(np.int32)
    rm = W.ReplicaMap(off, np.array([s for ss in slots_of for s in ss], np.int32),
                      np.array(slot_rank, np.int32))
    sep, one = run_one_launch(moe, cfg, logits, rm)
    assert_same_front(moe, cfg, sep, one)
    # and against the oracle (the separate calls share the greedy's device code)
    idx, _ = oracle.route_topk(logits, k)
    counts = oracle.demand_hist(idx, E)
    slot, er, act = oracle.replica_assign(counts, rm.replica_offsets, rm.replica_slots, rm.slot_rank, R)
    assert np.array_equal(one.expert_slot.cpu().numpy(), slot)
    assert np.array_equal(one.expert_rank.cpu().numpy(), er)
    assert np.array_equal(one.rank_active.cpu().numpy(), act)


def test_one_launch_front_zero_tokens(moe):
    cfg = W.CONFIGS["c1"].with_(T=0)
    rm = W.make_replica_map(W.CONFIGS["c1"], 0)
    sep, one = run_one_launch(moe, cfg, np.zeros((0, cfg.E), np.float32), rm)
    assert moe.get_status() == 0
    assert torch.equal(sep.counts, one.counts)
    assert torch.equal(sep.expert_slot, one.expert_slot)
    assert torch.equal(sep.rank_active, one.rank_active)
    assert int(one.layout.num_rows.item()) == 0


def test_one_launch_front_bounded_barrier(moe):
    """A block that never arrives at the first grid barrier: the others' waits
    run out and report MOE_ERR_TIMEOUT; the next call is correct."""
    cfg = W.CONFIGS["c2"]
    rm = W.make_replica_map(cfg, 0)
    logits = W.make_logits(cfg, 0)
    moe.debug_set_wait(20_000_000, 1)
    try:
        run_one_launch(moe, cfg, logits, rm)
        assert moe.get_status() == 4
    finally:
        moe.debug_set_wait(0, -1)
    sep, one = run_one_launch(moe, cfg, logits, rm)
    assert_same_front(moe, cfg, sep, one)
