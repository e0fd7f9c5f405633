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
