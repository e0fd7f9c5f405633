"""The CPU oracle against its pins (no GPU)."""
import numpy as np
import pytest

import oracle
import pins


def test_round_to_matches_library_casts():
    pins.check_round_to(oracle.round_to)


def test_route_brute_force_with_ties():
    pins.check_route_brute(oracle.route_topk)


def test_route_library_topk_softmax():
    pins.check_route_library(oracle.route_topk)


def test_route_special_cases():
    pins.check_route_special(oracle.route_topk)


def test_route_group_limited():
    pins.check_route_groups(oracle.route_topk)


def test_hist_counter():
    pins.check_hist(oracle.demand_hist)


def test_assign_hand_worked():
    pins.check_assign_hand(oracle.replica_assign)


def test_assign_page_toy_example():
    pins.check_assign_toy(oracle.replica_assign, oracle.token_balanced_active)


def test_assign_closed_forms():
    pins.check_assign_closed_forms(oracle.replica_assign)


def test_assign_vs_brute_force_optimum():
    gap = pins.check_assign_brute(oracle.replica_assign, oracle.optimal_max_active)
    # context, not a bound: the page's greedy was within 10.9% of the optimum on its workload
    assert 0.0 <= gap < 1.0


def test_layout_brute_force_all_modes():
    pins.check_layout_brute(oracle.build_layout)


def test_layout_invariants():
    pins.check_layout_invariants(oracle.build_layout)


def test_combine_brute_and_conservation():
    pins.check_combine(oracle.combine, oracle.build_layout)


def test_combine_two_hop_brute():
    pins.check_combine_two_hop(oracle.combine_two_hop, oracle.build_layout, oracle.round_to)


def test_pack_is_row_gather():
    rng = np.random.default_rng(0)
    x = rng.integers(0, 2 ** 16, size=(9, 5), dtype=np.uint16)
    rt = np.array([3, 3, 0, 8, 1], np.int32)
    p = oracle.pack(x, rt)
    for i, t in enumerate(rt):
        assert p[i].tobytes() == x[t].tobytes()
    assert oracle.pack(x, rt, rows=[4, 0]).tolist() == [x[1].tolist(), x[3].tolist()]


def test_ulp():
    assert oracle.ulp(np.array([1.0, 1.5, 2.0]), "bf16").tolist() == [2.0 ** -7, 2.0 ** -7, 2.0 ** -6]
    assert oracle.ulp(np.array([1e-7]), "f16").tolist() == [2.0 ** -24]


def test_gini_closed_forms():
    pins.check_gini(oracle.gini)


def test_dispatch_stats_hand_worked():
    pins.check_dispatch_stats(oracle.dispatch_stats)


def test_token_balanced_split():
    pins.check_token_balanced(oracle.token_balanced_split)


def test_uniform_own_row_share_single_pick():
    """With top-1 routing on E/R experts per rank, the own-rank row share is the
    own-rank pick share: 1/R in expectation (the 12.5% of one node of 8)."""
    import workloads as W
    cfg = W.CONFIGS["c1"].with_(T=8 * 4096, k=1)
    idx, w = oracle.route_topk(W.make_logits(cfg, seed=5), 1)
    L = oracle.build_layout(idx, w, W.expert_home_rank(cfg), cfg.T // 8, 8, oracle.DEDUP)
    share = oracle.dispatch_stats(oracle.demand_hist(idx, cfg.E), L["send_counts"])["own_rank_row_share"]
    assert abs(share - 0.125) < 5 * (0.125 * 0.875 / cfg.T) ** 0.5


def test_coselection_brute_force():
    pins.check_coselection(oracle.coselection)


def test_correlated_placement_closed_forms_and_brute_force():
    pins.check_placement(oracle.correlated_placement)


def test_derived_placement_shrinks_dedup_rows():
    """On the clustered training workload, the placement derived from the
    co-selection counts sends fewer dedup rows than round-robin placement
    (the direction of the summary's 'removes up to 58% of dispatched rows')."""
    import workloads as W
    cfg = W.CONFIGS["c3"]
    idx, w = oracle.route_topk(W.make_logits(cfg, 0), cfg.k)
    er = oracle.correlated_placement(oracle.coselection(idx, cfg.E), oracle.demand_hist(idx, cfg.E), cfg.R)
    rows = {}
    for name, rank in (("derived", er), ("roundrobin", W.expert_home_rank(cfg.with_(placement="roundrobin"))),
                       ("block", W.expert_home_rank(cfg))):
        rows[name] = int(oracle.build_layout(idx, w, rank, cfg.tokens_per_rank, cfg.R, oracle.DEDUP)["num_rows"])
    assert rows["derived"] < rows["roundrobin"]
    assert rows["derived"] <= 1.02 * rows["block"]      # close to the planted clusters


def test_optimal_max_active_pinned():
    # the greedy is strictly worse than the optimum on some random tiny maps,
    # as the page's "within 10.9%" implies it can be
    assert pins.check_optimal_max_active(oracle.optimal_max_active, oracle.replica_assign) > 0
