"""The oracle against numbers the pages print (no GPU)."""
import math

import numpy as np

import oracle
import pins
import workloads as W


def test_payload_example_bytes_and_link_times():
    g = pins.golden("p1_payload_example.json")
    R, Tr, H, b = g["gpus"], g["tokens_per_gpu"], g["hidden"], g["elem_bytes"]
    # one-hop dispatch: each local token goes to one destination (top-1 routing)
    cfg = W.CONFIGS["c1"].with_(k=1)
    logits = W.make_logits(cfg, seed=0)
    idx, w = oracle.route_topk(logits, 1)
    er = W.expert_home_rank(cfg)
    L = oracle.build_layout(idx, w, er, Tr, R, oracle.DEDUP)
    sent = oracle.dispatch_bytes_per_rank(L["send_counts"], H, b)
    assert sent.tolist() == [g["alltoall_bytes_per_gpu"]] * R          # 256 KB
    ag = oracle.allgather_bytes_per_rank(Tr, R, H, b)
    assert ag == g["allgather_bytes_per_gpu"]                            # 2 MB
    assert ag // g["alltoall_bytes_per_gpu"] == g["allgather_over_alltoall"]
    # ideal link times at 600 GB/s (decimal KB/MB in the page's time figures)
    bw = g["link_GBps"]
    assert round(oracle.link_time_us(256e3, bw), 1) == g["alltoall_us_about"]
    assert abs(oracle.link_time_us(2e6, bw) - g["allgather_us_about"]) < 0.5
    assert round(oracle.link_time_us(g["difference_MB"] * 1e6, bw), 1) == g["difference_us_about"]
    assert math.isclose(g["fixed_cost_us"] * 1e-6 * bw * 1e9 / 1e6, g["crossover_MB_about"])


def test_payload_example_top2_dedup_between_one_and_two_sends():
    cfg = W.CONFIGS["c1"]
    g = pins.golden("p1_payload_example.json")
    logits = W.make_logits(cfg, seed=0)
    idx, w = oracle.route_topk(logits, cfg.k)
    er = W.expert_home_rank(cfg)
    one = g["alltoall_bytes_per_gpu"]
    dd = oracle.build_layout(idx, w, er, cfg.tokens_per_rank, cfg.R, oracle.DEDUP)
    pp = oracle.build_layout(idx, w, er, cfg.tokens_per_rank, cfg.R, oracle.PER_PICK)
    sd = oracle.dispatch_bytes_per_rank(dd["send_counts"], cfg.H, cfg.elem_bytes)
    sp = oracle.dispatch_bytes_per_rank(pp["send_counts"], cfg.H, cfg.elem_bytes)
    assert np.all(sp == 2 * one)
    assert np.all((sd >= one) & (sd <= 2 * one))


def test_own_rank_share_uniform_eight_ranks():
    g = pins.golden("p2_own_rank_share.json")
    R = g["gpus"]
    cfg = W.CONFIGS["c1"].with_(T=R * 4096)
    logits = W.make_logits(cfg, seed=3)
    idx, _ = oracle.route_topk(logits, cfg.k)
    share = oracle.own_rank_share(idx, W.expert_home_rank(cfg), cfg.T // R)
    p = g["own_share"]
    sigma = math.sqrt(p * (1 - p) / (cfg.T * cfg.k))
    assert abs(share - p) < 5 * sigma, (share, p, sigma)


def test_dedup_and_correlated_placement_shrink_rows():
    cfg = W.CONFIGS["c3"]
    logits = W.make_logits(cfg, seed=0)
    idx, w = oracle.route_topk(logits, cfg.k)
    rows = {}
    for placement in ("block", "roundrobin"):
        er = W.expert_home_rank(cfg.with_(placement=placement))
        for mode in (oracle.PER_PICK, oracle.DEDUP):
            L = oracle.build_layout(idx, w, er, cfg.tokens_per_rank, cfg.R, mode)
            rows[placement, mode] = int(L["num_rows"])
    Tk = cfg.T * cfg.k
    assert rows["block", oracle.PER_PICK] == rows["roundrobin", oracle.PER_PICK] == Tk
    # single-send never exceeds per-pick; correlated placement sends fewer rows
    assert rows["block", oracle.DEDUP] < rows["roundrobin", oracle.DEDUP] <= Tk
