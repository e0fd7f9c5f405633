"""Shapes and determinism of the seeded synthetic inputs (no GPU)."""
import numpy as np
import pytest

import oracle
import workloads as W


def test_replica_maps_match_the_configs():
    rm = W.make_replica_map(W.CONFIGS["c1"])
    assert rm.S == 80 and np.bincount(rm.slot_rank).tolist() == [10] * 8
    rm2 = W.make_replica_map(W.CONFIGS["c2"])
    assert rm2.S == 288 and np.bincount(rm2.slot_rank).tolist() == [36] * 8
    for rm_, E in ((rm, 64), (rm2, 256)):
        assert rm_.replica_offsets[-1] == rm_.S and rm_.replica_offsets.shape == (E + 1,)
        for e in range(E):
            ranks = rm_.slot_rank[rm_.replica_slots[rm_.replica_offsets[e]:rm_.replica_offsets[e + 1]]]
            assert len(set(ranks.tolist())) == len(ranks) >= 1     # no two replicas on one rank
    # c2 replicates the 32 experts with the largest bias
    bias = W.expert_bias(W.CONFIGS["c2"], 0)
    reps = np.diff(rm2.replica_offsets)
    assert set(np.nonzero(reps == 2)[0].tolist()) == set(np.argsort(-bias)[:32].tolist())


@pytest.mark.parametrize("name", sorted(W.CONFIGS))
def test_inputs_are_seeded(name):
    cfg = W.CONFIGS[name]
    a = W.make_logits(cfg, seed=11, T=64)
    b = W.make_logits(cfg, seed=11, T=64)
    c = W.make_logits(cfg, seed=12, T=64)
    assert a.dtype == np.float32 and a.shape == (64, cfg.E)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    x = W.make_activations(cfg, seed=11, T=4)
    assert tuple(x.shape) == (4, cfg.H)
    assert cfg.T % cfg.R == 0


def test_clustered_logits_in_cluster_share():
    cfg = W.CONFIGS["c3"]
    logits = W.make_logits(cfg, seed=0)
    idx, _ = oracle.route_topk(logits, cfg.k)
    # the home cluster is the cluster with the raised logits
    per = cfg.E // cfg.clusters
    blk = logits.reshape(cfg.T, cfg.clusters, per).mean(axis=2)
    home = blk.argmax(axis=1)
    share = float(np.mean(idx // per == home[:, None]))
    assert 0.35 < share < 0.45, share


def test_sample_indices():
    s = W.sample_indices(1000, 50, seed=1)
    assert s[0] == 0 and s[-1] == 999 and len(s) == 50 and np.all(np.diff(s) > 0)
