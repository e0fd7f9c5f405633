"""GPU parity: dispatch statistics and the token-balanced comparison policy
against the CPU oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import pins
import workloads as W
from gpu_util import moe, to_dev  # noqa: F401

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", sorted(W.CONFIGS))
def test_dispatch_stats_configs(moe, name):
    cfg = W.CONFIGS[name]
    rm = W.make_replica_map(cfg, 0)
    idx, w = oracle.route_topk(W.make_logits(cfg, 0), cfg.k, cfg.n_groups, cfg.groups_per_token)
    counts = oracle.demand_hist(idx, cfg.E)
    _, er, _ = oracle.replica_assign(counts, rm.replica_offsets, rm.replica_slots, rm.slot_rank, cfg.R)
    L = oracle.build_layout(idx, w, er, cfg.tokens_per_rank, cfg.R, cfg.mode, max(cfg.ranks_per_group, 1))
    got = moe.dispatch_stats(to_dev(counts.astype(np.int32)), to_dev(L["send_counts"])).cpu().numpy()
    assert moe.get_status() == 0
    ref = oracle.dispatch_stats(counts, L["send_counts"])
    for i, key in enumerate(moe.STAT_NAMES):
        assert math.isclose(got[i], ref[key], rel_tol=1e-13, abs_tol=1e-15), (key, got[i], ref[key])


def test_dispatch_stats_hand_worked(moe):
    got = moe.dispatch_stats(to_dev(np.array([1, 1, 1, 5], np.int32)),
                             to_dev(np.array([[4, 1, 0], [0, 2, 2], [1, 0, 2]], np.int32))).cpu().numpy()
    assert np.allclose(got, [2.5, 8 / 72, 1.25, 8 / 12], rtol=1e-15)
    zero = moe.dispatch_stats(to_dev(np.zeros(4, np.int32)), to_dev(np.zeros((2, 2), np.int32)))
    assert zero.cpu().tolist() == [0.0, 0.0, 0.0, 0.0]


def _tb(moe, counts, off, slots, sr, R):
    st, act = moe.token_balanced_assign(to_dev(np.asarray(counts, np.int32)), to_dev(np.asarray(off, np.int32)),
                                        to_dev(np.asarray(slots, np.int32)), to_dev(np.asarray(sr, np.int32)), R)
    return st.cpu().numpy(), act.cpu().numpy()


def test_token_balanced_configs_and_toy(moe):
    for name in ("c1", "c2"):
        cfg = W.CONFIGS[name]
        rm = W.make_replica_map(cfg, 0)
        idx, _ = oracle.route_topk(W.make_logits(cfg, 0), cfg.k)
        counts = oracle.demand_hist(idx, cfg.E)
        st, act = _tb(moe, counts, rm.replica_offsets, rm.replica_slots, rm.slot_rank, cfg.R)
        rst, ract = oracle.token_balanced_split(counts, rm.replica_offsets, rm.replica_slots, rm.slot_rank,
                                                cfg.R, rm.S)
        assert np.array_equal(st, rst) and np.array_equal(act, ract)
    g, counts, off, slots, sr, R = pins.toy_instance()
    _, act = _tb(moe, counts, off, slots, sr, R)
    assert act.tolist() == [g["token_balanced_active_per_gpu"]] * R
    assert moe.get_status() == 0


def test_token_balanced_random_maps(moe):
    rng = np.random.default_rng(21)
    for trial in range(25):
        E, R = int(rng.integers(1, 200)), int(rng.integers(1, 65))
        nrep = rng.integers(1, min(R, 12) + 1, size=E)
        sr = np.concatenate([rng.choice(R, size=int(n), replace=False) for n in nrep]).astype(np.int32)
        S = sr.shape[0]
        perm = rng.permutation(S).astype(np.int32)
        sr_by = np.empty(S, np.int32)
        sr_by[perm] = sr
        off = np.zeros(E + 1, np.int32)
        off[1:] = np.cumsum(nrep)
        counts = rng.integers(0, 30, size=E).astype(np.int32)
        st, act = _tb(moe, counts, off, perm, sr_by, R)
        rst, ract = oracle.token_balanced_split(counts, off, perm, sr_by, R, S)
        assert np.array_equal(st, rst) and np.array_equal(act, ract), trial
    assert moe.get_status() == 0


def test_metro_activates_no_more_than_token_balance_on_replicated_configs(moe):
    """The page's comparison, on the two configs with redundant replicas: the
    METRO greedy's max activated experts per rank against token balancing."""
    for name in ("c1", "c2"):
        cfg = W.CONFIGS[name]
        rm = W.make_replica_map(cfg, 0)
        idx, _ = oracle.route_topk(W.make_logits(cfg, 0), cfg.k)
        c_d = moe.demand_hist(to_dev(idx), cfg.E)
        _, _, metro = moe.replica_assign(c_d, to_dev(rm.replica_offsets), to_dev(rm.replica_slots),
                                         to_dev(rm.slot_rank), cfg.R)
        _, tb = moe.token_balanced_assign(c_d, to_dev(rm.replica_offsets), to_dev(rm.replica_slots),
                                          to_dev(rm.slot_rank), cfg.R)
        assert int(metro.max()) <= int(tb.max())
        assert int(metro.sum()) <= int(tb.sum())
