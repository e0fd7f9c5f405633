"""GPU parity: router top-k, demand histogram and METRO assignment against the
CPU oracle, through the C ABI (bit-exact indices and counts, derived bounds
on the weights)."""
import numpy as np
import pytest
import torch

import oracle
import pins
import workloads as W
from gpu_util import assert_weights, moe, to_dev  # noqa: F401

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", sorted(W.CONFIGS))
def test_route_full_size_configs(moe, name):
    cfg = W.CONFIGS[name]
    logits = W.make_logits(cfg, seed=0)
    idx_d, w_d = moe.route_topk(to_dev(logits), cfg.k, cfg.n_groups, cfg.groups_per_token)
    assert moe.get_status() == 0
    idx, w = oracle.route_topk(logits, cfg.k, cfg.n_groups, cfg.groups_per_token)
    assert np.array_equal(idx_d.cpu().numpy(), idx)
    assert_weights(w_d.cpu().numpy(), w, logits, idx)


@pytest.mark.parametrize("T,E,k,G,gpt,renorm,ties", [
    (1, 64, 2, 0, 0, 0, False),
    (33, 40, 3, 0, 0, 0, False),        # E not a multiple of 32, ragged token count
    (300, 1024, 16, 0, 0, 0, False),    # largest E and k
    (77, 6, 6, 0, 0, 0, False),         # k = E
    (64, 1, 1, 0, 0, 0, False),
    (500, 256, 8, 0, 0, 1, False),      # renormalised weights
    (1000, 64, 8, 0, 0, 0, True),       # many exact ties
    (700, 128, 8, 8, 4, 0, False),      # group-limited, the two-hop config's shape
    (300, 96, 5, 32, 3, 0, True),       # 32 groups of 3, ties
    (129, 32, 4, 4, 1, 0, True),
    (257, 256, 8, 4, 2, 0, True),       # groups of 64: two whole slots each
    (257, 256, 8, 8, 3, 0, True),       # groups of 32: one slot each
    (100, 32, 2, 32, 2, 0, True),       # groups of one expert
    (100, 64, 4, 32, 3, 0, True),       # groups of 2
    (90, 40, 3, 5, 2, 0, True),         # groups of 8, the last slot partly empty
])
def test_route_edges(moe, T, E, k, G, gpt, renorm, ties):
    rng = np.random.default_rng(T * 7 + E)
    if ties:
        logits = (rng.integers(-2, 3, size=(T, E)) * 0.5).astype(np.float32)
        logits[::5] = 0.0
        logits[1::7, ::3] = -0.0            # -0 and +0 tie like the floats compare
    else:
        logits = rng.standard_normal((T, E)).astype(np.float32) * 3
    idx_d, w_d = moe.route_topk(to_dev(logits), k, G, gpt, bool(renorm))
    assert moe.get_status() == 0
    idx, w = oracle.route_topk(logits, k, G, gpt, bool(renorm))
    assert np.array_equal(idx_d.cpu().numpy(), idx)
    assert_weights(w_d.cpu().numpy(), w, logits, idx, renormalize=bool(renorm))


@pytest.mark.parametrize("E,k,G,gpt,renorm,ties", [
    (64, 6, 0, 0, 0, False),            # the training workload's shape
    (64, 8, 0, 0, 1, True),
    (128, 1, 0, 0, 0, False),
    (128, 8, 0, 0, 0, True),
    (256, 8, 0, 0, 0, False),           # the prefill workload's shape
    (256, 8, 0, 0, 1, True),
    (256, 3, 0, 0, 0, True),
    (256, 7, 0, 0, 0, False),
    (128, 8, 8, 4, 0, False),           # the two-hop workload's shape: 8 groups, keep 4
    (128, 8, 8, 4, 0, True),
    (256, 8, 4, 2, 1, True),            # groups of 4 chunks
    (64, 6, 16, 5, 0, False),           # groups of one chunk
    (256, 8, 16, 3, 0, True),
    (128, 2, 2, 1, 0, True),
    (256, 8, 32, 4, 0, False),          # 32 groups: not whole chunks, the warp kernel
])
def test_route_per_thread_kernel(moe, E, k, G, gpt, renorm, ties):
    """Large token sets of these shapes (128 tokens per SM and more) take the
    one-thread-per-token kernel; its picks and weights are bit-identical to the
    one-warp-per-token kernel's, which runs on token sets below the threshold
    (2000-token slices of the same logits) and on logits that are not 16-byte
    aligned."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    T = 256 * sms + 77                  # a ragged last block of 32 tokens
    rng = np.random.default_rng(E * 10 + k + G)
    if ties:
        logits = (rng.integers(-2, 3, size=(T, E)) * 0.5).astype(np.float32)
        logits[::5] = 0.0
        logits[1::7, ::3] = -0.0
    else:
        logits = rng.standard_normal((T, E)).astype(np.float32) * 3
    dev = to_dev(logits)
    idx_d, w_d = moe.route_topk(dev, k, G, gpt, bool(renorm))
    assert moe.get_status() == 0
    idx, w = oracle.route_topk(logits, k, G, gpt, bool(renorm))
    idx_h, w_h = idx_d.cpu().numpy(), w_d.cpu().numpy()
    assert np.array_equal(idx_h, idx)
    assert_weights(w_h, w, logits, idx, renormalize=bool(renorm))
    for t0 in range(0, T, 2000):
        i_s, w_s = moe.route_topk(dev[t0:t0 + 2000], k, G, gpt, bool(renorm))
        assert np.array_equal(i_s.cpu().numpy(), idx_h[t0:t0 + 2000])
        assert np.array_equal(w_s.cpu().numpy().view(np.uint32), w_h[t0:t0 + 2000].view(np.uint32))
    flat = torch.empty(T * E + 1, dtype=torch.float32, device="cuda")
    shifted = flat[1:].view(T, E)
    shifted.copy_(dev)
    i_m, w_m = moe.route_topk(shifted, k, G, gpt, bool(renorm))
    assert moe.get_status() == 0
    assert np.array_equal(i_m.cpu().numpy(), idx_h)
    assert np.array_equal(w_m.cpu().numpy().view(np.uint32), w_h.view(np.uint32))


def test_route_per_thread_kernel_nonfinite(moe):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    lg = np.random.default_rng(5).standard_normal((256 * sms + 3, 256)).astype(np.float32)
    lg[256 * sms + 1, 200] = np.inf     # in the ragged last block
    moe.route_topk(to_dev(lg), 8)
    assert moe.get_status() == 6            # MOE_ERR_BAD_INPUT


def test_route_group_fixtures(moe):
    g = pins.golden("p4_group_limited.json")
    for c in g["cases"]:
        lg = np.asarray([c["logits"]], np.float32)
        idx_d, _ = moe.route_topk(to_dev(lg), c["k"], c["n_groups"], c["groups_per_token"])
        assert idx_d.cpu().numpy()[0].tolist() == c["idx"]


def test_route_nonfinite_logit_reported(moe):
    lg = np.zeros((4, 8), np.float32)
    lg[2, 3] = np.nan
    moe.route_topk(to_dev(lg), 2)
    assert moe.get_status() == 6            # MOE_ERR_BAD_INPUT
    assert moe.get_status() == 0            # read-and-clear


def test_route_zero_tokens(moe):
    idx, w = moe.route_topk(torch.empty((0, 16), dtype=torch.float32, device="cuda"), 2)
    assert idx.shape == (0, 2) and moe.get_status() == 0


@pytest.mark.parametrize("name", sorted(W.CONFIGS))
def test_hist_full_size(moe, name):
    cfg = W.CONFIGS[name]
    idx, _ = oracle.route_topk(W.make_logits(cfg, 0), cfg.k, cfg.n_groups, cfg.groups_per_token)
    c_d = moe.demand_hist(to_dev(idx), cfg.E)
    assert moe.get_status() == 0
    assert np.array_equal(c_d.cpu().numpy(), oracle.demand_hist(idx, cfg.E))


def test_hist_bad_id_and_skew(moe):
    idx = np.zeros((5000, 4), np.int32)          # every pick on expert 0: worst contention
    idx[:, 1:] = np.arange(1, 4)
    idx[17, 2] = 99                               # out of range
    c_d = moe.demand_hist(to_dev(idx), 8)
    assert moe.get_status() == 6
    c = c_d.cpu().numpy()
    assert c[0] == 5000 and c[2] == 4999 and c.sum() == 5000 * 4 - 1
    idx[17, 2] = 2
    idx[4999, 3] = -1                             # negative, in the ragged last pass
    c = moe.demand_hist(to_dev(idx), 8).cpu().numpy()
    assert moe.get_status() == 6
    assert c[3] == 4999 and c.sum() == 5000 * 4 - 1


def _assign_dev(moe, counts, rm_off, rm_slots, slot_rank, R):
    s, r, a = moe.replica_assign(to_dev(np.asarray(counts, np.int32)), to_dev(np.asarray(rm_off, np.int32)),
                                 to_dev(np.asarray(rm_slots, np.int32)), to_dev(np.asarray(slot_rank, np.int32)), R)
    return s.cpu().numpy(), r.cpu().numpy(), a.cpu().numpy()


@pytest.mark.parametrize("name", sorted(W.CONFIGS))
def test_assign_configs(moe, name):
    cfg = W.CONFIGS[name]
    rm = W.make_replica_map(cfg, 0)
    idx, _ = oracle.route_topk(W.make_logits(cfg, 0), cfg.k, cfg.n_groups, cfg.groups_per_token)
    counts = oracle.demand_hist(idx, cfg.E)
    got = _assign_dev(moe, counts, rm.replica_offsets, rm.replica_slots, rm.slot_rank, cfg.R)
    assert moe.get_status() == 0
    ref = oracle.replica_assign(counts, rm.replica_offsets, rm.replica_slots, rm.slot_rank, cfg.R)
    for g, r in zip(got, ref):
        assert np.array_equal(g, r.astype(np.int32))


def test_assign_hand_worked_and_toy(moe):
    g = pins.golden("metro_greedy_hand.json")
    s, r, a = _assign_dev(moe, g["counts"], g["replica_offsets"], g["replica_slots"], g["slot_rank"], g["R"])
    assert s.tolist() == g["expert_slot"] and r.tolist() == g["expert_rank"]
    assert a.tolist() == g["rank_active"]
    gt, counts, off, slots, sr, R = pins.toy_instance()
    _, _, a = _assign_dev(moe, counts, off, slots, sr, R)
    assert int(a.max()) == gt["metro_max_active_per_gpu"]


def test_assign_random_maps_with_ties(moe):
    rng = np.random.default_rng(11)
    for trial in range(40):
        E, R = int(rng.integers(1, 300)), int(rng.integers(1, 65))
        nrep = rng.integers(1, min(R, 40) + 1, size=E)   # up to 40 replicas: two lane rounds
        if trial % 5 == 0:
            nrep[:] = 1
        reps = [rng.choice(R, size=int(n), replace=False) for n in nrep]
        slot_rank = np.concatenate(reps).astype(np.int32)
        S = slot_rank.shape[0]
        perm = rng.permutation(S)                        # slot ids not in expert order
        sr_by_slot = np.empty(S, np.int32)
        sr_by_slot[perm] = slot_rank
        off = np.zeros(E + 1, np.int32)
        off[1:] = np.cumsum(nrep)
        slots = perm.astype(np.int32)
        counts = rng.integers(0, 3, size=E).astype(np.int32)
        got = _assign_dev(moe, counts, off, slots, sr_by_slot, R)
        assert moe.get_status() == 0
        ref = oracle.replica_assign(counts, off, slots, sr_by_slot, R)
        for g, r in zip(got, ref):
            assert np.array_equal(g, r.astype(np.int32)), trial


def _random_map(rng, E, R, max_rep):
    """Replica map with 1..max_rep replicas per expert on distinct random
    ranks; slot ids shuffled so that they are not in expert order."""
    nrep = rng.integers(1, min(R, max_rep) + 1, size=E)
    reps = [rng.choice(R, size=int(n), replace=False) for n in nrep]
    slot_rank = np.concatenate(reps).astype(np.int32)
    S = slot_rank.shape[0]
    perm = rng.permutation(S)
    sr_by_slot = np.empty(S, np.int32)
    sr_by_slot[perm] = slot_rank
    off = np.zeros(E + 1, np.int32)
    off[1:] = np.cumsum(nrep)
    return off, perm.astype(np.int32), sr_by_slot


@pytest.mark.parametrize("R", [1, 5, 8, 9, 16, 17, 32, 33, 64])
def test_assign_small_replica_sets(moe, R):
    """No expert with more than 4 replicas and at most 255 with a choice: the
    one-thread walk, whose per-rank counters are bytes of 64-bit words (one
    word up to 8 ranks, then 2, 4 and 8 words); demand with zeros and ties."""
    rng = np.random.default_rng(100 + R)
    for trial in range(8):
        E = int(rng.integers(1, 400))
        off, slots, sr = _random_map(rng, E, R, 4)
        counts = rng.integers(0, 3, size=E).astype(np.int32)
        got = _assign_dev(moe, counts, off, slots, sr, R)
        assert moe.get_status() == 0
        ref = oracle.replica_assign(counts, off, slots, sr, R)
        for g, r in zip(got, ref):
            assert np.array_equal(g, r.astype(np.int32)), (R, trial)


@pytest.mark.parametrize("n_choice", [255, 256])
def test_assign_choice_count_boundary(moe, n_choice):
    """255 active experts with a choice take the one-thread walk, 256 the warp
    walk; both give the greedy's result."""
    rng = np.random.default_rng(n_choice)
    E, R = 400, 16
    nrep = np.ones(E, np.int64)
    nrep[:n_choice] = 2
    reps = [rng.choice(R, size=int(n), replace=False) for n in nrep]
    sr = np.concatenate(reps).astype(np.int32)
    off = np.zeros(E + 1, np.int32)
    off[1:] = np.cumsum(nrep)
    slots = np.arange(sr.shape[0], dtype=np.int32)
    counts = np.ones(E, np.int32)
    got = _assign_dev(moe, counts, off, slots, sr, R)
    assert moe.get_status() == 0
    ref = oracle.replica_assign(counts, off, slots, sr, R)
    for g, r in zip(got, ref):
        assert np.array_equal(g, r.astype(np.int32))


def test_assign_active_expert_without_replica(moe):
    counts = [1, 2, 0]
    s, r, a = _assign_dev(moe, counts, [0, 1, 1, 2], [0, 1], [0, 1], 2)
    assert moe.get_status() == 6
    assert s.tolist() == [0, -1, -1] and r.tolist() == [0, -1, -1] and a.tolist() == [1, 0]
