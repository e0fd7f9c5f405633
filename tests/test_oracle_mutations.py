"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that
the pins catch every one of them.  This is what makes the pins worth trusting:
a dropped term, a wrong sign or index, or a flipped tie rule fails a pin."""
import numpy as np
import pytest

import oracle
import pins


def _route_ascending(logits, k, n_groups=0, groups_per_token=0, renormalize=False):
    idx, w = oracle.route_topk(-np.asarray(logits, np.float32), k, n_groups, groups_per_token, renormalize)
    p = oracle.softmax(logits)
    return idx, np.take_along_axis(p, idx.astype(np.int64), 1)


def _route_high_tie(logits, k, n_groups=0, groups_per_token=0, renormalize=False):
    lg = np.asarray(logits, np.float32)[:, ::-1]
    idx, w = oracle.route_topk(lg, k, n_groups, groups_per_token, renormalize)
    idx = (lg.shape[1] - 1 - idx).astype(np.int32)
    p = oracle.softmax(logits)
    return idx, np.take_along_axis(p, idx.astype(np.int64), 1)


def _route_topk_softmax(logits, k, n_groups=0, groups_per_token=0, renormalize=False):
    # softmax over the k picks only (a dropped normalisation term)
    idx, w = oracle.route_topk(logits, k, n_groups, groups_per_token, True)
    return idx, w


def _route_group_sum(logits, k, n_groups=0, groups_per_token=0, renormalize=False):
    lg = np.asarray(logits, np.float32)
    T, E = lg.shape
    if not (groups_per_token and groups_per_token < n_groups):
        return oracle.route_topk(lg, k)
    gs = E // n_groups
    score = lg.astype(np.float64).reshape(T, n_groups, gs).sum(axis=2)
    keep = np.zeros((T, n_groups), bool)
    np.put_along_axis(keep, np.argsort(-score, axis=1, kind="stable")[:, :groups_per_token], True, axis=1)
    cand = np.where(np.repeat(keep, gs, axis=1), lg, -np.inf)
    idx = np.argsort(-cand, axis=1, kind="stable")[:, :k].astype(np.int32)
    return idx, np.take_along_axis(oracle.softmax(lg), idx.astype(np.int64), 1)


@pytest.mark.parametrize("mutant", [_route_ascending, _route_high_tie, _route_topk_softmax])
def test_route_mutants_caught(mutant):
    with pytest.raises(AssertionError):
        pins.check_route_brute(mutant)
        pins.check_route_special(mutant)


def test_group_score_by_sum_caught():
    with pytest.raises(AssertionError):
        pins.check_route_groups(_route_group_sum)


def _assign_high_rank_tie(counts, off, slots, sr, R):
    # ties on the activated count go to the HIGHER rank
    E = len(counts)
    act = np.zeros(R, np.int64)
    es, er = np.full(E, -1, np.int32), np.full(E, -1, np.int32)
    for e in range(E):
        if counts[e]:
            s = min(slots[off[e]:off[e + 1]], key=lambda s: (act[sr[s]], -sr[s], s))
            es[e], er[e] = s, sr[s]
            act[sr[s]] += 1
    return es, er, act


def _assign_token_count(counts, off, slots, sr, R):
    # balance demand (token counts) instead of activated experts
    E = len(counts)
    load = np.zeros(R, np.int64)
    act = np.zeros(R, np.int64)
    es, er = np.full(E, -1, np.int32), np.full(E, -1, np.int32)
    for e in range(E):
        if counts[e]:
            s = min(slots[off[e]:off[e + 1]], key=lambda s: (load[sr[s]], sr[s], s))
            es[e], er[e] = s, sr[s]
            load[sr[s]] += counts[e]
            act[sr[s]] += 1
    return es, er, act


@pytest.mark.parametrize("mutant", [_assign_high_rank_tie, _assign_token_count])
def test_assign_mutants_caught(mutant):
    with pytest.raises(AssertionError):
        pins.check_assign_hand(mutant)


def _layout_unstable(idx, w, er, tpr, R, mode, ranks_per_group=0):
    L = oracle.build_layout(idx, w, er, tpr, R, mode, ranks_per_group)
    L = dict(L)
    off = L["rank_offsets"]
    rt = L["row_token"].copy()
    for d in range(R):                     # reverse each destination segment
        rt[off[d]:off[d + 1]] = rt[off[d]:off[d + 1]][::-1]
    L["row_token"] = rt
    return L


def _layout_no_dedup(idx, w, er, tpr, R, mode, ranks_per_group=0):
    return oracle.build_layout(idx, w, er, tpr, R, 0 if mode == 1 else mode, ranks_per_group)


@pytest.mark.parametrize("mutant", [_layout_unstable, _layout_no_dedup])
def test_layout_mutants_caught(mutant):
    with pytest.raises(AssertionError):
        pins.check_layout_brute(mutant)


def _combine_drop_last(y, token_rows, coef, tokens=None):
    tr = np.asarray(token_rows).copy()
    last = (tr >= 0).sum(axis=1) - 1
    tr[np.arange(tr.shape[0]), last] = -1
    return oracle.combine(y, tr, coef, tokens)


def _combine_transposed(y, token_rows, coef, tokens=None):
    # coefficient of the token instead of the row (an index mix-up)
    tr = np.asarray(token_rows)
    c = np.asarray(coef, np.float64)
    c2 = c[np.minimum(np.arange(c.shape[0]), tr.shape[0] - 1)]
    return oracle.combine(y, tr, c2, tokens)


@pytest.mark.parametrize("mutant", [_combine_drop_last, _combine_transposed])
def test_combine_mutants_caught(mutant):
    with pytest.raises(AssertionError):
        pins.check_combine(mutant, oracle.build_layout)


def test_two_hop_without_wire_rounding_caught():
    def mutant(y2, L, coef, wire_fmt, tokens=None):
        return oracle.combine_two_hop(y2, L, coef, "f32" if wire_fmt == "bf16" else wire_fmt, tokens)
    with pytest.raises(AssertionError):
        pins.check_combine_two_hop(mutant, oracle.build_layout, oracle.round_to)


def test_round_half_away_caught():
    def mutant(x, fmt):
        r = oracle.round_to(x, fmt)
        q = oracle.ulp(x, fmt)
        tie = np.abs(np.abs(np.asarray(x, np.float64) - r) - q / 2) == 0
        return np.where(tie, np.sign(x) * (np.abs(r) + q * (np.abs(r) < np.abs(x))), r)
    with pytest.raises(AssertionError):
        pins.check_round_to(mutant)


def test_gini_without_mean_normalisation_caught():
    def mutant(x):
        x = np.asarray(x, np.float64)
        n = x.shape[0]
        return float(np.abs(x[:, None] - x[None, :]).sum() / (2.0 * n * n)) if x.sum() else 0.0
    with pytest.raises(AssertionError):
        pins.check_gini(mutant)


def test_token_balanced_listed_order_caught():
    # deals tokens in the listed order instead of ascending slot id
    def mutant(counts, off, slots, sr, R, S):
        st = np.zeros(S, np.int64)
        act = np.zeros(R, np.int64)
        for e in range(len(counts)):
            ls = [int(s) for s in slots[off[e]:off[e + 1]]]
            for i, s in enumerate(ls):
                st[s] = counts[e] // len(ls) + (1 if i < counts[e] % len(ls) else 0)
                act[sr[s]] += st[s] > 0
        return st, act
    with pytest.raises(AssertionError):
        pins.check_token_balanced(mutant)


def test_placement_ignoring_affinity_caught():
    def mutant(C, counts, R):
        return oracle.correlated_placement(np.zeros_like(C), counts, R)
    with pytest.raises(AssertionError):
        pins.check_placement(mutant)


def _opt_zero(counts, off, slots, sr, R):
    return 0


def _opt_max_over_choices(counts, off, slots, sr, R):
    # the worst choice instead of the best
    import itertools
    active = [e for e in range(len(counts)) if counts[e] > 0]
    ch = [sorted({int(sr[s]) for s in slots[off[e]:off[e + 1]]}) for e in active]
    return max((int(np.bincount(np.asarray(p, np.int64), minlength=R).max()) for p in itertools.product(*ch)),
               default=0)


def _opt_first_replica(counts, off, slots, sr, R):
    # no choice at all: every active expert on its first listed replica
    load = np.zeros(R, np.int64)
    for e in range(len(counts)):
        if counts[e] > 0:
            load[sr[slots[off[e]]]] += 1
    return int(load.max())


def _opt_counting_bound(counts, off, slots, sr, R):
    return -(-int(np.count_nonzero(counts)) // R)


def _opt_counts_inactive(counts, off, slots, sr, R):
    # inactive experts treated as active
    return oracle.optimal_max_active(np.ones(len(counts), np.int64), off, slots, sr, R)


def _opt_slot_as_rank(counts, off, slots, sr, R):
    # the slot id taken for the rank
    return oracle.optimal_max_active(counts, off, slots, np.arange(int(np.max(slots)) + 1) % max(R, 1), R)


@pytest.mark.parametrize("mutant", [_opt_zero, _opt_max_over_choices, _opt_first_replica,
                                    _opt_counting_bound, _opt_counts_inactive, _opt_slot_as_rank])
def test_optimal_max_active_mutants_caught(mutant):
    with pytest.raises(AssertionError):
        pins.check_optimal_max_active(mutant, oracle.replica_assign)
