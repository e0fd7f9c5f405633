"""Host-side logic of the package that needs no GPU."""
import pytest

import workloads as W
from combine_router_softmax_02_b200.path import token_ranges


@pytest.mark.parametrize("T,chunks", [(0, 8), (1, 8), (7, 8), (8, 8), (9, 8), (65536, 8), (1000, 3),
                                      (5, 1), (100, 1000)])
def test_token_ranges_cover_in_order(T, chunks):
    r = token_ranges(T, chunks)
    assert all(b > a for a, b in r)                      # non-empty
    flat = [t for a, b in r for t in range(a, b)]
    assert flat == list(range(T))                        # contiguous, in order, no overlap
    assert len(r) == (min(chunks, T) if T else 0)
    if r:
        sizes = [b - a for a, b in r]
        assert max(sizes) - min(sizes) <= 1


def test_step_trace_structure():
    """bench's step trace: replicas of active experts only, rows and bytes per
    rank, and the dispatch/combine matrices, from a hand-made tiny layout."""
    import numpy as np
    import bench
    import workloads as W
    cfg = W.CONFIGS["c1"].with_(R=2, E=4, k=2, T=4)
    counts = np.array([3, 0, 4, 1])
    slot = np.array([0, -1, 5, 3])
    rank = np.array([0, -1, 1, 1])
    active = np.array([1, 2])
    offsets = np.array([0, 3, 7])                # rank 0: 3 rows, rank 1: 4 rows
    send = np.array([[2, 0], [1, 4]])            # rows by (source rank, destination rank)
    tr = bench.make_trace(cfg, counts, slot, rank, active, offsets, send,
                          calls=[("route_topk", 0.0, 5.0), ("pack", 5.0, 2.5)])
    b = cfg.H * cfg.elem_bytes
    assert [r["expert"] for r in tr["replicas"]] == [0, 2, 3]
    assert tr["replicas"][1] == {"expert": 2, "demand": 4, "slot": 5, "rank": 1}
    assert [d["rows"] for d in tr["rank_detail"]] == [3, 4]
    assert tr["rank_detail"][1]["recv_bytes"] == 4 * b
    disp, comb = tr["collectives"]
    assert disp["bytes"] == comb["bytes"] == 7 * b
    assert disp["bytes_src_dst"] == [[2 * b, 0], [1 * b, 4 * b]]
    assert comb["bytes_src_dst"] == [[2 * b, 1 * b], [0, 4 * b]]  # combine reverses the direction
    # the rows each rank receives equal the column sums of the send matrix
    assert [sum(col) for col in zip(*disp["bytes_src_dst"])] == [d["recv_bytes"] for d in tr["rank_detail"]]
    assert tr["calls_us"][1] == {"call": "pack", "start": 5.0, "duration": 2.5}


def test_step_trace_two_hop_groups():
    """The two-hop trace adds the hop-1 exchange (rows per group) before the
    rank-level dispatch, and reports each rank's group."""
    import numpy as np
    import bench
    import workloads as W
    cfg = W.CONFIGS["c5"].with_(R=4, ranks_per_group=2, E=8, k=2, T=6)
    b = cfg.H * cfg.elem_bytes
    tr = bench.make_trace(cfg, np.ones(8, int), np.arange(8), np.arange(8) % 4, np.array([2, 2, 2, 2]),
                          np.array([0, 2, 4, 7, 9]), np.ones((4, 4), int), group_offsets=np.array([0, 5, 8]))
    hop1 = tr["collectives"][0]
    assert hop1["name"].startswith("dispatch hop 1")
    assert hop1["bytes"] == 8 * b and hop1["group_bytes"] == [5 * b, 3 * b]
    assert [d["group"] for d in tr["rank_detail"]] == [0, 0, 1, 1]
    assert "calls_us" not in tr


@pytest.mark.parametrize("name", ["c4", "c5"])
def test_parallel_oracle_matches_serial(name):
    """The all-cores CPU baseline runs the same oracle functions over disjoint
    chunks in spawned processes: its packed rows and combined tokens equal a
    single-process pass over the same sample."""
    import numpy as np
    import bench
    import oracle
    import workloads as W
    cfg = W.CONFIGS[name]
    sub, logits, x32, rm = bench.oracle_sample(cfg, 192, 0)
    par = bench.ParallelOracle(sub, logits, x32, 2)
    try:
        rows = par.step(rm)
        P = np.array(bench._shm_array(*par.p)[:rows])
        out = np.array(bench._shm_array(*par.out))
        idx, w = oracle.route_topk(logits, sub.k, sub.n_groups, sub.groups_per_token)
        counts = oracle.demand_hist(idx, sub.E)
        _, er, _ = oracle.replica_assign(counts, rm.replica_offsets, rm.replica_slots, rm.slot_rank, sub.R)
        L = oracle.build_layout(idx, w, er, -(-sub.T // sub.R), sub.R, sub.mode, max(sub.ranks_per_group, 1))
        assert rows == int(L["num_rows"])
        if sub.mode == W.TWO_HOP:
            p2 = oracle.pack(oracle.pack(x32, L["hop1_row_token"]), L["hop2_src_row"])
            ref, _ = oracle.combine_two_hop(p2, L, L["row_coef"], sub.dtype)
        else:
            p2 = oracle.pack(x32, L["row_token"])
            ref = oracle.combine(p2, L["token_rows"], L["row_coef"])
        assert np.array_equal(P, p2)
        assert np.array_equal(out, ref)
    finally:
        for shm in bench._SHM.values():  # this process's own views of the blocks
            shm.close()
        bench._SHM.clear()
        par.close()


def test_bench_extra_runs_are_well_formed():
    """Every workload the default bench run measures beside the headline names
    a config, applies only Config fields, carries a unique label, and asks for
    a CUDA graph only together with the one-launch front end."""
    import bench
    labels = [r[0] for r in bench.EXTRA_RUNS]
    assert len(labels) == len(set(labels))
    for label, name, over, fused, graph, e2e in bench.EXTRA_RUNS:
        assert name in W.CONFIGS, label
        cfg = W.CONFIGS[name].with_(**over)     # raises on an unknown field
        assert cfg.name == name
        assert not graph or fused, label
        assert isinstance(e2e, bool)


def test_bench_steps_for_bounds():
    import bench
    assert bench.steps_for(0.0, 1.0, 20) == 20
    assert bench.steps_for(2.6, 1.0, 20) == 385      # ceil(1000 / 2.6)
    assert bench.steps_for(0.001, 1.0, 20, cap=100000) == 100000
    assert bench.steps_for(5000.0, 1.0, 20) == 20
