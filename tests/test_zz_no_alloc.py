"""moe_build_layout_static: the layout entry point for callers that cannot
allocate device memory (a serving loop whose memory is all reserved at
start-up, or a host framework that only hands over its existing buffers).

It takes its scratch from a fixed device array inside the library instead of
a caller-supplied workspace.  This test calls it through the C ABI, twice in
a row on different workloads (the shared array keeps the previous call's
contents), and checks each result against the regular moe_build_layout with
its own workspace: integer fields bit-exact, coefficients within the layout
tests' bound.  The file is named to be collected last.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from gpu_util import layout_fields, moe, to_dev  # noqa: F401

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
U = 2.0 ** -24


def static_limit() -> int:
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        m = re.search(r"#define\s+MOE_LAYOUT_STATIC_SCRATCH_BYTES\s+\(1u\s*<<\s*(\d+)\)", f.read())
    return 1 << int(m.group(1))


def routed(name):
    cfg = W.CONFIGS[name]
    rm = W.make_replica_map(cfg, 0)
    idx, w = oracle.route_topk(W.make_logits(cfg, 0), cfg.k, cfg.n_groups, cfg.groups_per_token)
    counts = oracle.demand_hist(idx, cfg.E)
    _, er, _ = oracle.replica_assign(counts, rm.replica_offsets, rm.replica_slots, rm.slot_rank, cfg.R)
    return cfg, to_dev(idx), to_dev(w.astype(np.float32)), to_dev(er)


def static_layout(moe, cfg, idx, w, er):
    rpg = max(cfg.ranks_per_group, 1)
    L = moe.Layout(cfg.T, cfg.k, cfg.E, cfg.R, cfg.mode, cfg.tokens_per_rank, rpg)
    rc = moe.lib().moe_build_layout_static(idx.data_ptr(), w.data_ptr(), er.data_ptr(), cfg.T,
                                           cfg.tokens_per_rank, cfg.k, cfg.E, cfg.R, rpg, cfg.mode,
                                           ctypes.byref(L.struct), torch.cuda.current_stream().cuda_stream)
    assert rc == 0, moe.status_string(rc)
    return L


def regular_layout(moe, cfg, idx, w, er):
    rpg = max(cfg.ranks_per_group, 1)
    L = moe.Layout(cfg.T, cfg.k, cfg.E, cfg.R, cfg.mode, cfg.tokens_per_rank, rpg)
    moe.build_layout(idx, w, er, L)
    return L


def assert_same(a, b, k):
    for key, va in a.items():
        vb = b[key]
        if key == "row_coef":
            assert np.all(np.abs(va.astype(np.float64) - vb) <= k * U * np.abs(vb.astype(np.float64)))
        else:
            assert np.array_equal(np.asarray(va), np.asarray(vb)), key


def test_static_scratch_layout_matches_regular_twice(moe):
    limit = static_limit()
    # sizes whose workspace would not fit are refused before any launch
    big = moe.layout_workspace_size(1 << 20, 8, 1024, 64, 1, W.PER_PICK)
    assert big > limit
    P = ctypes.c_void_p(256)
    L0 = moe.moe_layout()
    assert moe.lib().moe_build_layout_static(P, P, P, 1 << 20, 1 << 14, 8, 1024, 64, 1, W.PER_PICK,
                                             ctypes.byref(L0), None) == 2     # MOE_ERR_UNSUPPORTED
    for name in ("c3", "c5"):            # two calls in a row through the shared scratch
        cfg, idx, w, er = routed(name)
        assert moe.layout_workspace_size(cfg.T, cfg.k, cfg.E, cfg.R, max(cfg.ranks_per_group, 1),
                                         cfg.mode) <= limit
        Ls = static_layout(moe, cfg, idx, w, er)
        assert moe.get_status() == 0
        Lr = regular_layout(moe, cfg, idx, w, er)
        assert moe.get_status() == 0
        assert_same(layout_fields(Ls, cfg.mode), layout_fields(Lr, cfg.mode), cfg.k)
