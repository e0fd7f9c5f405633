"""moe_build_layout_static: the layout entry point for callers that cannot
allocate device memory (a serving loop whose memory is all reserved at
start-up, or a host framework that only hands over its existing buffers).

It takes its scratch from a fixed device array inside the library instead of
a caller-supplied workspace.  This test calls it through the C ABI several
times in a row on different workloads, up to the sizes the header documents
(the shared array keeps the previous call's contents), and checks each result
against the regular moe_build_layout with its own workspace: every field
bit-exact.  The file is named to be collected
last.
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


def static_limit() -> int:
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        m = re.search(r"#define\s+MOE_LAYOUT_STATIC_SCRATCH_BYTES\s+\(1u\s*<<\s*(\d+)\)", f.read())
    return 1 << int(m.group(1))


def routed(name, mode=None):
    cfg = W.CONFIGS[name] if mode is None else W.CONFIGS[name].with_(mode=mode)
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


def assert_same(a, b):
    """Both calls run the same kernel on the same inputs, so every field,
    the float32 coefficients included, must be identical bit for bit."""
    for key, va in a.items():
        vb = b[key]
        if key == "row_coef":
            assert np.array_equal(va.view(np.int32), vb.view(np.int32)), key
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
    # calls in a row through the shared scratch, up to the documented sizes:
    # 65536 tokens over 64 ranks (DEDUP) and over 256 experts (PER_PICK)
    for name, mode in (("c3", None), ("c5", None), ("c4", None), ("c4", W.PER_PICK), ("c3", None)):
        cfg, idx, w, er = routed(name, mode)
        assert moe.layout_workspace_size(cfg.T, cfg.k, cfg.E, cfg.R, max(cfg.ranks_per_group, 1),
                                         cfg.mode) <= limit
        Ls = static_layout(moe, cfg, idx, w, er)
        assert moe.get_status() == 0
        Lr = regular_layout(moe, cfg, idx, w, er)
        assert moe.get_status() == 0
        assert_same(layout_fields(Ls, cfg.mode), layout_fields(Lr, cfg.mode))
