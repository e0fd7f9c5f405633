"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the CPU oracle on the same seeded inputs, and compare them.

Tolerances come from the arithmetic (float32 on the device, float64 in the
oracle), with u = 2**-24 the float32 unit roundoff:

* gate weight of a pick with logit v, token max m and token minimum lo, when
  E experts are spread over ceil(E/32) slots per lane:
  |w_dev - w| <= (2.25 (m - v + m - lo) + ceil(E/32) + 14) * u * w.  Each
  exponential is exp2f(t * log2 e), t = v - m: the subtraction rounds t by a
  relative u, the float32 log2 e is off by 0.23 u, the product rounds by u,
  so the argument is off by at most 2.23 |t| u in relative terms, which is
  2.23 |t| u relative in the result; exp2f adds 2 ulp (<= 4 u).  The
  numerator's term is 2.23 (m - v) + 4; the sum over experts carries the
  worst term's 2.23 (m - lo) + 4 plus ceil(E/32) + 5 roundings of positive
  terms; the division one more.
* dedup coefficient (sum of a token's weights on a rank, float32 in pick
  order): the largest weight bound plus k u.
* combine: |out_dev - out| <= 1e-5 * sum_i |c_i y_i| plus one unit in the last
  place of the output format at |out| (the final rounding); float32
  accumulation of <= 16 terms and the coefficient errors above stay well
  inside 1e-5.  Two-hop adds one output-format ulp per rounded group partial.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W

U = 2.0 ** -24


@pytest.fixture(scope="session")
def moe():
    from combine_router_softmax_02_b200 import build as moe_build
    moe_build.build()
    import combine_router_softmax_02_b200 as m
    m.lib()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)) if isinstance(a, np.ndarray) else a
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda().contiguous()


def fmt_of(dtype) -> str:
    return {torch.float16: "f16", torch.bfloat16: "bf16", torch.float32: "f32"}[dtype]


def torch_dtype(name: str):
    return {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[name]


def weight_tol(logits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Relative bound on each gate weight (see the module docstring)."""
    lg = logits.astype(np.float64)
    m = lg.max(axis=1, keepdims=True)
    lo = lg.min(axis=1, keepdims=True)
    v = np.take_along_axis(lg, idx.astype(np.int64), axis=1)
    epl = math.ceil(lg.shape[1] / 32)
    return (2.25 * ((m - v) + (m - lo)) + epl + 14) * U


def assert_weights(w_dev, w_ref, logits, idx, renormalize=False):
    tol = weight_tol(logits, idx)
    if renormalize:
        tol = 2 * tol.max(axis=1, keepdims=True) + (idx.shape[1] + 2) * U
    err = np.abs(w_dev.astype(np.float64) - w_ref)
    bad = err > tol * np.abs(w_ref)
    assert not bad.any(), f"{bad.sum()} weights out of bound; worst rel {np.max(err / np.abs(w_ref))}"


def combine_bound(terms_abs_sum: np.ndarray, ref: np.ndarray, fmt: str) -> np.ndarray:
    return 1e-5 * terms_abs_sum + oracle.ulp(ref, fmt)


def assert_close_combine(dev: np.ndarray, ref: np.ndarray, abs_terms: np.ndarray, fmt: str,
                         extra: np.ndarray | float = 0.0, what="combine"):
    dev = dev.astype(np.float64)
    bound = combine_bound(abs_terms, ref, fmt) + extra
    err = np.abs(dev - ref)
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} elements out of bound; "
                           f"worst err {err.max():.3e}, at bound {bound.ravel()[np.argmax(err)]:.3e}")


def layout_fields(L, mode):
    """The device layout's buffers as numpy arrays, trimmed to num_rows."""
    n = int(L.num_rows.item())
    out = {
        "num_rows": n,
        "rank_offsets": L.rank_offsets.cpu().numpy(),
        "send_counts": L.send_counts.cpu().numpy(),
        "row_token": L.row_token[:n].cpu().numpy(),
        "row_coef": L.row_coef[:n].cpu().numpy(),
        "token_rows": L.token_rows.cpu().numpy(),
    }
    if mode == W.TWO_HOP:
        n1 = int(L.num_rows_hop1.item())
        out.update(num_rows_hop1=n1, group_offsets=L.group_offsets.cpu().numpy(),
                   hop1_row_token=L.hop1_row_token[:n1].cpu().numpy(),
                   token_groups=L.token_groups.cpu().numpy(),
                   hop2_src_row=L.hop2_src_row[:n].cpu().numpy(),
                   hop1_children=L.hop1_children[:n1].cpu().numpy())
    return out


def assert_layout_equal(dev, ref, mode, w_tol=None):
    """Integer fields bit-exact; coefficients within their float bound."""
    assert dev["num_rows"] == int(ref["num_rows"])
    for key in ("rank_offsets", "send_counts", "row_token", "token_rows"):
        assert np.array_equal(dev[key], ref[key].astype(np.int32)), key
    if mode == W.TWO_HOP:
        assert dev["num_rows_hop1"] == int(ref["num_rows_hop1"])
        for key in ("group_offsets", "hop1_row_token", "token_groups", "hop2_src_row", "hop1_children"):
            assert np.array_equal(dev[key], ref[key].astype(np.int32)), key
    rc = ref["row_coef"]
    tol = (w_tol if w_tol is not None else 4e-6)
    err = np.abs(dev["row_coef"].astype(np.float64) - rc)
    assert np.all(err <= tol * np.abs(rc) + 1e-30), f"row_coef worst rel {np.max(err / np.abs(rc))}"


def row_coef_tol(logits, idx, k):
    return float(weight_tol(logits, idx).max()) + k * U


class Case:
    """One seeded workload on both sides."""

    def __init__(self, cfg: W.Config, seed=0, T=None, with_x=True):
        self.cfg = cfg if T is None else cfg.with_(T=T)
        c = self.cfg
        self.logits = W.make_logits(c, seed)
        self.rm = W.make_replica_map(c, seed)
        self.x_cpu = W.make_activations(c, seed) if with_x else None
        self.tpr = -(-c.T // c.R)

    def oracle_route(self):
        c = self.cfg
        idx, w = oracle.route_topk(self.logits, c.k, c.n_groups, c.groups_per_token)
        counts = oracle.demand_hist(idx, c.E)
        slot, er, act = oracle.replica_assign(counts, self.rm.replica_offsets, self.rm.replica_slots,
                                              self.rm.slot_rank, c.R)
        L = oracle.build_layout(idx, w, er, self.tpr, c.R, c.mode, c.ranks_per_group)
        return dict(idx=idx, w=w, counts=counts, expert_slot=slot, expert_rank=er,
                    rank_active=act, layout=L)

    def device_path(self, moe, out_dtype=None):
        c = self.cfg
        dc = moe.DispatchCombine(c.T, c.H, c.E, c.k, c.R, to_dev(self.rm.replica_offsets),
                                 to_dev(self.rm.replica_slots), to_dev(self.rm.slot_rank), c.mode,
                                 self.tpr, max(c.ranks_per_group, 1), c.n_groups, c.groups_per_token,
                                 dtype=torch_dtype(c.dtype), out_dtype=out_dtype)
        return dc
