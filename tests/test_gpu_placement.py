"""GPU parity of the co-selection histogram and the correlated placement
against the CPU oracle (both integer: bit-exact)."""
import numpy as np
import pytest
import torch

import oracle
import pins
import workloads as W
from gpu_util import moe, to_dev  # noqa: F401

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["c1", "c3", "c4"])
def test_coselection_and_placement_configs(moe, name):
    cfg = W.CONFIGS[name]
    idx, w = oracle.route_topk(W.make_logits(cfg, 0), cfg.k)
    C_d = moe.coselection_hist(to_dev(idx), cfg.E)
    C = oracle.coselection(idx, cfg.E)
    assert np.array_equal(C_d.cpu().numpy(), C)
    counts = oracle.demand_hist(idx, cfg.E)
    er_d = moe.correlated_placement(C_d, to_dev(counts.astype(np.int32)), cfg.R)
    assert moe.get_status() == 0
    assert np.array_equal(er_d.cpu().numpy(), oracle.correlated_placement(C, counts, cfg.R))


def test_placement_pins_on_device(moe):
    """The oracle's placement pins, run against the device kernel."""
    def dev_placement(C, counts, R):
        return moe.correlated_placement(to_dev(np.asarray(C, np.int32)),
                                        to_dev(np.asarray(counts, np.int32)), R).cpu().numpy()
    pins.check_placement(dev_placement)
    assert moe.get_status() == 0


def test_derived_placement_in_the_path(moe):
    """Route the clustered training batch, derive a placement on the device,
    and lay it out: fewer dedup rows than round-robin placement."""
    cfg = W.CONFIGS["c3"]
    lg = to_dev(W.make_logits(cfg, 0))
    idx, w = moe.route_topk(lg, cfg.k)
    counts = moe.demand_hist(idx, cfg.E)
    er = moe.correlated_placement(moe.coselection_hist(idx, cfg.E), counts, cfg.R)
    rows = {}
    for name, rank in (("derived", er), ("roundrobin", to_dev(W.expert_home_rank(cfg.with_(placement="roundrobin"))))):
        L = moe.Layout(cfg.T, cfg.k, cfg.E, cfg.R, W.DEDUP, cfg.tokens_per_rank)
        moe.build_layout(idx, w, rank, L)
        rows[name] = int(L.num_rows.item())
    assert moe.get_status() == 0
    assert rows["derived"] < rows["roundrobin"]
