"""The whole path captured in a CUDA graph: replays give the eager outputs
bit for bit, on new inputs copied into the captured buffers."""
import numpy as np
import pytest
import torch

import workloads as W
from gpu_util import Case, moe, to_dev  # noqa: F401

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["c1", "c2", "c5"])
def test_graph_replay_matches_eager(moe, name):
    cfg = W.CONFIGS[name]
    case = Case(cfg)
    dc = case.device_path(moe)
    logits = to_dev(case.logits)
    x = case.x_cpu.cuda()
    dc.step(logits, x)                          # warm-up outside the capture
    assert moe.get_status() == 0
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dc.step(logits, x)
    for seed in (3, 4):                         # new inputs into the captured buffers
        logits.copy_(to_dev(W.make_logits(cfg, seed)))
        x.copy_(W.make_activations(cfg, seed).cuda())
        g.replay()
        torch.cuda.synchronize()
        got = dc.out.clone()
        n_got = int(dc.layout.num_rows.item())
        dc.step(logits, x)
        assert moe.get_status() == 0
        assert int(dc.layout.num_rows.item()) == n_got
        assert torch.equal(got.view(torch.uint8), dc.out.view(torch.uint8))
    del g
