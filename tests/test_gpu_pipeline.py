"""The host-buffer pipeline (chunked copies overlapped with the kernels, token
ranges of pack and combine) gives the outputs of whole-range steps bit for bit."""
import numpy as np
import pytest
import torch

import workloads as W
from gpu_util import Case, moe, to_dev  # noqa: F401

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,chunks", [("c1", 3), ("c2", 8), ("c5", 5), ("c3", 1)])
def test_pipeline_matches_whole_steps(moe, name, chunks):
    cfg = W.CONFIGS[name] if name != "c5" else W.CONFIGS[name].with_(T=4096)
    case = Case(cfg, with_x=False)
    dc = case.device_path(moe)
    pipe = moe.HostPipeline(dc, chunks=chunks)
    tdt = dc.dtype
    seeds = (1, 2, 3)
    ins = [(W.make_logits(case.cfg, s), W.make_activations(case.cfg, s)) for s in seeds]
    hosts = [(torch.from_numpy(np.ascontiguousarray(lg)).pin_memory(), x.pin_memory(),
              torch.empty((case.cfg.T, case.cfg.H), dtype=tdt).pin_memory()) for lg, x in ins]
    for lg_h, x_h, out_h in hosts:          # three steps in flight, double-buffered
        pipe.step(lg_h, x_h, out_h)
    pipe.join()
    torch.cuda.synchronize()
    assert moe.get_status() == 0
    for (lg, x), (_, _, out_h) in zip(ins, hosts):
        dc.step(to_dev(lg), x.cuda())
        torch.cuda.synchronize()
        assert torch.equal(out_h.view(torch.uint8), dc.out.cpu().view(torch.uint8))
    assert moe.get_status() == 0


def test_token_ranges_match_whole_calls(moe):
    cfg = W.CONFIGS["c5"].with_(T=1000)
    case = Case(cfg)
    dc = case.device_path(moe)
    x = case.x_cpu.cuda()
    dc.step(to_dev(case.logits), x)
    whole, whole_h1 = dc.packed.clone(), dc.packed_hop1.clone()
    out_whole = dc.out.clone()
    dc.packed.zero_()
    dc.packed_hop1.zero_()
    for a, b in ((700, 1000), (0, 333), (333, 700)):   # any order
        moe.pack(x, dc.layout, dc.packed, dc.packed_hop1, tokens=(a, b))
    n, n1 = int(dc.layout.num_rows.item()), int(dc.layout.num_rows_hop1.item())
    assert torch.equal(dc.packed[:n].view(torch.int16), whole[:n].view(torch.int16))
    assert torch.equal(dc.packed_hop1[:n1].view(torch.int16), whole_h1[:n1].view(torch.int16))
    out = torch.zeros_like(dc.out)
    for a, b in ((500, 1000), (0, 1), (1, 500)):
        moe.combine(dc.packed, dc.layout, out, dc.out_dtype, None, dc.hop1_buf, tokens=(a, b))
    assert torch.equal(out.view(torch.int16), out_whole.view(torch.int16))
    assert moe.get_status() == 0
    with pytest.raises(ValueError):
        moe.pack(x, dc.layout, dc.packed, dc.packed_hop1, tokens=(0, 1001))
