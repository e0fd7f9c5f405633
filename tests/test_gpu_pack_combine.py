"""GPU parity: pack (bit copy) and combine (float32 accumulation) against the
CPU oracle, one-hop and two-hop, plus conservation (combine after pack with
0/1 coefficients is the identity) and the full path at the benchmark sizes."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from gpu_util import (Case, assert_close_combine, assert_layout_equal, fmt_of, layout_fields, moe,  # noqa: F401
                      row_coef_tol, to_dev, torch_dtype)

pytestmark = pytest.mark.gpu


def bits(t: torch.Tensor) -> np.ndarray:
    return t.cpu().contiguous().view(torch.int16 if t.element_size() == 2 else torch.int32).numpy()


def compact_rows(token_rows, tokens):
    """Rows used by the sampled tokens, and token_rows re-indexed into them."""
    tr = token_rows[tokens].astype(np.int64)
    used = np.unique(tr[tr >= 0])
    remap = np.full(tr.shape, -1, np.int64)
    m = tr >= 0
    remap[m] = np.searchsorted(used, tr[m])
    return used, remap


def check_combine_sampled(out_dev, y_rows_f64, token_rows, coef, tokens, fmt):
    """Oracle combine on sampled tokens; y_rows_f64(rows) gives the rows' values."""
    used, remap = compact_rows(token_rows, tokens)
    y = y_rows_f64(used)
    c = np.asarray(coef, np.float64)[used]
    ref = oracle.combine(y, remap, c)
    absum = oracle.combine(np.abs(y), remap, np.abs(c))
    got = out_dev[torch.from_numpy(np.asarray(tokens, np.int64)).cuda()].double().cpu().numpy()
    assert_close_combine(got, ref, absum, fmt)


class PackedRows:
    """The oracle's packed rows ``Y[i] = X[row_token[i]]`` (identity experts)
    as float64, gathered on demand so that a full-size combine can run in
    token chunks without holding every row at once."""

    def __init__(self, x64_of, row_token, H):
        self.x64_of, self.row_token, self.shape = x64_of, np.asarray(row_token, np.int64), (len(row_token), H)

    def __getitem__(self, rows):
        return self.x64_of(self.row_token[rows])


def assert_rows_bit_exact(dev_rows, x_bits, row_token, chunk=32768):
    """Every packed row on the device equals the oracle's pack of the token
    bits, compared in chunks of rows copied back to the host."""
    n = len(row_token)
    for r0 in range(0, n, chunk):
        r1 = min(n, r0 + chunk)
        got = bits(dev_rows[r0:r1])
        want = oracle.pack(x_bits, row_token[r0:r1])
        if not np.array_equal(got, want):
            bad = np.flatnonzero(np.any(got != want, axis=1))
            raise AssertionError(f"{len(bad)} packed rows differ in rows [{r0}, {r1}); first {r0 + bad[0]}")


def check_combine_all_tokens(out_dev, y, token_rows, coef, fmt, chunk=4096):
    """Oracle combine of every token, in token chunks, against the device output."""
    T = token_rows.shape[0]
    c = np.asarray(coef, np.float64)
    for t0 in range(0, T, chunk):
        toks = np.arange(t0, min(T, t0 + chunk))
        ref = oracle.combine(y, token_rows, c, tokens=toks)
        absum = oracle.combine(_Abs(y), token_rows, np.abs(c), tokens=toks)
        got = out_dev[t0:t0 + len(toks)].double().cpu().numpy()
        assert_close_combine(got, ref, absum, fmt, what=f"combine tokens [{t0}, {t0 + len(toks)})")


class _Abs:
    """|Y| of a row source, for the bound's sum of absolute terms."""

    def __init__(self, y):
        self.y, self.shape = y, y.shape

    def __getitem__(self, rows):
        return np.abs(np.asarray(self.y[rows], np.float64))


SMALL = [("c1", W.DEDUP), ("c1", W.PER_PICK), ("c2", W.DEDUP), ("c3", W.DEDUP), ("c3", W.PER_PICK)]


@pytest.mark.parametrize("name,mode", SMALL)
@pytest.mark.parametrize("out_dtype", ["same", "f32"])
def test_path_small_configs_every_row(moe, name, mode, out_dtype):
    cfg = W.CONFIGS[name].with_(mode=mode)
    case = Case(cfg)
    ref = case.oracle_route()
    odt = None if out_dtype == "same" else torch.float32
    dc = case.device_path(moe, odt)
    x = case.x_cpu.cuda()
    out = dc.step(to_dev(case.logits), x)
    assert moe.get_status() == 0
    assert np.array_equal(dc.topk_idx.cpu().numpy(), ref["idx"])
    assert np.array_equal(dc.expert_rank.cpu().numpy(), ref["expert_rank"])
    lay = layout_fields(dc.layout, mode)
    assert_layout_equal(lay, ref["layout"], mode, w_tol=row_coef_tol(case.logits, ref["idx"], cfg.k))
    n = lay["num_rows"]
    # pack: every row is a bit copy of its token
    xb = bits(case.x_cpu)
    assert np.array_equal(bits(dc.packed[:n]), xb[ref["layout"]["row_token"]])
    # combine with identity experts against the oracle on every token
    fmt = fmt_of(dc.out_dtype)
    x64 = case.x_cpu.double().numpy()
    rt = ref["layout"]["row_token"]
    check_combine_sampled(out, lambda rows: x64[rt[rows]], ref["layout"]["token_rows"],
                          ref["layout"]["row_coef"], np.arange(cfg.T), fmt)


def test_combine_random_outputs_and_coefs(moe):
    """Expert outputs that differ per row (so terms can cancel) and random
    float32 coefficients given to both sides."""
    cfg = W.CONFIGS["c3"]
    case = Case(cfg, with_x=False)
    r = case.oracle_route()
    ref = r["layout"]
    n = int(ref["num_rows"])
    rng = np.random.default_rng(3)
    y = rng.standard_normal((n, cfg.H)).astype(np.float32)
    coef = W.make_uniform_coefs(n, seed=4) * np.where(rng.random(n) < 0.3, -1, 1).astype(np.float32)
    L = moe.Layout(cfg.T, cfg.k, cfg.E, cfg.R, W.DEDUP, cfg.tokens_per_rank)
    moe.build_layout(to_dev(r["idx"]), to_dev(r["w"].astype(np.float32)), to_dev(r["expert_rank"]), L)
    for dt in (torch.bfloat16, torch.float16, torch.float32):
        y_d = torch.from_numpy(y).to(dt).cuda()
        for odt in (torch.float32, dt):
            out = moe.combine(y_d, L, out_dtype=odt, row_coef=to_dev(coef))
            assert moe.get_status() == 0
            y64 = y_d.double().cpu().numpy()
            check_combine_sampled(out, lambda rows: y64[rows], ref["token_rows"], coef,
                                  np.arange(cfg.T), fmt_of(odt))


def test_conservation_and_all_ones(moe):
    """combine(pack(x)) with coefficient 1 on each token's first row and 0 on
    the rest returns x exactly; all-ones coefficients with float32 output
    return d_t * x exactly (d_t <= 8 rows).  Exact means equal values: an
    input -0.0 comes back as +0.0 (IEEE -0 + +0 = +0), in the oracle too; the
    non-zero elements must match bit for bit."""
    for name in ("c1", "c3"):
        cfg = W.CONFIGS[name]
        case = Case(cfg)
        dc = case.device_path(moe)
        x = case.x_cpu.cuda()
        dc.dispatch(to_dev(case.logits), x)
        n = int(dc.layout.num_rows.item())
        tr = dc.layout.token_rows.long()
        c01 = torch.zeros(n, dtype=torch.float32, device="cuda")
        c01[tr[:, 0]] = 1.0
        out = moe.combine(dc.packed[:n], dc.layout, row_coef=c01)
        assert torch.equal(out, x)                                   # values, -0 == +0
        nz = x != 0
        assert torch.equal(out.view(torch.int16)[nz], x.view(torch.int16)[nz])
        ref0 = oracle.combine(np.array([[-0.0]]), np.array([[0]]), np.array([1.0]))
        assert ref0[0, 0] == 0.0 and not np.signbit(ref0[0, 0])     # the oracle agrees on -0
        ones = torch.ones(n, dtype=torch.float32, device="cuda")
        out32 = moe.combine(dc.packed[:n], dc.layout, out_dtype=torch.float32, row_coef=ones)
        d = (tr >= 0).sum(dim=1, keepdim=True).float()
        assert torch.equal(out32, d * x.float())
        assert moe.get_status() == 0


def check_two_hop_tokens(out, hop1_buf, RL, x_of, toks, fmt):
    """Two-hop combine of the tokens `toks` against the oracle: each group's
    rank rows summed and rounded to the wire dtype, then the groups summed;
    and the stored group partials of those tokens, each within its own bound."""
    tr, tg = RL["token_rows"][toks], RL["token_groups"][toks]
    used2, used1 = np.unique(tr[tr >= 0]), np.unique(tg[tg >= 0])
    sub = {"token_rows": np.where(tr >= 0, np.searchsorted(used2, tr), -1),
           "token_groups": np.where(tg >= 0, np.searchsorted(used1, tg), -1),
           "hop2_src_row": np.searchsorted(used1, RL["hop2_src_row"][used2])}
    y2 = x_of(RL["row_token"][used2])
    c2 = RL["row_coef"][used2]
    o, zs = oracle.combine_two_hop(y2, sub, c2, fmt)
    absum, _ = oracle.combine_two_hop(np.abs(y2), sub, np.abs(c2), "f32")
    extra = np.zeros_like(o)
    for gi in range(sub["token_groups"].shape[1]):    # one output ulp per rounded group partial
        col = sub["token_groups"][:, gi]
        have = col >= 0
        if have.any():
            z = np.stack([zs[int(r)] for r in col[have]])
            extra[have] += oracle.ulp(z, fmt)
    assert_close_combine(out[torch.from_numpy(toks).cuda()].double().cpu().numpy(), o, absum, fmt,
                         extra=extra, what="two-hop combine")
    z_dev = hop1_buf[torch.from_numpy(used1.astype(np.int64)).cuda()].double().cpu().numpy()
    z_ref = np.stack([zs[i] for i in range(len(used1))])
    zabs = np.zeros_like(z_ref)
    for i2, s1 in enumerate(sub["hop2_src_row"]):
        zabs[s1] += np.abs(c2[i2] * y2[i2])
    assert_close_combine(z_dev, z_ref, zabs, fmt, extra=oracle.ulp(z_ref, fmt), what="group partials")


def check_two_hop(moe, cfg, chunk=4096):
    """The two-hop path against the oracle: layout bit-exact, every hop-1 and
    hop-2 packed row bit-exact, every token's combine and group partial
    within its bound (in token chunks)."""
    case = Case(cfg)
    ref = case.oracle_route()
    RL = ref["layout"]
    dc = case.device_path(moe)
    x = case.x_cpu.cuda()
    out = dc.step(to_dev(case.logits), x)
    assert moe.get_status() == 0
    lay = layout_fields(dc.layout, W.TWO_HOP)
    assert_layout_equal(lay, RL, W.TWO_HOP, w_tol=row_coef_tol(case.logits, ref["idx"], cfg.k))
    n, n1 = lay["num_rows"], lay["num_rows_hop1"]
    xb = bits(case.x_cpu)
    assert_rows_bit_exact(dc.packed_hop1[:n1], xb, RL["hop1_row_token"])
    assert_rows_bit_exact(dc.packed[:n], xb, RL["row_token"])
    fmt = fmt_of(dc.out_dtype)
    xs = case.x_cpu
    x_of = lambda t: xs[torch.from_numpy(np.asarray(t, np.int64))].double().numpy()  # noqa: E731
    for t0 in range(0, cfg.T, chunk):
        check_two_hop_tokens(out, dc.hop1_buf, RL, x_of, np.arange(t0, min(cfg.T, t0 + chunk)), fmt)
    # not storing the partials changes nothing else
    out2 = moe.combine(dc.packed, dc.layout, out_dtype=dc.out_dtype, store_hop1=False)
    assert torch.equal(out2.view(torch.int16), out.view(torch.int16))
    assert moe.get_status() == 0


def test_two_hop_small_every_row(moe):
    check_two_hop(moe, W.CONFIGS["c5"].with_(T=2048))


def test_two_hop_full_size_every_row(moe):
    """The two-hop benchmark workload (32768 tokens x 4096 bf16) in full."""
    check_two_hop(moe, W.CONFIGS["c5"])


def test_full_size_prefill_path_every_row(moe):
    """The benchmark's workload and launch configuration (DispatchCombine.step
    on 65536 tokens x 7168 bf16): layout bit-exact, every packed row bit-exact,
    every output token within the combine bound."""
    cfg = W.CONFIGS["c4"]
    case = Case(cfg)
    ref = case.oracle_route()
    RL = ref["layout"]
    dc = case.device_path(moe)
    x = case.x_cpu.cuda()
    out = dc.step(to_dev(case.logits), x)
    assert moe.get_status() == 0
    assert np.array_equal(dc.topk_idx.cpu().numpy(), ref["idx"])
    lay = layout_fields(dc.layout, W.DEDUP)
    assert_layout_equal(lay, RL, W.DEDUP, w_tol=row_coef_tol(case.logits, ref["idx"], cfg.k))
    assert_rows_bit_exact(dc.packed[:lay["num_rows"]], bits(case.x_cpu), RL["row_token"])
    xs = case.x_cpu
    y = PackedRows(lambda t: xs[torch.from_numpy(t)].double().numpy(), RL["row_token"], cfg.H)
    check_combine_all_tokens(out, y, RL["token_rows"], RL["row_coef"], "bf16")
