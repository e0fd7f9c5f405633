"""The C-ABI library loads and exports every entry point include/moe.h
declares, and its host-side checks reject bad arguments before any launch
(no GPU needed: nothing here reaches a kernel)."""
import ctypes
import os
import re
import subprocess

import pytest

import combine_router_softmax_02_b200 as moe
from combine_router_softmax_02_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.lib()


def header_symbols():
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            with open(os.path.join(ROOT, "include", h)) as f:
                names |= set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", f.read()))
    return names


def test_header_declares_the_path():
    syms = header_symbols()
    for name in ("moe_route_topk", "moe_demand_hist", "moe_replica_assign", "moe_build_layout",
                 "moe_pack", "moe_combine", "moe_layout_workspace_size", "moe_get_status"):
        assert name in syms


def test_every_declared_symbol_is_exported(lib):
    for name in header_symbols():
        assert hasattr(lib, name), name


def test_struct_layout_matches_header(tmp_path):
    """The ctypes mirror of moe_layout has the C compiler's size and offsets."""
    fields = [f for f, _ in moe.moe_layout._fields_]
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "moe.h"\nint main(void){\n'
                   '  printf("%zu\\n", sizeof(moe_layout));\n' +
                   "".join(f'  printf("%zu\\n", offsetof(moe_layout, {f}));\n' for f in fields) +
                   "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    vals = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True,
                                           check=True).stdout.split()]
    assert vals[0] == ctypes.sizeof(moe.moe_layout)
    assert vals[1:] == [getattr(moe.moe_layout, f).offset for f in fields]


def test_status_strings(lib):
    for code, name in enumerate(moe.STATUS_NAMES):
        assert moe.status_string(code) == name
    assert moe.status_string(99) == "MOE_ERR_UNKNOWN"


def test_workspace_size(lib):
    # a header of 16 barrier words and a 1024-entry demand scratch, then one int
    # per (block, bin) with bins padded to a multiple of 4; at most 512 blocks,
    # and at most one per 8 tokens
    H = 4 * (16 + 1024)
    assert moe.layout_workspace_size(65536, 8, 256, 64, 1, moe.DEDUP) == H + 512 * 64 * 4
    assert moe.layout_workspace_size(100, 6, 64, 32, 1, moe.PER_PICK) == H + 13 * 64 * 4
    assert moe.layout_workspace_size(32768, 8, 128, 64, 8, moe.TWO_HOP) == H + 512 * 72 * 4
    assert moe.layout_workspace_size(1, 2, 10, 3, 1, moe.DEDUP) == H + 1 * 4 * 4
    assert moe.layout_workspace_size(10, 3, 2, 4, 1, moe.DEDUP) == 0        # k > E
    assert moe.layout_workspace_size(10, 2, 8, 65, 1, moe.DEDUP) == 0       # R > 64
    assert moe.layout_workspace_size(10, 2, 8, 8, 3, moe.TWO_HOP) == 0      # rpg does not divide R


def test_bad_arguments_rejected_before_launch(lib):
    P = ctypes.c_void_p(16)
    INVALID, UNSUPPORTED = 1, 2
    assert lib.moe_route_topk(P, 4, 8, 9, 0, 0, 0, P, P, None) == INVALID          # k > E
    assert lib.moe_route_topk(P, 4, 2048, 2, 0, 0, 0, P, P, None) == INVALID       # E > 1024
    assert lib.moe_route_topk(None, 4, 8, 2, 0, 0, 0, P, P, None) == INVALID       # null logits
    assert lib.moe_route_topk(P, 4, 8, 2, 3, 1, 0, P, P, None) == INVALID          # groups do not divide E
    assert lib.moe_route_topk(P, 4, 8, 4, 4, 1, 0, P, P, None) == INVALID          # gpt * E/G < k
    assert lib.moe_route_topk(P, 1 << 28, 64, 16, 0, 0, 0, P, P, None) == UNSUPPORTED
    assert lib.moe_demand_hist(P, 4, 2, 8, None, None) == INVALID
    assert lib.moe_replica_assign(P, 8, P, P, 8, P, 0, 4, P, P, P, None) == INVALID  # S = 0
    L = moe.moe_layout()
    assert lib.moe_build_layout(P, P, P, 8, 1, 2, 8, 4, 1, 1, ctypes.byref(L), P, 1 << 20, None) == INVALID
    L.rank_offsets = L.send_counts = L.num_rows = L.token_rows = L.row_token = L.row_coef = 16
    L.capacity = 16
    # tokens_per_rank * R < T
    assert lib.moe_build_layout(P, P, P, 8, 1, 2, 8, 4, 1, 1, ctypes.byref(L), P, 1 << 20, None) == INVALID
    # workspace too small
    assert lib.moe_build_layout(P, P, P, 8, 2, 2, 8, 4, 1, 1, ctypes.byref(L), P, 8, None) == INVALID
    L.T, L.k, L.E, L.R, L.mode = 8, 2, 8, 4, 1
    assert lib.moe_pack(P, 1, 7, ctypes.byref(L), P, None, None) == UNSUPPORTED    # 14-byte rows
    assert lib.moe_pack(P, 5, 8, ctypes.byref(L), P, None, None) == INVALID        # bad dtype
    assert lib.moe_pack(ctypes.c_void_p(8), 1, 8, ctypes.byref(L), P, None, None) == INVALID  # misaligned
    assert lib.moe_combine(P, 1, 8, ctypes.byref(L), None, P, 7, None, None) == INVALID
    assert lib.moe_debug_set_wait(0, -2) == INVALID


def test_one_launch_front_ends_reject_bad_arguments(lib):
    """moe_route_assign_layout and moe_route_layout_single_replica check their
    arguments on the host and return before any launch (no GPU is touched)."""
    P = ctypes.c_void_p(256)
    INVALID, UNSUPPORTED = 1, 2
    L = moe.moe_layout()
    L.rank_offsets = L.send_counts = L.num_rows = L.token_rows = L.row_token = L.row_coef = 256
    L.capacity = 64
    ws = 1 << 20

    def ral(T=32, E=16, k=2, ng=0, gpt=0, ren=0, n_entries=16, S=16, tpr=8, R=4, rpg=1, mode=1,
            logits=P, offs=P, slots=P, srank=P, counts=P, eslot=P, erank=P, active=P, wsb=ws, wsp=P):
        return lib.moe_route_assign_layout(logits, T, E, k, ng, gpt, ren, offs, slots, n_entries, srank, S,
                                           tpr, R, rpg, mode, P, P, counts, eslot, erank, active,
                                           ctypes.byref(L), wsp, wsb, None)

    assert ral(k=17) == INVALID                      # k > E
    assert ral(E=2048) == INVALID                    # E > 1024
    assert ral(R=65) == INVALID                      # R > 64
    assert ral(mode=3) == INVALID                    # no such layout mode
    assert ral(tpr=7) == INVALID                     # tokens_per_rank * R < T
    assert ral(ng=3, gpt=1) == INVALID               # groups do not divide E
    assert ral(ren=2) == INVALID                     # renormalize is 0 or 1
    assert ral(S=0) == INVALID                       # no replica slots
    assert ral(n_entries=40000) == INVALID           # more replica entries than slots allowed
    assert ral(offs=None) == INVALID
    assert ral(slots=None) == INVALID                # entries but no slot list
    assert ral(srank=None) == INVALID
    assert ral(counts=None) == INVALID
    assert ral(eslot=None) == INVALID
    assert ral(erank=None) == INVALID
    assert ral(active=None) == INVALID
    assert ral(logits=None) == INVALID
    assert ral(wsb=8) == INVALID                     # workspace too small
    assert ral(wsp=ctypes.c_void_p(264)) == INVALID  # workspace not 16-byte aligned
    assert ral(mode=2, rpg=3) == INVALID             # ranks per group must divide R
    assert ral(T=1 << 28, k=16, tpr=1 << 26) == UNSUPPORTED  # T * k overflows 31 bits
    assert lib.moe_route_layout_single_replica(P, 32, 16, 2, 0, 0, 0, None, 8, 4, 1, 1, P, P, P, P,
                                               ctypes.byref(L), P, ws, None) == INVALID  # no expert_rank
