"""ctypes binding of libmoe.so: the C ABI of include/moe.h, same names.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch provides device memory and the current stream.  There is no
fallback: if libmoe.so is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK = 0
STATUS_NAMES = ["MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_UNSUPPORTED", "MOE_ERR_CUDA",
                "MOE_ERR_TIMEOUT", "MOE_ERR_BOUNDS", "MOE_ERR_BAD_INPUT", "MOE_ERR_CAPACITY"]
F16, BF16, F32 = 0, 1, 2
PER_PICK, DEDUP, TWO_HOP = 0, 1, 2
_DT = {torch.float16: F16, torch.bfloat16: BF16, torch.float32: F32}
_TORCH_DT = {v: k for k, v in _DT.items()}


class MoeError(RuntimeError):
    def __init__(self, what: str, code: int):
        name = STATUS_NAMES[code] if 0 <= code < len(STATUS_NAMES) else str(code)
        super().__init__(f"{what} failed: {name}")
        self.code = code


class moe_layout(ctypes.Structure):
    _fields_ = [
        ("rank_offsets", ctypes.c_void_p), ("send_counts", ctypes.c_void_p),
        ("row_token", ctypes.c_void_p), ("row_coef", ctypes.c_void_p),
        ("token_rows", ctypes.c_void_p), ("num_rows", ctypes.c_void_p),
        ("capacity", ctypes.c_int32),
        ("group_offsets", ctypes.c_void_p), ("hop1_row_token", ctypes.c_void_p),
        ("token_groups", ctypes.c_void_p), ("hop2_src_row", ctypes.c_void_p),
        ("hop1_children", ctypes.c_void_p), ("num_rows_hop1", ctypes.c_void_p),
        ("capacity_hop1", ctypes.c_int32),
        ("T", ctypes.c_int32), ("k", ctypes.c_int32), ("R", ctypes.c_int32),
        ("E", ctypes.c_int32), ("ranks_per_group", ctypes.c_int32), ("mode", ctypes.c_int32),
    ]


_lib = None
_P, _I, _SZ, _S = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_void_p
_SIGS = {
    "moe_route_topk": (ctypes.c_int, [_P, _I, _I, _I, _I, _I, _I, _P, _P, _S]),
    "moe_demand_hist": (ctypes.c_int, [_P, _I, _I, _I, _P, _S]),
    "moe_replica_assign": (ctypes.c_int, [_P, _I, _P, _P, _I, _P, _I, _I, _P, _P, _P, _S]),
    "moe_layout_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "moe_build_layout": (ctypes.c_int, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                        ctypes.POINTER(moe_layout), _P, _SZ, _S]),
    "moe_build_layout_static": (ctypes.c_int, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                               ctypes.POINTER(moe_layout), _S]),
    "moe_pack": (ctypes.c_int, [_P, _I, _I, ctypes.POINTER(moe_layout), _P, _P, _S]),
    "moe_combine": (ctypes.c_int, [_P, _I, _I, ctypes.POINTER(moe_layout), _P, _P, _I, _P, _S]),
    "moe_get_status": (ctypes.c_int, [_S]),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_debug_set_wait": (ctypes.c_int, [ctypes.c_uint64, _I]),
    "moe_kernel_launches": (ctypes.c_uint64, []),
    "moe_route_layout_single_replica": (ctypes.c_int, [_P, _I, _I, _I, _I, _I, _I, _P, _I, _I, _I, _I,
                                                       _P, _P, _P, _P, ctypes.POINTER(moe_layout),
                                                       _P, _SZ, _S]),
    "moe_route_assign_layout": (ctypes.c_int, [_P, _I, _I, _I, _I, _I, _I, _P, _P, _I, _P, _I, _I, _I,
                                               _I, _I, _P, _P, _P, _P, _P, _P,
                                               ctypes.POINTER(moe_layout), _P, _SZ, _S]),
    "moe_coselection_hist": (ctypes.c_int, [_P, _I, _I, _I, _P, _S]),
    "moe_correlated_placement": (ctypes.c_int, [_P, _P, _I, _I, _P, _S]),
    "moe_dispatch_stats": (ctypes.c_int, [_P, _I, _P, _I, _P, _S]),
    "moe_token_balanced_assign": (ctypes.c_int, [_P, _I, _P, _P, _I, _P, _I, _I, _P, _P, _S]),
}


def lib() -> ctypes.CDLL:
    """The loaded libmoe.so (raises ImportError if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m combine_router_softmax_02_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _p(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, dtype, name: str, ndim: Optional[int] = None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")


def _check(rc: int, what: str):
    if rc != MOE_OK:
        raise MoeError(what, rc)


def status_string(code: int) -> str:
    return lib().moe_status_string(code).decode()


def get_status(stream=None) -> int:
    """Synchronises the stream; returns and clears the device status word."""
    return lib().moe_get_status(_stream(stream))


def check_status(stream=None):
    rc = get_status(stream)
    if rc != MOE_OK:
        raise MoeError("device", rc)


def kernel_launches() -> int:
    """Kernels libmoe.so has launched in this process (counted by the library)."""
    return int(lib().moe_kernel_launches())


def debug_set_wait(wait_limit_ns: int = 0, layout_silent_tile: int = -1):
    _check(lib().moe_debug_set_wait(wait_limit_ns, layout_silent_tile), "moe_debug_set_wait")


# ----------------------------------------------------------------- route ----
def route_topk(logits: torch.Tensor, k: int, n_groups: int = 0, groups_per_token: int = 0,
               renormalize: bool = False, topk_idx=None, topk_w=None, stream=None):
    _need(logits, torch.float32, "logits", 2)
    T, E = logits.shape
    dev = logits.device
    topk_idx = torch.empty((T, k), dtype=torch.int32, device=dev) if topk_idx is None else topk_idx
    topk_w = torch.empty((T, k), dtype=torch.float32, device=dev) if topk_w is None else topk_w
    _need(topk_idx, torch.int32, "topk_idx")
    _need(topk_w, torch.float32, "topk_w")
    _check(lib().moe_route_topk(_p(logits), T, E, k, n_groups, groups_per_token, int(renormalize),
                                _p(topk_idx), _p(topk_w), _stream(stream)), "moe_route_topk")
    return topk_idx, topk_w


def demand_hist(topk_idx: torch.Tensor, E: int, counts=None, stream=None):
    _need(topk_idx, torch.int32, "topk_idx", 2)
    T, k = topk_idx.shape
    counts = torch.empty(E, dtype=torch.int32, device=topk_idx.device) if counts is None else counts
    _need(counts, torch.int32, "counts")
    _check(lib().moe_demand_hist(_p(topk_idx), T, k, E, _p(counts), _stream(stream)), "moe_demand_hist")
    return counts


def replica_assign(counts, replica_offsets, replica_slots, slot_rank, R: int,
                   expert_slot=None, expert_rank=None, rank_active=None, stream=None):
    for t, n in ((counts, "counts"), (replica_offsets, "replica_offsets"),
                 (replica_slots, "replica_slots"), (slot_rank, "slot_rank")):
        _need(t, torch.int32, n, 1)
    E = counts.numel()
    dev = counts.device
    expert_slot = torch.empty(E, dtype=torch.int32, device=dev) if expert_slot is None else expert_slot
    expert_rank = torch.empty(E, dtype=torch.int32, device=dev) if expert_rank is None else expert_rank
    rank_active = torch.empty(R, dtype=torch.int32, device=dev) if rank_active is None else rank_active
    _check(lib().moe_replica_assign(_p(counts), E, _p(replica_offsets), _p(replica_slots),
                                    replica_slots.numel(), _p(slot_rank), slot_rank.numel(), R,
                                    _p(expert_slot), _p(expert_rank), _p(rank_active),
                                    _stream(stream)), "moe_replica_assign")
    return expert_slot, expert_rank, rank_active


# ---------------------------------------------------------------- layout ----
def layout_workspace_size(T: int, k: int, E: int, R: int, ranks_per_group: int, mode: int) -> int:
    return lib().moe_layout_workspace_size(T, k, E, R, ranks_per_group, mode)


class Layout:
    """Device buffers of one layout (caller-owned memory, allocated with torch)
    and the C struct that points at them."""

    def __init__(self, T: int, k: int, E: int, R: int, mode: int, tokens_per_rank: int,
                 ranks_per_group: int = 1, capacity: Optional[int] = None,
                 capacity_hop1: Optional[int] = None, device="cuda"):
        self.T, self.k, self.E, self.R, self.mode = T, k, E, R, mode
        self.tokens_per_rank, self.ranks_per_group = tokens_per_rank, ranks_per_group
        cap = T * k if capacity is None else capacity
        i32 = dict(dtype=torch.int32, device=device)
        self.rank_offsets = torch.zeros(R + 1, **i32)
        self.send_counts = torch.zeros((R, R), **i32)
        self.row_token = torch.empty(max(cap, 1), **i32)
        self.row_coef = torch.empty(max(cap, 1), dtype=torch.float32, device=device)
        self.token_rows = torch.empty((T, k), **i32)
        self.num_rows = torch.zeros(1, **i32)
        self.capacity = cap
        self.struct = moe_layout()
        s = self.struct
        s.rank_offsets, s.send_counts = _p(self.rank_offsets), _p(self.send_counts)
        s.row_token, s.row_coef = _p(self.row_token), _p(self.row_coef)
        s.token_rows, s.num_rows, s.capacity = _p(self.token_rows), _p(self.num_rows), cap
        if mode == TWO_HOP:
            G = R // ranks_per_group
            cap1 = T * k if capacity_hop1 is None else capacity_hop1
            self.capacity_hop1 = cap1
            self.group_offsets = torch.zeros(G + 1, **i32)
            self.hop1_row_token = torch.empty(max(cap1, 1), **i32)
            self.token_groups = torch.empty((T, k), **i32)
            self.hop2_src_row = torch.empty(max(cap, 1), **i32)
            self.hop1_children = torch.empty((max(cap1, 1), k), **i32)
            self.num_rows_hop1 = torch.zeros(1, **i32)
            s.group_offsets, s.hop1_row_token = _p(self.group_offsets), _p(self.hop1_row_token)
            s.token_groups, s.hop2_src_row = _p(self.token_groups), _p(self.hop2_src_row)
            s.hop1_children, s.num_rows_hop1 = _p(self.hop1_children), _p(self.num_rows_hop1)
            s.capacity_hop1 = cap1
        else:
            self.capacity_hop1 = 0
        ws = layout_workspace_size(T, k, E, R, ranks_per_group, mode)
        if T > 0 and ws == 0:
            raise MoeError("moe_layout_workspace_size", 1)
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=device)

    def tokens(self, t0: int, t1: int) -> moe_layout:
        """A copy of the C struct for the token range [t0, t1), as moe_pack and
        moe_combine accept it: the token-indexed arrays start at token t0 and
        T = t1 - t0; the row-indexed arrays are shared."""
        if not 0 <= t0 <= t1 <= self.T:
            raise ValueError(f"token range [{t0}, {t1}) outside [0, {self.T})")
        s = moe_layout.from_buffer_copy(self.struct)
        s.T = t1 - t0
        if self.T > 0:
            s.token_rows = self.struct.token_rows + t0 * self.k * 4
            if self.mode == TWO_HOP:
                s.token_groups = self.struct.token_groups + t0 * self.k * 4
        return s


def build_layout(topk_idx, topk_w, expert_rank, layout: Layout, stream=None) -> Layout:
    _need(topk_idx, torch.int32, "topk_idx", 2)
    _need(topk_w, torch.float32, "topk_w", 2)
    _need(expert_rank, torch.int32, "expert_rank", 1)
    L = layout
    if tuple(topk_idx.shape) != (L.T, L.k) or expert_rank.numel() != L.E:
        raise ValueError("topk_idx / expert_rank do not match the layout's sizes")
    _check(lib().moe_build_layout(_p(topk_idx), _p(topk_w), _p(expert_rank), L.T, L.tokens_per_rank,
                                  L.k, L.E, L.R, L.ranks_per_group, L.mode, ctypes.byref(L.struct),
                                  _p(L.workspace), L.workspace.numel(), _stream(stream)),
           "moe_build_layout")
    return L


# ----------------------------------------------------------- pack/combine ----
def _token_slice(layout: Layout, t: torch.Tensor, tokens, name: str):
    """(struct, pointer) for the whole layout, or for a token range of it with
    the pointer of the [T][H] tensor t moved to the range's first token."""
    if t.shape[0] != layout.T:
        raise ValueError(f"{name} must have the layout's {layout.T} token rows")
    if tokens is None:
        return layout.struct, _p(t)
    t0, t1 = tokens
    s = layout.tokens(t0, t1)
    return s, _p(t) + t0 * t.shape[1] * t.element_size()


def pack(x: torch.Tensor, layout: Layout, packed=None, packed_hop1=None, stream=None, tokens=None):
    """tokens=(t0, t1): pack only that token range of x (the rows it fills are
    the same as in a full call)."""
    if x.dtype not in _DT:
        raise TypeError("x must be float16, bfloat16 or float32")
    _need(x, x.dtype, "x", 2)
    L = layout
    H = x.shape[1]
    if packed is None:
        packed = torch.empty((max(L.capacity, 1), H), dtype=x.dtype, device=x.device)
    if L.mode == TWO_HOP and packed_hop1 is None:
        packed_hop1 = torch.empty((max(L.capacity_hop1, 1), H), dtype=x.dtype, device=x.device)
    st, xp = _token_slice(L, x, tokens, "x")
    _check(lib().moe_pack(xp, _DT[x.dtype], H, ctypes.byref(st), _p(packed),
                          _p(packed_hop1), _stream(stream)), "moe_pack")
    return (packed, packed_hop1) if L.mode == TWO_HOP else packed


def combine(y: torch.Tensor, layout: Layout, out=None, out_dtype=None, row_coef=None,
            hop1_buf=None, stream=None, store_hop1: bool = True, tokens=None):
    """TWO_HOP: the group partials go to hop1_buf (allocated if None), or are
    not stored at all with store_hop1=False.  tokens=(t0, t1): combine only that
    token range into out[t0:t1]."""
    if y.dtype not in _DT:
        raise TypeError("y must be float16, bfloat16 or float32")
    _need(y, y.dtype, "y", 2)
    L = layout
    H = y.shape[1]
    out_dtype = y.dtype if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty((L.T, H), dtype=out_dtype, device=y.device)
    _need(out, out_dtype, "out", 2)
    if row_coef is not None:
        _need(row_coef, torch.float32, "row_coef", 1)
    if L.mode == TWO_HOP and hop1_buf is None and store_hop1:
        hop1_buf = torch.empty((max(L.capacity_hop1, 1), H), dtype=y.dtype, device=y.device)
    if not store_hop1:
        hop1_buf = None
    st, op = _token_slice(L, out, tokens, "out")
    _check(lib().moe_combine(_p(y), _DT[y.dtype], H, ctypes.byref(st), _p(row_coef), op,
                             _DT[out_dtype], _p(hop1_buf), _stream(stream)), "moe_combine")
    return out


# ------------------------------------------------------------- statistics ----
STAT_NAMES = ("expert_max_mean", "rank_gini", "rank_max_mean", "own_rank_row_share")


def dispatch_stats(counts: torch.Tensor, send_counts: torch.Tensor, out=None, stream=None):
    """The four statistics as a float64 device tensor [4] (see STAT_NAMES)."""
    _need(counts, torch.int32, "counts", 1)
    _need(send_counts, torch.int32, "send_counts")
    R = int(round(send_counts.numel() ** 0.5))
    if R * R != send_counts.numel():
        raise ValueError("send_counts must be R x R")
    out = torch.empty(4, dtype=torch.float64, device=counts.device) if out is None else out
    _need(out, torch.float64, "out", 1)
    _check(lib().moe_dispatch_stats(_p(counts), counts.numel(), _p(send_counts), R, _p(out),
                                    _stream(stream)), "moe_dispatch_stats")
    return out


def token_balanced_assign(counts, replica_offsets, replica_slots, slot_rank, R: int,
                          slot_tokens=None, rank_active=None, stream=None):
    for t, n in ((counts, "counts"), (replica_offsets, "replica_offsets"),
                 (replica_slots, "replica_slots"), (slot_rank, "slot_rank")):
        _need(t, torch.int32, n, 1)
    S = slot_rank.numel()
    dev = counts.device
    slot_tokens = torch.empty(S, dtype=torch.int32, device=dev) if slot_tokens is None else slot_tokens
    rank_active = torch.empty(R, dtype=torch.int32, device=dev) if rank_active is None else rank_active
    _check(lib().moe_token_balanced_assign(_p(counts), counts.numel(), _p(replica_offsets),
                                           _p(replica_slots), replica_slots.numel(), _p(slot_rank), S, R,
                                           _p(slot_tokens), _p(rank_active), _stream(stream)),
           "moe_token_balanced_assign")
    return slot_tokens, rank_active


def route_layout_single_replica(logits: torch.Tensor, k: int, expert_rank: torch.Tensor, layout: Layout,
                                n_groups: int = 0, groups_per_token: int = 0, renormalize: bool = False,
                                topk_idx=None, topk_w=None, counts=None, rank_active=None, stream=None):
    """route_topk + demand_hist + replica_assign + build_layout in one pass for
    placements with one replica per expert (expert_rank: that replica's rank)."""
    _need(logits, torch.float32, "logits", 2)
    _need(expert_rank, torch.int32, "expert_rank", 1)
    T, E = logits.shape
    L = layout
    if (T, k, E) != (L.T, L.k, L.E):
        raise ValueError("logits / k do not match the layout's sizes")
    dev = logits.device
    topk_idx = torch.empty((T, k), dtype=torch.int32, device=dev) if topk_idx is None else topk_idx
    topk_w = torch.empty((T, k), dtype=torch.float32, device=dev) if topk_w is None else topk_w
    counts = torch.empty(E, dtype=torch.int32, device=dev) if counts is None else counts
    _check(lib().moe_route_layout_single_replica(
        _p(logits), T, E, k, n_groups, groups_per_token, int(renormalize), _p(expert_rank),
        L.tokens_per_rank, L.R, L.ranks_per_group, L.mode, _p(topk_idx), _p(topk_w), _p(counts),
        _p(rank_active), ctypes.byref(L.struct), _p(L.workspace), L.workspace.numel(), _stream(stream)),
        "moe_route_layout_single_replica")
    return topk_idx, topk_w, counts


def route_assign_layout(logits: torch.Tensor, k: int, replica_offsets, replica_slots, slot_rank,
                        layout: Layout, n_groups: int = 0, groups_per_token: int = 0,
                        renormalize: bool = False, topk_idx=None, topk_w=None, counts=None,
                        expert_slot=None, expert_rank=None, rank_active=None, stream=None):
    """route_topk + demand_hist + replica_assign + build_layout in one launch, for
    any replica map.  Returns (topk_idx, topk_w, counts, expert_slot, expert_rank,
    rank_active)."""
    _need(logits, torch.float32, "logits", 2)
    for t, n in ((replica_offsets, "replica_offsets"), (replica_slots, "replica_slots"),
                 (slot_rank, "slot_rank")):
        _need(t, torch.int32, n, 1)
    T, E = logits.shape
    L = layout
    if (T, k, E) != (L.T, L.k, L.E):
        raise ValueError("logits / k do not match the layout's sizes")
    dev = logits.device
    i32 = dict(dtype=torch.int32, device=dev)
    topk_idx = torch.empty((T, k), **i32) if topk_idx is None else topk_idx
    topk_w = torch.empty((T, k), dtype=torch.float32, device=dev) if topk_w is None else topk_w
    counts = torch.empty(E, **i32) if counts is None else counts
    expert_slot = torch.empty(E, **i32) if expert_slot is None else expert_slot
    expert_rank = torch.empty(E, **i32) if expert_rank is None else expert_rank
    rank_active = torch.empty(L.R, **i32) if rank_active is None else rank_active
    _check(lib().moe_route_assign_layout(
        _p(logits), T, E, k, n_groups, groups_per_token, int(renormalize), _p(replica_offsets),
        _p(replica_slots), replica_slots.numel(), _p(slot_rank), slot_rank.numel(), L.tokens_per_rank,
        L.R, L.ranks_per_group, L.mode, _p(topk_idx), _p(topk_w), _p(counts), _p(expert_slot),
        _p(expert_rank), _p(rank_active), ctypes.byref(L.struct), _p(L.workspace), L.workspace.numel(),
        _stream(stream)), "moe_route_assign_layout")
    return topk_idx, topk_w, counts, expert_slot, expert_rank, rank_active


def coselection_hist(topk_idx: torch.Tensor, E: int, cosel=None, stream=None):
    _need(topk_idx, torch.int32, "topk_idx", 2)
    T, k = topk_idx.shape
    cosel = torch.empty((E, E), dtype=torch.int32, device=topk_idx.device) if cosel is None else cosel
    _need(cosel, torch.int32, "cosel")
    _check(lib().moe_coselection_hist(_p(topk_idx), T, k, E, _p(cosel), _stream(stream)),
           "moe_coselection_hist")
    return cosel


def correlated_placement(cosel: torch.Tensor, counts: torch.Tensor, R: int, expert_rank=None, stream=None):
    _need(cosel, torch.int32, "cosel", 2)
    _need(counts, torch.int32, "counts", 1)
    E = counts.numel()
    expert_rank = torch.empty(E, dtype=torch.int32, device=counts.device) if expert_rank is None else expert_rank
    _check(lib().moe_correlated_placement(_p(cosel), _p(counts), E, R, _p(expert_rank), _stream(stream)),
           "moe_correlated_placement")
    return expert_rank
