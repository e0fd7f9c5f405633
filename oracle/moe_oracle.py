"""Plain CPU oracle for the on-device MoE dispatch/combine path.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, links or runs
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use it.  It
shares no code with the CUDA library; it takes plain numpy arrays (drawn by
the ``workloads`` generators) and returns numpy arrays.

Every step is written from its definition, in float64 for floating point, with
numpy's library primitives (stable sort, fancy indexing, sums) as steps and no
blocking, fusion or reordering beyond the definition:

1. ``route_topk``      per-token softmax over all E experts and top-k by
   logit, ties to the lower expert index; optional group-limited routing.
2. ``demand_hist``     global per-expert count of top-k selections.
3. ``replica_assign``  METRO greedy: each active expert to one replica on the
   rank with the fewest already-activated experts.
4. ``build_layout``    stable (destination, token) row order, per-destination
   offsets, send-count matrix, per-row combine coefficients; PER_PICK, DEDUP
   (single send per rank) and TWO_HOP (group, then rank in group).
5. ``pack``            row gather ``P[row] = X[row_token[row]]``.
6. ``combine``         ``out[t] = sum over t's rows of coef * Y[row]``.

Pins (in ``tests/``, marked ``not gpu``) tie each function to the pages and to
mathematics other than itself: closed forms, library routines on special
cases, brute force on tiny inputs, and the pages' worked numbers.  No function
here is "parity unpinned".
"""
from __future__ import annotations

import itertools
from typing import Dict, Optional, Sequence

import numpy as np

PER_PICK = 0
DEDUP = 1
TWO_HOP = 2


# --------------------------------------------------------------------------
# rounding to the storage formats (round to nearest, ties to even)
# --------------------------------------------------------------------------
_FORMATS = {           # (explicit mantissa bits, minimum normal exponent, max finite)
    "f16": (10, -14, 65504.0),
    "bf16": (7, -126, 3.3895313892515355e38),
    "f32": (23, -126, 3.4028234663852886e38),
}


def round_to(x: np.ndarray, fmt: str) -> np.ndarray:
    """Round float64 values to the nearest value of a binary format, ties to even.

    The textbook definition: with ``e = floor(log2 |x|)`` clamped below at the
    format's minimum normal exponent (which gives the subnormal spacing), the
    spacing is ``q = 2**(e - mantissa_bits)`` and the result is
    ``rint(x / q) * q`` (``rint`` rounds halves to even).  Scaling by a power of
    two is exact in float64, so only the ``rint`` step rounds.  Returns float64.
    """
    mbits, emin, vmax = _FORMATS[fmt]
    x = np.asarray(x, np.float64)
    assert np.all(np.isfinite(x)), "non-finite value"
    _, ex = np.frexp(x)                      # x = m * 2**ex, 0.5 <= |m| < 1
    e = np.maximum(ex.astype(np.int64) - 1, emin)
    q = np.ldexp(1.0, (e - mbits).astype(np.int32))
    r = np.rint(x / q) * q
    r = np.where(x == 0, x, r)
    assert np.all(np.abs(r) <= vmax), "overflow in round_to"
    return r


def ulp(x: np.ndarray, fmt: str) -> np.ndarray:
    """Spacing of the format at |x| (the subnormal spacing below the normal range)."""
    mbits, emin, _ = _FORMATS[fmt]
    x = np.abs(np.asarray(x, np.float64))
    _, ex = np.frexp(x)
    e = np.maximum(ex.astype(np.int64) - 1, emin)
    return np.ldexp(1.0, (e - mbits).astype(np.int32))


# --------------------------------------------------------------------------
# 1. router softmax + top-k
# --------------------------------------------------------------------------
def softmax(logits: np.ndarray) -> np.ndarray:
    """Row softmax in float64: exp(l - max) / sum exp(l - max)."""
    l = np.asarray(logits, np.float64)
    z = np.exp(l - l.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def route_topk(logits: np.ndarray, k: int, n_groups: int = 0,
               groups_per_token: int = 0, renormalize: bool = False):
    """Top-k gate of each token over the gathered token set.

    "METRO AllGather vs AllToAll for MoE decode", section "changes the routing
    information": every rank sees the full token set and computes the top-k
    expert choices of every token.  Selection is on the logits (the softmax is
    monotone, so the order is the same in exact arithmetic), descending, ties
    to the lower expert index (a stable sort of the negated logits).  The gate
    weight of a pick is its softmax probability over all E experts; with
    ``renormalize`` the k weights are divided by their sum.

    Group-limited routing (TerraceMoE editorial, "The core problem": a routing
    constraint that fixes per-token fan-out and a per-selected-group quota):
    experts form ``n_groups`` contiguous blocks; a group's score is its largest
    logit; each token keeps its ``groups_per_token`` best groups (ties to the
    lower group) and takes its top-k among their experts only.  The softmax
    stays over all E experts.

    Returns ``idx`` int32 [T][k] and ``w`` float64 [T][k].
    """
    logits = np.asarray(logits, np.float32)
    assert np.all(np.isfinite(logits)), "logits must be finite"
    T, E = logits.shape
    assert 1 <= k <= E
    p = softmax(logits)
    cand = logits.astype(np.float64)
    if groups_per_token and groups_per_token < n_groups:
        gs = E // n_groups
        assert gs * n_groups == E and groups_per_token * gs >= k
        score = cand.reshape(T, n_groups, gs).max(axis=2)
        gorder = np.argsort(-score, axis=1, kind="stable")
        keep = np.zeros((T, n_groups), bool)
        np.put_along_axis(keep, gorder[:, :groups_per_token], True, axis=1)
        cand = np.where(np.repeat(keep, gs, axis=1), cand, -np.inf)
    order = np.argsort(-cand, axis=1, kind="stable")
    idx = order[:, :k].astype(np.int32)
    w = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    if renormalize:
        w = w / w.sum(axis=1, keepdims=True)
    return idx, w


# --------------------------------------------------------------------------
# 2. global expert demand vector
# --------------------------------------------------------------------------
def demand_hist(idx: np.ndarray, E: int) -> np.ndarray:
    """counts[e] = number of (token, pick) pairs that selected expert e.

    "METRO AllGather vs AllToAll for MoE decode", section "changes the routing
    information": the global expert demand vector, the same on every rank.
    """
    counts = np.zeros(E, np.int64)
    np.add.at(counts, np.asarray(idx, np.int64).ravel(), 1)
    return counts


# --------------------------------------------------------------------------
# 3. METRO greedy replica assignment
# --------------------------------------------------------------------------
def replica_assign(counts, replica_offsets, replica_slots, slot_rank, R: int):
    """METRO greedy assignment of active experts to replicas.

    "METRO AllGather vs AllToAll for MoE decode", sections "changes the routing
    information" and "Add the expert-weight traffic term": each active expert
    (demand > 0) is assigned to one of its replicas, on the GPU with the
    lowest count of already-activated experts; the greedy does not solve the
    optimal min-max assignment.  Readings where the page is silent: experts are
    visited in ascending id; ties go to the lower rank, then the lower slot id;
    every replica is available.

    Returns ``expert_slot``, ``expert_rank`` (int32 [E], -1 for inactive
    experts) and ``rank_active`` (int64 [R]).
    """
    counts = np.asarray(counts)
    E = counts.shape[0]
    expert_slot = np.full(E, -1, np.int32)
    expert_rank = np.full(E, -1, np.int32)
    rank_active = np.zeros(R, np.int64)
    for e in range(E):
        if counts[e] == 0:
            continue
        slots = [int(s) for s in replica_slots[replica_offsets[e]:replica_offsets[e + 1]]]
        assert slots, f"active expert {e} has no replica"
        best = min(slots, key=lambda s: (rank_active[slot_rank[s]], int(slot_rank[s]), s))
        expert_slot[e] = best
        expert_rank[e] = slot_rank[best]
        rank_active[slot_rank[best]] += 1
    return expert_slot, expert_rank, rank_active


def optimal_max_active(counts, replica_offsets, replica_slots, slot_rank, R: int) -> int:
    """Brute force over every replica choice: the minimum possible max activated
    experts per rank (the "expensive optimal assignment" the page contrasts
    with the greedy).  Tiny inputs only.  Pinned by hand-worked optima (one
    where the greedy is strictly worse), the page's toy example and a
    bipartite-matching optimum computed by a library routine."""
    active = [e for e in range(len(counts)) if counts[e] > 0]
    choices = [sorted({int(slot_rank[s]) for s in replica_slots[replica_offsets[e]:replica_offsets[e + 1]]})
               for e in active]
    best = None
    for pick in itertools.product(*choices):
        load = np.bincount(np.asarray(pick, np.int64), minlength=R) if pick else np.zeros(R, np.int64)
        m = int(load.max())
        best = m if best is None else min(best, m)
    return 0 if best is None else best


def token_balanced_split(counts, replica_offsets, replica_slots, slot_rank, R: int, S: int):
    """Token-balanced routing, the comparison policy of "METRO AllGather vs
    AllToAll for MoE decode" (sections "Add the expert-weight traffic term" and
    "Know what the paper actually measured": EPLB token routing, which spreads
    an expert's tokens over its replicas).  The c tokens of expert e are dealt
    round-robin over its n replicas in ascending slot id, so the i-th replica
    gets floor(c / n) + (1 if i < c mod n else 0) tokens; a replica with at
    least one token is activated.

    Returns ``slot_tokens`` (int64 [S]) and ``rank_active`` (int64 [R])."""
    slot_tokens = np.zeros(S, np.int64)
    act = np.zeros(R, np.int64)
    for e in range(len(counts)):
        c = int(counts[e])
        slots = sorted(int(s) for s in replica_slots[replica_offsets[e]:replica_offsets[e + 1]])
        if c <= 0 or not slots:
            continue
        n = len(slots)
        for i, s in enumerate(slots):
            slot_tokens[s] = c // n + (1 if i < c % n else 0)
            if slot_tokens[s] > 0:
                act[slot_rank[s]] += 1
    return slot_tokens, act


def token_balanced_active(counts, replica_offsets, replica_slots, slot_rank, R: int) -> np.ndarray:
    """Activated replicas per rank under token-balanced routing (above)."""
    S = int(np.max(np.asarray(replica_slots), initial=-1)) + 1
    return token_balanced_split(counts, replica_offsets, replica_slots, slot_rank, R, S)[1]


# --------------------------------------------------------------------------
# correlated expert placement
# --------------------------------------------------------------------------
def coselection(idx: np.ndarray, E: int) -> np.ndarray:
    """C[e][f] = number of tokens that picked both e and f (e != f); symmetric,
    zero diagonal.  The co-selection statistics behind correlated expert
    placement (ainewsletter summary of arXiv:2610.09372, "Correlations in
    router choices": 0.8% of expert pairs jointly selected by 42% of tokens)."""
    idx = np.asarray(idx, np.int64)
    C = np.zeros((E, E), np.int64)
    T, k = idx.shape
    for i in range(k):
        for j in range(k):
            if i != j:
                np.add.at(C, (idx[:, i], idx[:, j]), 1)
    return C


def correlated_placement(C: np.ndarray, counts: np.ndarray, R: int) -> np.ndarray:
    """Place experts that are often selected together on the same rank
    (same summary, "Two locality techniques").  The page gives no algorithm;
    this grows one rank at a time, E/R experts each: the rank is seeded with
    the unplaced expert of highest demand, then takes the unplaced expert that
    shares the most co-selections with the rank's experts so far, until full
    (ties: higher demand, then the lower id).

    Returns expert_rank (int32 [E])."""
    E = C.shape[0]
    assert E % R == 0
    cap = E // R
    rank = np.full(E, -1, np.int64)
    for r in range(R):
        free = [e for e in range(E) if rank[e] < 0]
        seed = max(free, key=lambda e: (int(counts[e]), -e))
        rank[seed] = r
        aff = np.asarray(C[:, seed], np.int64).copy()          # co-selections with the rank
        for _ in range(cap - 1):
            free = [e for e in range(E) if rank[e] < 0]
            nxt = max(free, key=lambda e: (int(aff[e]), int(counts[e]), -e))
            rank[nxt] = r
            aff += C[:, nxt]
    return rank.astype(np.int32)


# --------------------------------------------------------------------------
# dispatch statistics of the send-count matrix
# --------------------------------------------------------------------------
def gini(x) -> float:
    """Gini coefficient: sum over all ordered pairs |x_i - x_j| / (2 n^2 mean);
    0 when every value is 0."""
    x = np.asarray(x, np.float64)
    n, tot = x.shape[0], x.sum()
    if n == 0 or tot == 0:
        return 0.0
    return float(np.abs(x[:, None] - x[None, :]).sum() / (2.0 * n * n * (tot / n)))


def dispatch_stats(counts, send_counts) -> Dict[str, float]:
    """Scalar summaries of one dispatch (gist.science summary of DODOCO,
    "Methodology": the per-expert max/mean ratio measures routing skew
    independent of the expert-to-rank map; the Gini coefficient measures
    per-rank load imbalance).  Per-rank load = rows each destination rank
    receives (column sums of the send-count matrix S).  Also the share of rows
    that stay on their source rank (the diagonal of S)."""
    counts = np.asarray(counts, np.float64)
    S = np.asarray(send_counts, np.float64)
    load = S.sum(axis=0)
    return {
        "expert_max_mean": float(counts.max() / counts.mean()) if counts.sum() else 0.0,
        "rank_gini": gini(load),
        "rank_max_mean": float(load.max() / load.mean()) if load.sum() else 0.0,
        "own_rank_row_share": float(np.trace(S) / S.sum()) if S.sum() else 0.0,
    }


# --------------------------------------------------------------------------
# 4. layout
# --------------------------------------------------------------------------
def build_layout(idx: np.ndarray, w: np.ndarray, expert_rank: np.ndarray,
                 tokens_per_rank: int, R: int, mode: int,
                 ranks_per_group: int = 0) -> Dict[str, np.ndarray]:
    """Per-destination send layout of the gathered token set.

    Rows (the AllToAll-v destination chunks of "METRO AllGather vs AllToAll
    for MoE decode", section "Distinguish METRO from backend names"):

    * PER_PICK: one row per (token, pick), ordered by (destination rank,
      expert, token).
    * DEDUP: one row per (destination rank, token) with the rank in the token's
      destination set -- the single-send dispatcher of the arXiv:2610.09372
      summary ("Two locality techniques") -- ordered by (rank, token).  The row
      carries the sum of the token's gate weights on that rank.
    * TWO_HOP (TerraceMoE editorial, "The core problem"): hop-1 rows per
      (group, token), ordered by (group, token), with group = rank //
      ranks_per_group; hop-2 rows are the DEDUP rows, and each reads from the
      hop-1 row of its own group and token.

    ``token_rows[t]`` lists t's (hop-2) rows in ascending row id, -1 padded to
    k; ``send_counts[src][dst]`` counts the rows from source rank
    ``t // tokens_per_rank`` to ``dst``.
    """
    idx = np.asarray(idx, np.int64)
    T, k = idx.shape
    dst = np.asarray(expert_rank, np.int64)[idx]                  # [T][k]
    assert np.all((dst >= 0) & (dst < R)), "picked expert without a rank"
    assert tokens_per_rank >= 1 and tokens_per_rank * R >= T, "source rank out of range"
    tok = np.repeat(np.arange(T, dtype=np.int64), k)
    pd, pe, pw = dst.ravel(), idx.ravel(), np.asarray(w, np.float64).ravel()
    out: Dict[str, np.ndarray] = {}
    if mode == PER_PICK:
        order = np.lexsort((tok, pe, pd))                        # by (dst, e, t)
        row_token, row_dst, row_coef = tok[order], pd[order], pw[order]
        out["row_expert"] = pe[order].astype(np.int32)
        row_of_pick = np.empty(T * k, np.int64)
        row_of_pick[order] = np.arange(T * k)
        token_rows = np.sort(row_of_pick.reshape(T, k), axis=1)
    elif mode in (DEDUP, TWO_HOP):
        key = pd * T + tok                                        # (dst, t)
        uniq, inv = np.unique(key, return_inverse=True)           # sorted by (dst, t)
        row_dst, row_token = uniq // T, uniq % T
        row_coef = np.zeros(uniq.shape[0], np.float64)
        np.add.at(row_coef, inv, pw)                              # sum of t's weights on dst
        token_rows = _rows_per_token(row_token, T, k)
    else:
        raise ValueError(mode)
    n = row_token.shape[0]
    out["num_rows"] = np.int64(n)
    out["row_token"] = row_token.astype(np.int32)
    out["row_dst"] = row_dst.astype(np.int32)
    out["row_coef"] = row_coef
    out["token_rows"] = token_rows.astype(np.int32)
    off = np.zeros(R + 1, np.int64)
    off[1:] = np.cumsum(np.bincount(row_dst, minlength=R))
    out["rank_offsets"] = off.astype(np.int32)
    sc = np.zeros((R, R), np.int64)
    np.add.at(sc, (row_token // tokens_per_rank, row_dst), 1)
    out["send_counts"] = sc.astype(np.int32)
    if mode == TWO_HOP:
        rpg = ranks_per_group
        assert rpg >= 1 and R % rpg == 0
        G = R // rpg
        gkey = np.unique((pd // rpg) * T + tok)                   # (group, t), sorted
        h1_group, h1_token = gkey // T, gkey % T
        out["num_rows_hop1"] = np.int64(gkey.shape[0])
        out["hop1_row_token"] = h1_token.astype(np.int32)
        out["hop1_group"] = h1_group.astype(np.int32)
        goff = np.zeros(G + 1, np.int64)
        goff[1:] = np.cumsum(np.bincount(h1_group, minlength=G))
        out["group_offsets"] = goff.astype(np.int32)
        out["token_groups"] = _rows_per_token(h1_token, T, k).astype(np.int32)
        # hop-2 row (dst, t) reads hop-1 row (dst // rpg, t)
        src_key = (row_dst // rpg) * T + row_token
        out["hop2_src_row"] = np.searchsorted(gkey, src_key).astype(np.int32)
        # each hop-1 row's hop-2 rows, ascending
        out["hop1_children"] = _rows_per_token(out["hop2_src_row"].astype(np.int64),
                                               gkey.shape[0], k).astype(np.int32)
    return out


def _rows_per_token(row_token: np.ndarray, T: int, width: int) -> np.ndarray:
    """For each token, its row ids in ascending order, -1 padded to ``width``."""
    order = np.argsort(row_token, kind="stable")                  # rows grouped by token, ascending id
    cnt = np.bincount(row_token, minlength=T)
    start = np.zeros(T + 1, np.int64)
    start[1:] = np.cumsum(cnt)
    res = np.full((T, width), -1, np.int64)
    pos = np.arange(order.shape[0]) - start[row_token[order]]
    res[row_token[order], pos] = order
    return res


def own_rank_share(idx: np.ndarray, expert_rank: np.ndarray, tokens_per_rank: int) -> float:
    """Share of token->expert assignments served on the token's own rank
    (arXiv:2610.09372 summary, "Two locality techniques": 12.5% on one node
    of 8 without token shuffling)."""
    idx = np.asarray(idx, np.int64)
    home = np.arange(idx.shape[0])[:, None] // tokens_per_rank
    return float(np.mean(np.asarray(expert_rank)[idx] == home))


# --------------------------------------------------------------------------
# 5. pack
# --------------------------------------------------------------------------
def pack(x: np.ndarray, row_token: np.ndarray, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Send buffer rows: ``P[row] = X[row_token[row]]`` (a bit copy).

    The local half of the AllToAll dispatch ("METRO AllGather vs AllToAll for
    MoE decode", section "Work the 8-GPU payload example": AllToAll splits each
    rank's input into per-destination chunks).  ``rows`` restricts the result
    to a sample of rows.  Works on any dtype, including raw uint16 bit views.
    """
    rt = np.asarray(row_token, np.int64)
    if rows is not None:
        rt = rt[np.asarray(rows, np.int64)]
    return np.asarray(x)[rt]


# --------------------------------------------------------------------------
# 6. combine
# --------------------------------------------------------------------------
def combine(y: np.ndarray, token_rows: np.ndarray, coef: np.ndarray,
            tokens: Optional[Sequence[int]] = None) -> np.ndarray:
    """Weighted combine back to token order, in float64.

    ``out[t] = sum over t's rows i, in ascending row order, of coef[i] * Y[i]``
    (the combine after the experts in "METRO AllGather vs AllToAll for MoE
    decode", section "changes the routing information").  ``y`` holds float
    values (upcast by the caller from f16/bf16/f32); ``tokens`` restricts the
    result to a sample of tokens.  Returns float64 [len(tokens)][H].
    """
    tr = np.asarray(token_rows, np.int64)
    if tokens is not None:
        tr = tr[np.asarray(tokens, np.int64)]
    coef = np.asarray(coef, np.float64)
    out = np.zeros((tr.shape[0], y.shape[1]), np.float64)
    for j in range(tr.shape[1]):
        r = tr[:, j]
        m = r >= 0
        out[m] += coef[r[m]][:, None] * np.asarray(y[r[m]], np.float64)
    return out


def combine_two_hop(y2: np.ndarray, layout: Dict[str, np.ndarray], coef: np.ndarray,
                    wire_fmt: str, tokens: Optional[Sequence[int]] = None):
    """Two-hop reverse: rank rows into group rows, then group rows into tokens.

    TerraceMoE editorial, "The core problem": dispatch goes by group and then
    by rank in the group, and the combine runs in reverse.  The group partial
    ``z(g, t) = sum over t's rank rows in g of coef * Y2`` would cross the
    slow fabric, so it is rounded to the activation dtype ``wire_fmt``;
    ``out[t] = sum over t's group rows of z``.  Returns (out float64, z float64
    for the hop-1 rows touched).
    """
    T = layout["token_rows"].shape[0]
    toks = np.arange(T) if tokens is None else np.asarray(tokens, np.int64)
    tr = layout["token_rows"][toks].astype(np.int64)
    tg = layout["token_groups"][toks].astype(np.int64)
    src = layout["hop2_src_row"].astype(np.int64)
    coef = np.asarray(coef, np.float64)
    H = y2.shape[1]
    out = np.zeros((toks.shape[0], H), np.float64)
    zs = {}
    for gi in range(tg.shape[1]):
        r1 = tg[:, gi]
        z = np.zeros((toks.shape[0], H), np.float64)
        for j in range(tr.shape[1]):
            r2 = tr[:, j]
            m = (r1 >= 0) & (r2 >= 0)
            m[m] = src[r2[m]] == r1[m]
            z[m] += coef[r2[m]][:, None] * np.asarray(y2[r2[m]], np.float64)
        have = r1 >= 0
        z[have] = round_to(z[have], wire_fmt)
        out[have] += z[have]
        for t_i in np.nonzero(have)[0]:
            zs[int(r1[t_i])] = z[t_i]
    return out, zs


# --------------------------------------------------------------------------
# byte accounting of the exchange the layout stands for
# --------------------------------------------------------------------------
def dispatch_bytes_per_rank(send_counts: np.ndarray, H: int, elem_bytes: int) -> np.ndarray:
    """Bytes each source rank puts into its AllToAll(-v) send buffer:
    rows it sends (own rank included) x H x bytes per element.
    ("METRO AllGather vs AllToAll for MoE decode", section "Work the 8-GPU
    payload example": AllToAll splits each rank's input into destination chunks.)"""
    return np.asarray(send_counts, np.int64).sum(axis=1) * H * elem_bytes


def allgather_bytes_per_rank(tokens_per_rank: int, R: int, H: int, elem_bytes: int) -> int:
    """Bytes of the gathered token set on every rank: AllGather of N values
    from each of R ranks yields R x N values everywhere (same section)."""
    return R * tokens_per_rank * H * elem_bytes


def link_time_us(nbytes: float, GBps: float) -> float:
    """Ideal transfer time of a payload at a link bandwidth, decimal units."""
    return nbytes / (GBps * 1e9) * 1e6
