/*
 * moe.h -- C ABI of the on-device MoE expert-parallel dispatch/combine path
 * (libmoe.so, hand-written CUDA for sm_100a).
 *
 * The path: per-token router softmax + top-k over a gathered token set, a
 * global per-expert demand histogram, METRO greedy assignment of each active
 * expert to one replica, a stable per-destination row layout (with per-rank
 * dedup, and a two-hop group/rank variant), a pack of token rows into
 * contiguous per-rank send buffers, and the weighted combine back to token
 * order.  Expert-parallel ranks are logical partitions of one GPU's memory.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every array argument is DEVICE memory owned by the caller; the library
 *   never allocates, frees or keeps a pointer after the call returns.  The
 *   moe_layout struct itself is HOST memory; the pointers inside it are device
 *   memory.
 * - Calls are asynchronous and ordered on `stream` (NULL = the legacy default
 *   stream).  Nothing synchronises except moe_get_status().
 * - Row-major, densely packed arrays; int32 indices; float32 weights.
 * - Errors a host can see (null pointer, size out of range, unsupported
 *   combination) return a non-zero moe_status BEFORE anything is launched.
 *   A failed launch returns MOE_ERR_CUDA.  Errors only the device can see
 *   (bad index in an input, capacity exceeded, a bounded wait that ran out)
 *   are recorded in a per-device status word (first error wins), and the
 *   offending element is skipped; moe_get_status() reads and clears it.
 * - The library keeps, per device, the device addresses of its own status
 *   word (and of the scratch array of moe_build_layout_static), looked up on
 *   the first call on that device.  It is not usable across cudaDeviceReset:
 *   a reset destroys the context those addresses belong to.
 * - Limits: 1 <= E <= 1024; 1 <= k <= min(E, 16); 1 <= R <= 64;
 *   T * k < 2^31; replica slots S <= 32768; H * element size a multiple of
 *   16 bytes; n_groups <= 32.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

struct CUstream_st;                       /* same type as cudaStream_t */
typedef struct CUstream_st *moe_stream_t;

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* host-checked: null pointer, size or enum out of range */
  MOE_ERR_UNSUPPORTED = 2,  /* host-checked: outside the library's limits */
  MOE_ERR_CUDA = 3,         /* a CUDA runtime call or a launch failed */
  MOE_ERR_TIMEOUT = 4,      /* device: a bounded wait ran out (outputs invalid) */
  MOE_ERR_BOUNDS = 5,       /* device: an index outside its buffer was skipped */
  MOE_ERR_BAD_INPUT = 6,    /* device: non-finite logit, expert/slot/rank id out of
                               range, or an active expert without a replica */
  MOE_ERR_CAPACITY = 7      /* device: more rows than `capacity`; rows past it dropped */
} moe_status;

typedef enum moe_dtype { MOE_F16 = 0, MOE_BF16 = 1, MOE_F32 = 2 } moe_dtype;

typedef enum moe_layout_mode {
  MOE_LAYOUT_PER_PICK = 0,  /* one row per (token, pick), ordered (rank, expert, token) */
  MOE_LAYOUT_DEDUP = 1,     /* one row per (rank, token): single send per rank */
  MOE_LAYOUT_TWO_HOP = 2    /* hop 1 per (group, token), hop 2 per (rank, token) */
} moe_layout_mode;

/*
 * Row layout of one dispatch.  The caller allocates every buffer and sets the
 * pointers and capacities; moe_build_layout fills the buffers (on the device)
 * and the shape fields (on the host).
 *
 * Rows: see moe_build_layout.  "Hop-2 rows" below means the rank rows of
 * TWO_HOP; for PER_PICK and DEDUP they are simply the rows.
 */
typedef struct moe_layout {
  int32_t *rank_offsets;   /* [R+1] first row of each destination rank; [R] = rows */
  int32_t *send_counts;    /* [R*R] rows from source rank s to rank d at s*R+d;
                              source rank of token t = t / tokens_per_rank */
  int32_t *row_token;      /* [capacity] token each row carries */
  float   *row_coef;       /* [capacity] combine coefficient of each row: the gate
                              weight of the pick (PER_PICK) or the sum of the
                              token's gate weights on that rank (DEDUP, TWO_HOP) */
  int32_t *token_rows;     /* [T*k] rows of token t in ascending order, -1 padded */
  int32_t *num_rows;       /* [1] total rows (may exceed capacity: see MOE_ERR_CAPACITY) */
  int32_t  capacity;       /* rows the row_* buffers hold; T*k is always enough */
  /* TWO_HOP only; ignored (may be NULL / 0) for the other modes */
  int32_t *group_offsets;  /* [G+1] first hop-1 row of each group, G = R / ranks_per_group */
  int32_t *hop1_row_token; /* [capacity_hop1] token of each hop-1 row */
  int32_t *token_groups;   /* [T*k] hop-1 rows of token t in ascending order, -1 padded */
  int32_t *hop2_src_row;   /* [capacity] hop-1 row each hop-2 row is forwarded from */
  int32_t *hop1_children;  /* [capacity_hop1 * k] hop-2 rows forwarded from each hop-1
                              row, ascending, -1 padded */
  int32_t *num_rows_hop1;  /* [1] total hop-1 rows */
  int32_t  capacity_hop1;
  /* written by moe_build_layout, read by moe_pack / moe_combine */
  int32_t  T, k, R, E, ranks_per_group, mode;
} moe_layout;

/*
 * Router softmax + top-k.  One token per warp; large token sets (at least
 * 128 tokens per SM) with E = 64, 128 or 256, k <= 8, no group limit or
 * n_groups dividing 16, and 16-byte aligned logits take one token per thread
 * instead, with bit-identical results.
 * Source: "METRO AllGather vs AllToAll for MoE decode" (fanout.sh), section
 * "changes the routing information": every rank computes the top-k expert
 * choices of the full gathered token set.  Group-limited routing: TerraceMoE
 * editorial (lyndhub), section "The core problem" (a routing constraint that
 * fixes per-token fan-out and a per-selected-group quota).
 *
 * logits    [T][E] float32, finite (a non-finite logit sets MOE_ERR_BAD_INPUT)
 * topk_idx  [T][k] int32 out: experts by descending logit, ties to the lower id
 * topk_w    [T][k] float32 out: softmax probability over all E experts of each
 *           pick (divided by the sum of the k picks when renormalize != 0)
 * n_groups, groups_per_token: 0 = no limit.  Otherwise experts form n_groups
 *           contiguous groups (n_groups | E, n_groups <= 32), a group scores its
 *           largest logit, the token keeps its best groups_per_token groups
 *           (ties to the lower group) and picks top-k among their experts;
 *           groups_per_token * E / n_groups >= k.
 */
MOE_API int moe_route_topk(const float *logits, int32_t T, int32_t E, int32_t k,
                   int32_t n_groups, int32_t groups_per_token, int32_t renormalize,
                   int32_t *topk_idx, float *topk_w, moe_stream_t stream);

/*
 * Global per-expert demand vector: counts[e] = number of (token, pick) pairs
 * with topk_idx == e.  Source: same page, same section ("the same global
 * expert demand vector").  counts [E] int32 is zeroed by the call; ids outside
 * [0, E) are skipped and set MOE_ERR_BAD_INPUT.
 */
MOE_API int moe_demand_hist(const int32_t *topk_idx, int32_t T, int32_t k, int32_t E,
                    int32_t *counts, moe_stream_t stream);

/*
 * METRO greedy replica assignment (one CTA; the serial part walks only the
 * experts with more than one valid replica).  Source: same page, sections
 * "changes the routing information" and "Add the expert-weight traffic term":
 * each active expert goes to one of its replicas on the rank with the fewest
 * already-activated experts.  Experts are visited in ascending id; ties go to
 * the lower rank, then the lower slot id.
 *
 * counts          [E]   demand vector (active = count > 0)
 * replica_offsets [E+1] CSR: slots of expert e are replica_slots[off[e]..off[e+1])
 * replica_slots   [S']  slot ids in [0, S)
 * slot_rank       [S]   rank hosting each slot, in [0, R)
 * expert_slot     [E]   out: chosen slot, -1 for inactive experts
 * expert_rank     [E]   out: rank of the chosen slot, -1 for inactive experts
 * rank_active     [R]   out: activated experts per rank
 * An active expert with no valid replica gets -1 and sets MOE_ERR_BAD_INPUT.
 */
MOE_API int moe_replica_assign(const int32_t *counts, int32_t E, const int32_t *replica_offsets,
                       const int32_t *replica_slots, int32_t n_replica_entries,
                       const int32_t *slot_rank, int32_t S, int32_t R,
                       int32_t *expert_slot, int32_t *expert_rank, int32_t *rank_active,
                       moe_stream_t stream);

/* Bytes of device scratch moe_build_layout needs for these sizes (0 on bad args). */
MOE_API size_t moe_layout_workspace_size(int32_t T, int32_t k, int32_t E, int32_t R,
                                 int32_t ranks_per_group, int32_t mode);

/*
 * Stable per-destination row layout (one cooperative launch: per-block bin
 * counts, a bounded grid barrier, then each block's prefix from the count
 * table and its rows; at most 512 tokens in the DEDUP and TWO_HOP modes take
 * one pass instead, every block counting every token, with no barrier and
 * without touching the workspace).
 * Sources: the AllToAll(-v) destination chunks of "METRO AllGather vs AllToAll
 * for MoE decode", sections "Work the 8-GPU payload example" and "Distinguish
 * METRO from backend names"; the single-send dispatcher of the ainewsletter
 * summary of arXiv:2610.09372, section "Two locality techniques"; the two-hop
 * dispatch of the TerraceMoE editorial, section "The core problem".
 *
 * Destination rank of a pick = expert_rank[topk_idx].
 *  PER_PICK: rows (rank, expert, token) for every pick, in that order.
 *  DEDUP:    rows (rank, token) for every rank in the token's destination set,
 *            ordered by (rank, token); row_coef = sum of the token's gate
 *            weights on that rank, added in ascending pick order (float32).
 *  TWO_HOP:  hop-2 rows as DEDUP; hop-1 rows (group, token) with group =
 *            rank / ranks_per_group, ordered by (group, token);
 *            hop2_src_row of hop-2 row (rank, t) = hop-1 row (rank / rpg, t).
 * topk_idx [T][k], topk_w [T][k], expert_rank [E] (from moe_replica_assign).
 * tokens_per_rank: source rank of token t is t / tokens_per_rank (< R).
 * workspace: device scratch of moe_layout_workspace_size() bytes, 16-byte
 * aligned; its contents on entry do not matter.  It holds the launch's grid
 * barrier, so calls whose executions overlap on the GPU (other streams, other
 * host threads) need workspaces of their own.  The kernel is a cooperative
 * launch sized to the blocks that fit on the GPU at once; its barrier waits
 * are bounded (MOE_ERR_TIMEOUT).  Fills every buffer of `layout` and its shape
 * fields.  Rows past layout->capacity are dropped (their token_rows entries
 * are -1) and set MOE_ERR_CAPACITY.
 */
MOE_API int moe_build_layout(const int32_t *topk_idx, const float *topk_w, const int32_t *expert_rank,
                     int32_t T, int32_t tokens_per_rank, int32_t k, int32_t E, int32_t R,
                     int32_t ranks_per_group, int32_t mode, moe_layout *layout,
                     void *workspace, size_t workspace_bytes, moe_stream_t stream);

/*
 * moe_build_layout without a workspace argument.  The paper has no
 * counterpart: this is a convenience of this library.
 *
 * Some callers cannot allocate device memory on the call path -- a serving
 * loop that reserves all of its memory at start-up and allows no allocation
 * per request, or a host framework that hands a library only its existing
 * input and output buffers and exposes no allocator -- so they cannot supply
 * the scratch workspace moe_build_layout needs.  This variant takes its
 * scratch from a fixed array of MOE_LAYOUT_STATIC_SCRATCH_BYTES in device
 * memory that the library reserves when it is loaded (every GPU that loads the
 * library holds it until the process exits) and calls no allocator.
 *
 * Arguments, outputs and device-side errors are those of moe_build_layout.
 * Returns MOE_ERR_UNSUPPORTED, before anything is launched, when
 * moe_layout_workspace_size() for these sizes exceeds
 * MOE_LAYOUT_STATIC_SCRATCH_BYTES (for example 65536 tokens over 64 ranks
 * needs 135 KB in DEDUP mode; 65536 tokens over 256 experts, 528 KB in
 * PER_PICK mode).  The first call on a device looks up the array's device
 * address with that device current and keeps it; make that first call before
 * any stream capture (a first call on a capturing stream returns
 * MOE_ERR_UNSUPPORTED and launches nothing).  All calls share the one array, whose contents
 * persist from call to call (each call clears what must start at zero):
 * calls whose executions overlap on the GPU -- on different streams, or from
 * different host threads -- race on it and must be serialised by the caller.
 */
#define MOE_LAYOUT_STATIC_SCRATCH_BYTES (1u << 20)
MOE_API int moe_build_layout_static(const int32_t *topk_idx, const float *topk_w,
                                    const int32_t *expert_rank, int32_t T, int32_t tokens_per_rank,
                                    int32_t k, int32_t E, int32_t R, int32_t ranks_per_group,
                                    int32_t mode, moe_layout *layout, moe_stream_t stream);

/*
 * Pack: packed[row] = x[row_token[row]] for every row (a bit copy), token
 * major: each token row is read once and written to each of its rows.
 * Source: the local half of the AllToAll dispatch ("METRO AllGather vs
 * AllToAll for MoE decode", section "Work the 8-GPU payload example").
 * x [T][H] of `dtype`; packed [capacity][H].  TWO_HOP: packed_hop1
 * [capacity_hop1][H] receives the hop-1 (group) rows and packed the hop-2
 * (rank) rows, which equal the group rows they are forwarded from; both are
 * written from one read of each token.  packed_hop1 is ignored otherwise.
 * Token ranges: pack reads only layout->T, k, mode, capacities, token_rows and
 * token_groups (rows [0, T) of each) and writes absolute rows, so a copy of the
 * layout with T = t1 - t0 and token_rows / token_groups advanced by t0 * k,
 * given x advanced by t0 rows, packs tokens [t0, t1) exactly as a whole call
 * would; calls on disjoint ranges may run in any order.
 */
MOE_API int moe_pack(const void *x, int32_t dtype, int32_t H, const moe_layout *layout,
             void *packed, void *packed_hop1, moe_stream_t stream);

/*
 * Combine: out[t] = sum over t's rows i, ascending, of coef[i] * y[i],
 * accumulated in float32 and rounded to nearest-even into out_dtype.
 * Source: the combine after the experts ("METRO AllGather vs AllToAll for MoE
 * decode", section "changes the routing information").
 * y [capacity][H] of `dtype` (expert outputs, one per row); row_coef [capacity]
 * or NULL for layout->row_coef; out [T][H] of out_dtype.
 * TWO_HOP: the reverse of the two hops, in one pass per token.  Each group
 * partial, the sum over the group's rank rows in ascending order, is rounded to
 * `dtype` (the dtype that would cross the slow fabric); out[t] = the sum of t's
 * rounded group partials in ascending group order.  hop1_buf [capacity_hop1][H]
 * of `dtype` receives the group partials at their hop-1 rows, or is NULL to
 * skip storing them.  hop1_buf is ignored for the other modes.
 * Token ranges as for moe_pack: a layout copy with T = t1 - t0 and token_rows
 * advanced by t0 * k, with out advanced by t0 rows, combines tokens [t0, t1)
 * (row_coef, hop2_src_row and the row buffers are indexed by absolute row).
 */
MOE_API int moe_combine(const void *y, int32_t dtype, int32_t H, const moe_layout *layout,
                const float *row_coef, void *out, int32_t out_dtype, void *hop1_buf,
                moe_stream_t stream);

/*
 * moe_route_topk, moe_demand_hist, moe_replica_assign and moe_build_layout in
 * one pass, for placements with exactly one replica per expert.  Source: with
 * a single replica, the METRO assignment of "METRO AllGather vs AllToAll for
 * MoE decode" (sections "changes the routing information" and "Add the
 * expert-weight traffic term") has no choice to make, so each pick's
 * destination rank is known as soon as the pick is; one cooperative kernel
 * routes the tokens while counting the demand vector and the layout's bins,
 * and after its grid barrier writes the layout's rows and the send matrix.
 * Every output equals that of the separate calls.
 * expert_rank [E]: rank of each expert's only replica (every entry in [0, R);
 * a pick of an expert outside it sets MOE_ERR_BAD_INPUT and is skipped).
 * counts [E] out: the demand vector.  rank_active [R] out, or NULL: activated
 * experts per rank.  topk_idx, topk_w, the layout and the workspace as in
 * moe_route_topk and moe_build_layout.
 */
MOE_API int moe_route_layout_single_replica(
    const float *logits, int32_t T, int32_t E, int32_t k, int32_t n_groups,
    int32_t groups_per_token, int32_t renormalize, const int32_t *expert_rank,
    int32_t tokens_per_rank, int32_t R, int32_t ranks_per_group, int32_t mode, int32_t *topk_idx,
    float *topk_w, int32_t *counts, int32_t *rank_active, moe_layout *layout, void *workspace,
    size_t workspace_bytes, moe_stream_t stream);

/*
 * moe_route_topk, moe_demand_hist, moe_replica_assign and moe_build_layout in
 * one launch, for any replica map.  Source: "METRO AllGather vs AllToAll for
 * MoE decode", section "changes the routing information" (every rank computes
 * the global routing, the demand vector and the assignment: at decode sizes
 * their launch cost is what the global information costs).  One cooperative
 * kernel routes the tokens and counts the demand vector; after a grid barrier
 * every block runs the METRO greedy over it (the same deterministic result in
 * each, written out by block 0) and builds its part of the layout, with one
 * more grid barrier unless the layout takes one pass (at most 512 tokens,
 * DEDUP or TWO_HOP).  Every output equals that of the four separate calls.
 * Arguments as in those calls; the workspace is moe_layout_workspace_size()
 * bytes as for moe_build_layout.  Returns MOE_ERR_UNSUPPORTED, before anything
 * is launched, if one block's shared memory cannot hold the replica map and
 * the layout bins (within the limits of moe_replica_assign and
 * moe_build_layout they take at most 173 KB).
 */
MOE_API int moe_route_assign_layout(
    const float *logits, int32_t T, int32_t E, int32_t k, int32_t n_groups, int32_t groups_per_token,
    int32_t renormalize, const int32_t *replica_offsets, const int32_t *replica_slots,
    int32_t n_replica_entries, const int32_t *slot_rank, int32_t S, int32_t tokens_per_rank, int32_t R,
    int32_t ranks_per_group, int32_t mode, int32_t *topk_idx, float *topk_w, int32_t *counts,
    int32_t *expert_slot, int32_t *expert_rank, int32_t *rank_active, moe_layout *layout,
    void *workspace, size_t workspace_bytes, moe_stream_t stream);

/*
 * Co-selection counts: cosel[e*E + f] = number of tokens whose picks include
 * both e and f (e != f); symmetric, zero diagonal; zeroed by the call.
 * Source: the ainewsletter summary of arXiv:2610.09372, "Correlations in
 * router choices" (experts jointly selected by the same tokens).
 * topk_idx [T][k] (distinct experts per token); cosel [E*E] int32 out.
 */
MOE_API int moe_coselection_hist(const int32_t *topk_idx, int32_t T, int32_t k, int32_t E,
                                 int32_t *cosel, moe_stream_t stream);

/*
 * Correlated expert placement (one CTA).  Source: same summary, "Two locality
 * techniques": experts often selected together go to the same GPU, so that a
 * single-send dispatcher sends fewer rows.  The page gives no algorithm; this
 * one grows the ranks one at a time, E/R experts each (R | E): the rank is
 * seeded with the unplaced expert of highest demand, then takes the unplaced
 * expert with the most co-selections with the rank's experts so far (ties:
 * higher demand, then the lower id).
 * cosel [E*E] symmetric (as moe_coselection_hist writes it), counts [E] (the
 * demand vector), expert_rank [E] out: a placement with one replica per expert.
 */
MOE_API int moe_correlated_placement(const int32_t *cosel, const int32_t *counts, int32_t E,
                                     int32_t R, int32_t *expert_rank, moe_stream_t stream);

/*
 * Statistics of one dispatch (one CTA).  Source: gist.science summary of
 * DODOCO, "Methodology": the per-expert max/mean ratio measures routing skew
 * independent of the expert-to-rank map; the Gini coefficient measures
 * per-rank load imbalance.  Per-rank load = rows each destination rank
 * receives (column sums of send_counts).
 * counts [E] (demand vector), send_counts [R*R] (from moe_build_layout).
 * stats [4] float64 out: per-expert max/mean, Gini of the per-rank load
 * (sum over ordered pairs |x_i - x_j| / (2 R^2 mean)), per-rank max/mean, and
 * the share of rows that stay on their source rank; 0 when there is no load.
 */
MOE_API int moe_dispatch_stats(const int32_t *counts, int32_t E, const int32_t *send_counts,
                               int32_t R, double *stats, moe_stream_t stream);

/*
 * Token-balanced replica routing, the comparison policy of "METRO AllGather vs
 * AllToAll for MoE decode" (sections "Add the expert-weight traffic term" and
 * "Know what the paper actually measured": EPLB token routing).  Each
 * expert's c tokens are dealt round-robin over its n valid replicas in
 * ascending slot id: the i-th gets floor(c / n) + (i < c mod n) tokens.  A
 * replica with a token is activated.  Map arguments as moe_replica_assign.
 * slot_tokens [S] out (0 for slots of inactive experts), rank_active [R] out.
 */
MOE_API int moe_token_balanced_assign(const int32_t *counts, int32_t E,
                                      const int32_t *replica_offsets, const int32_t *replica_slots,
                                      int32_t n_replica_entries, const int32_t *slot_rank, int32_t S,
                                      int32_t R, int32_t *slot_tokens, int32_t *rank_active,
                                      moe_stream_t stream);

/*
 * Synchronises `stream`, then returns and clears the device status word of the
 * current device (MOE_OK if no device-side error was recorded since the last
 * call).  The word is shared by every stream on the device.
 */
MOE_API int moe_get_status(moe_stream_t stream);

/*
 * Number of kernels this library has launched in this process (all devices,
 * all streams), counted on the host at each successful launch.  Memsets and
 * copies are not kernels and are not counted.
 */
MOE_API uint64_t moe_kernel_launches(void);

/* Static string naming a moe_status value. */
MOE_API const char *moe_status_string(int status);

/*
 * Test hook for the bounded waits.  wait_limit_ns: limit of every device-side
 * wait started after this call (0 restores the default of one second).
 * layout_silent_tile: index of one block of the layout launches (moe_build_layout
 * and moe_route_layout_single_replica) that never arrives at the grid barrier
 * (-1 = none), so that the other blocks' waits run out and report
 * MOE_ERR_TIMEOUT instead of hanging.  Host-side settings, read at launch.
 */
MOE_API int moe_debug_set_wait(uint64_t wait_limit_ns, int32_t layout_silent_tile);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
