// Pieces of the layout shared by the layout kernel (build_layout.cu) and the
// one-launch front ends (route_layout_static.cu, route_assign_layout.cu):
// arguments, the shared-memory plan, per-token pick loading, warp bin
// ballots, the grid barrier (counted in rounds, so one launch can pass several),
// and the two phases that turn picks into bin counts and bin counts into rows.
//
// One launch, two phases.  Every block owns a contiguous chunk of tokens.
// Phase 1 counts the rows of every bin ("bins" are ranks for DEDUP, ranks then
// groups for TWO_HOP, experts for PER_PICK) over the block's chunk and stores
// the counts in its row of the workspace.  After a grid barrier every block
// reads all blocks' counts: their sum per bin gives the segment offsets, the
// sum over earlier blocks its own base in every bin.  Phase 2 then walks the
// chunk again in tiles of 256 tokens; within a tile a warp's ballot of a bin
// gives both the bin's count in the warp and each lane's position (token
// order), and one thread per bin scans the warps.  The grid is sized so that
// every block is resident at once (cooperative launch) and the barrier wait is
// bounded.
#pragma once

#include "moe_internal.cuh"

namespace moe {
namespace layout {

constexpr int kTile = 256;  // threads per block, tokens per phase-2 tile
constexpr int kWarps = kTile / 32;
constexpr int kMaxBlocks = 512;  // grid cap (rows of the count table)
constexpr int kBlocksPerSm = 2;  // layout grid: blocks per SM (when resident)
constexpr int kHeaderInts = 16 + kMaxE;  // workspace header: barrier words, then a demand scratch
constexpr unsigned kFull = 0xffffffffu;

struct LayoutArgs {
  const int *idx;
  const float *w;
  const int *expert_rank;
  int T, tpr, k, E, R, rpg, G, mode, NB, NBp;
  int nblk;        // blocks of the launch
  int chunk;       // tokens per block, a multiple of 8
  unsigned *bar;   // [0] barrier arrivals, [1] blocks done
  int *cnt;        // [E] demand scratch of the fused front ends (cleared with the barrier words)
  int *agg;        // [nblk][NBp] per-block bin counts
  moe_layout L;
};

// Shared memory of one block, in ints.
struct SmemPlan {
  int er, cnt, base, w, woff, ptot, ppre, seg, send, hist, total;
};

__host__ __device__ inline SmemPlan smem_plan(int E, int NBp, int R, bool fused) {
  SmemPlan s;
  int o = 0;
  s.er = o;   o += (E + 3) & ~3;
  s.cnt = o;  o += NBp;           // block counts, then per-bin totals
  s.base = o; o += NBp;           // running row base of every bin
  s.w = o;    o += kWarps * NBp;  // per-warp ballots (mask bins) or counts (experts)
  s.woff = o; o += kWarps * NBp;  // per-warp row offsets (mask bins)
  s.ptot = o; o += 1024;          // partial sums of the count table
  s.ppre = o; o += 1024;
  s.seg = o;  o += NBp + 2 * kMaxR + 4;  // segment offsets, rank totals and bases
  s.send = o; o += R * R;         // the block's send-count matrix
  s.hist = o; o += fused ? ((E + 3) & ~3) : 0;
  s.total = o;
  return s;
}

// ---------------------------------------------------------------- tokens ----
// One token's picks as seen by one thread.
template <int KM>
struct TokenPicks {
  int e[KM];
  int r[KM];
  float w[KM];
  uint32_t present;          // picks with a valid expert and rank
  unsigned long long dmask;  // ranks of the token
  unsigned long long gmask;  // groups of the token (TWO_HOP)
};

template <int KM, int MODE>
__device__ __forceinline__ void load_picks(const LayoutArgs &a, const int *s_er, int t, bool live,
                                           bool want_w, TokenPicks<KM> &p, bool &bad) {
  p.present = 0;
  p.dmask = 0;
  p.gmask = 0;
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    p.e[j] = 0;
    p.r[j] = 0;
    p.w[j] = 0.0f;
    if (j < a.k && live) {
      const int e = a.idx[(size_t)t * a.k + j];
      if ((unsigned)e < (unsigned)a.E) {
        const int r = s_er[e];
        if ((unsigned)r < (unsigned)a.R) {
          p.e[j] = e;
          p.r[j] = r;
          p.present |= 1u << j;
          p.dmask |= 1ull << r;
          p.gmask |= 1ull << (r / a.rpg);
          if (want_w) p.w[j] = a.w[(size_t)t * a.k + j];
        } else {
          bad = true;
        }
      } else {
        bad = true;
      }
    }
  }
  if (MODE == MOE_LAYOUT_PER_PICK) {  // the row order needs distinct experts per token
#pragma unroll
    for (int i = 0; i < KM; ++i)
#pragma unroll
      for (int j = i + 1; j < KM; ++j)
        if ((p.present >> i & 1u) && (p.present >> j & 1u) && p.e[i] == p.e[j]) {
          bad = true;
          p.present &= ~(1u << j);
        }
  }
}

__device__ __forceinline__ unsigned long long warp_or64(unsigned long long m) {
  const unsigned lo = __reduce_or_sync(kFull, (unsigned)m);
  const unsigned hi = __reduce_or_sync(kFull, (unsigned)(m >> 32));
  return ((unsigned long long)hi << 32) | lo;
}

__device__ __forceinline__ unsigned long long group_bits(int g, int rpg) {
  const unsigned long long ones = (rpg >= 64) ? ~0ull : ((1ull << rpg) - 1ull);
  return (rpg >= 64) ? ones : (ones << (g * rpg));
}

// The warp's ballots of bins [0, n) (n <= 64) of a 64-bit mask per lane:
// lane i gets the ballots of bins i (b0) and i + 32 (b1).
__device__ __forceinline__ void warp_bin_ballots(unsigned long long m, int n, int lane,
                                                 unsigned &b0, unsigned &b1) {
  b0 = 0;
  b1 = 0;
  const unsigned lo = (unsigned)m, hi = (unsigned)(m >> 32);
  const int n0 = n < 32 ? n : 32;
#pragma unroll 8
  for (int i = 0; i < n0; ++i) {
    const unsigned bal = __ballot_sync(kFull, (lo >> i) & 1u);
    if (lane == i) b0 = bal;
  }
#pragma unroll 8
  for (int i = 32; i < n; ++i) {
    const unsigned bal = __ballot_sync(kFull, (hi >> (i - 32)) & 1u);
    if (lane == i - 32) b1 = bal;
  }
}

// ------------------------------------------------------------- experts ----
// Merge the lanes' distinct (rank << 10 | expert) keys in ascending order.  For
// every key present in the warp, f(key, has, ball, c, matched) runs on all
// lanes: `has` says whether this lane's token has the key, `ball` which lanes
// do, `c` how many distinct keys this lane had before, `matched` its picks
// with the key.
template <int KM, class F>
__device__ __forceinline__ void warp_merge(const TokenPicks<KM> &p, F &&f) {
  uint32_t key[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) key[j] = ((uint32_t)p.r[j] << 10) | (uint32_t)p.e[j];
  uint32_t rem = p.present;
  int c = 0;
  while (true) {
    uint32_t mine = 0xffffffffu;
#pragma unroll
    for (int j = 0; j < KM; ++j)
      if (rem >> j & 1u) mine = min(mine, key[j]);
    const uint32_t b = __reduce_min_sync(kFull, mine);
    if (b == 0xffffffffu) break;
    const bool has = (mine == b);
    const unsigned ball = __ballot_sync(kFull, has);
    uint32_t matched = 0;
#pragma unroll
    for (int j = 0; j < KM; ++j)
      if ((rem >> j & 1u) && key[j] == b) matched |= 1u << j;
    f(b, has, ball, c, matched);
    if (has) {
      rem &= ~matched;
      ++c;
    }
  }
}

// ------------------------------------------------------------- phase 1 ----
// One warp's ballots of the mask bins: lane i holds those of ranks i, i + 32
// (b0, b1) and of groups i, i + 32 (g0, g1).
struct Ballots {
  unsigned b0, b1, g0, g1;
};

// The warp's ballots of its tokens' ranks (and groups); a warp with no live
// token skips the ballots (all zero).
template <int MODE>
__device__ __forceinline__ Ballots mask_ballots(const LayoutArgs &a, unsigned long long dmask,
                                                unsigned long long gmask, bool live, int lane) {
  Ballots bl{0u, 0u, 0u, 0u};
  if (!__any_sync(kFull, live)) return bl;
  warp_bin_ballots(dmask, a.R, lane, bl.b0, bl.b1);
  if (MODE == MOE_LAYOUT_TWO_HOP) warp_bin_ballots(gmask, a.G, lane, bl.g0, bl.g1);
  return bl;
}

// Adds one tile's bin counts of this warp into lane-held totals: c[0], c[1]
// for ranks lane and lane + 32, c[2], c[3] for groups lane and lane + 32
// (mask modes; the tile's ballots are returned in bl); experts go straight
// to the block counts (PER_PICK).
template <int KM, int MODE>
__device__ __forceinline__ void count_tile(const LayoutArgs &a, const TokenPicks<KM> &p, bool live,
                                           int lane, int *s_cnt, int (&c)[4], Ballots &bl) {
  if (MODE == MOE_LAYOUT_PER_PICK) {
    warp_merge<KM>(p, [&](uint32_t b, bool, unsigned ball, int, uint32_t) {
      if (lane == 0) atomicAdd(&s_cnt[b & 1023u], __popc(ball));
    });
    return;
  }
  bl = mask_ballots<MODE>(a, p.dmask, p.gmask, live, lane);
  c[0] += __popc(bl.b0);
  c[1] += __popc(bl.b1);
  c[2] += __popc(bl.g0);
  c[3] += __popc(bl.g1);
}

// Moves the lane-held mask-bin totals into the block counts.
template <int MODE>
__device__ __forceinline__ void flush_counts(const LayoutArgs &a, int lane, int *s_cnt,
                                             const int (&c)[4]) {
  if (MODE == MOE_LAYOUT_PER_PICK) return;
  if (lane < a.R && c[0]) atomicAdd(&s_cnt[lane], c[0]);
  if (lane + 32 < a.R && c[1]) atomicAdd(&s_cnt[lane + 32], c[1]);
  if (MODE == MOE_LAYOUT_TWO_HOP) {
    if (lane < a.G && c[2]) atomicAdd(&s_cnt[a.R + lane], c[2]);
    if (lane + 32 < a.G && c[3]) atomicAdd(&s_cnt[a.R + lane + 32], c[3]);
  }
}

// ------------------------------------------------------------- barrier ----
__device__ __forceinline__ void red_release_add(unsigned *p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid-wide barrier over the launch's blocks (all resident: cooperative
// launch); `round` counts the barriers of the launch from 1 (each block adds
// one arrival per round).  Returns false on every thread of the block when the
// wait ran out (MOE_ERR_TIMEOUT is set) or the block is the test hook's silent
// block, which never arrives.
__device__ __forceinline__ bool grid_barrier(const LayoutArgs &a, const DeviceCtx &ctx, int *s_flag,
                                             unsigned round = 1) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned target = round * (unsigned)a.nblk;
    if ((int)blockIdx.x == ctx.silent_tile) {
      ok = 0;
    } else {
      red_release_add(a.bar, 1u);
      if (ld_acquire_u32(a.bar) < target) {
        const uint64_t t0 = global_ns();
        while (ld_acquire_u32(a.bar) < target) {
          __nanosleep(32);
          if (global_ns() - t0 > ctx.wait_limit_ns || ld_volatile_i32(ctx.status) == MOE_ERR_TIMEOUT) {
            set_status(ctx.status, MOE_ERR_TIMEOUT);
            ok = 0;
            break;
          }
        }
      }
    }
    *s_flag = ok;
  }
  __syncthreads();
  return *s_flag != 0;
}

// ------------------------------------------------------------- phase 2 ----
// Per-bin totals (into s_cnt) and this block's base (into s_base) from the
// count table.
__device__ __forceinline__ void gather_counts(const LayoutArgs &a, const SmemPlan &P, int *sm) {
  const int tid = threadIdx.x;
  const int V = a.NBp / 4;                      // 16-byte vectors per table row
  const int Q = V >= kTile ? 1 : kTile / V;     // row groups
  int *s_cnt = sm + P.cnt, *s_base = sm + P.base, *s_ptot = sm + P.ptot, *s_ppre = sm + P.ppre;
  const int blk = blockIdx.x;
  for (int x = tid; x < Q * V; x += kTile) {
    const int q = x / V, v = x % V;
    int4 tot = make_int4(0, 0, 0, 0), pre = make_int4(0, 0, 0, 0);
#pragma unroll 8
    for (int g = q; g < a.nblk; g += Q) {
      const int4 c = __ldcg(reinterpret_cast<const int4 *>(a.agg + (size_t)g * a.NBp) + v);
      tot.x += c.x; tot.y += c.y; tot.z += c.z; tot.w += c.w;
      if (g < blk) {
        pre.x += c.x; pre.y += c.y; pre.z += c.z; pre.w += c.w;
      }
    }
    reinterpret_cast<int4 *>(s_ptot + q * a.NBp)[v] = tot;
    reinterpret_cast<int4 *>(s_ppre + q * a.NBp)[v] = pre;
  }
  __syncthreads();
  // the Q partial rows summed per bin: with few bins (Q >= 32 partial rows) G
  // threads per bin (a power of two <= 32), each over every G-th row, then a
  // shuffle tree; with many bins one thread per bin
  const int G = a.NB > 32 ? 1 : min(32, 1 << (31 - __clz(kTile / a.NB)));
  for (int b0 = 0; b0 < a.NB; b0 += kTile / G) {  // uniform trip count over the block
    const int b = b0 + tid / G, sub = tid % G;
    int tot = 0, pre = 0;
    if (b < a.NB)
      for (int q = sub; q < Q; q += G) {
        tot += s_ptot[q * a.NBp + b];
        pre += s_ppre[q * a.NBp + b];
      }
    for (int d = G >> 1; d > 0; d >>= 1) {
      tot += __shfl_down_sync(kFull, tot, d, G);
      pre += __shfl_down_sync(kFull, pre, d, G);
    }
    if (b < a.NB && sub == 0) {
      s_cnt[b] = tot;
      s_base[b] = pre;
    }
  }
  __syncthreads();
}

// Segment offsets from the per-bin totals (s_cnt); every bin's running base
// (s_base, the rows of the bin before this block) moves past them.  Block 0
// writes the layout's offsets and row counts.
template <int MODE>
__device__ __forceinline__ void segment_offsets(const LayoutArgs &a, const SmemPlan &P, int *sm,
                                                DeviceCtx ctx) {
  const int tid = threadIdx.x, blk = blockIdx.x;
  int *s_cnt = sm + P.cnt, *s_base = sm + P.base;

  // segment offsets
  int *s_seg = sm + P.seg;
  int *s_rtot = s_seg + a.NBp;    // PER_PICK: rows per rank
  int *s_rbase = s_rtot + kMaxR;  // PER_PICK: first row of each rank
  const int *s_er = sm + P.er;
  const moe_layout &L = a.L;
  const int lane = tid & 31;
  if (MODE == MOE_LAYOUT_PER_PICK) {
    if (tid < a.R) {  // each rank walks its experts in ascending order
      int run = 0;
      for (int e = 0; e < a.E; ++e)
        if (s_er[e] == tid) {
          s_seg[e] = run;
          run += s_cnt[e];
        }
      s_rtot[tid] = run;
    }
    __syncthreads();
    if (tid < 32) {  // exclusive scan of the rank totals (R <= 64)
      const int v0 = lane < a.R ? s_rtot[lane] : 0, v1 = lane + 32 < a.R ? s_rtot[lane + 32] : 0;
      int i0 = v0, i1 = v1;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int n0 = __shfl_up_sync(kFull, i0, d), n1 = __shfl_up_sync(kFull, i1, d);
        if (lane >= d) {
          i0 += n0;
          i1 += n1;
        }
      }
      const int tot0 = __shfl_sync(kFull, i0, 31);
      const int tot1 = __shfl_sync(kFull, i1, 31);  // every lane takes part
      if (lane < a.R) s_rbase[lane] = i0 - v0;
      if (lane + 32 < a.R) s_rbase[lane + 32] = tot0 + i1 - v1;
      if (lane == 0) s_rbase[kMaxR] = tot0 + tot1;
    }
    __syncthreads();
    for (int e = tid; e < a.E; e += kTile) {
      const int r = s_er[e];
      s_seg[e] = ((unsigned)r < (unsigned)a.R) ? s_seg[e] + s_rbase[r] : 0;
    }
    if (blk == 0) {
      for (int r = tid; r <= a.R; r += kTile) L.rank_offsets[r] = r < a.R ? s_rbase[r] : s_rbase[kMaxR];
      if (tid == 0) {
        const int n = s_rbase[kMaxR];
        *L.num_rows = n;
        if (n > L.capacity) set_status(ctx.status, MOE_ERR_CAPACITY);
      }
    }
  } else if (tid < 32) {
    // exclusive scans of the rank totals and of the group totals (<= 64 each)
    for (int part = 0; part < (MODE == MOE_LAYOUT_TWO_HOP ? 2 : 1); ++part) {
      const int n = part ? a.G : a.R, off = part ? a.R : 0;
      const int v0 = lane < n ? s_cnt[off + lane] : 0, v1 = lane + 32 < n ? s_cnt[off + lane + 32] : 0;
      int i0 = v0, i1 = v1;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int n0 = __shfl_up_sync(kFull, i0, d), n1 = __shfl_up_sync(kFull, i1, d);
        if (lane >= d) {
          i0 += n0;
          i1 += n1;
        }
      }
      const int tot0 = __shfl_sync(kFull, i0, 31);
      const int total = tot0 + __shfl_sync(kFull, i1, 31);
      if (lane < n) s_seg[off + lane] = i0 - v0;
      if (lane + 32 < n) s_seg[off + lane + 32] = tot0 + i1 - v1;
      if (blk == 0) {
        int *offs = part ? L.group_offsets : L.rank_offsets;
        if (lane < n) offs[lane] = i0 - v0;
        if (lane + 32 < n) offs[lane + 32] = tot0 + i1 - v1;
        if (lane == 0) {
          offs[n] = total;
          if (part == 0) {
            *L.num_rows = total;
            if (total > L.capacity) set_status(ctx.status, MOE_ERR_CAPACITY);
          } else {
            *L.num_rows_hop1 = total;
            if (total > L.capacity_hop1) set_status(ctx.status, MOE_ERR_CAPACITY);
          }
        }
      }
    }
  }
  __syncthreads();
  for (int b = tid; b < a.NB; b += kTile) s_base[b] += s_seg[b];
  __syncthreads();
}

// Adds one tile's rows to the block's send-count matrix: source rank of the
// token -> its ranks (lane i holds the warp's ballots of ranks i, i + 32).
__device__ __forceinline__ void add_send_counts(const LayoutArgs &a, const SmemPlan &P, int *sm,
                                                unsigned long long dmask, const Ballots &bl, int t,
                                                bool live) {
  const int lane = threadIdx.x & 31;
  int *s_send = sm + P.send;
  const int src = live ? t / a.tpr : 0;
  const int src0 = __shfl_sync(kFull, src, 0);
  if (__all_sync(kFull, !live || src == src0)) {
    if (bl.b0) atomicAdd(&s_send[src0 * a.R + lane], __popc(bl.b0));
    if (bl.b1) atomicAdd(&s_send[src0 * a.R + lane + 32], __popc(bl.b1));
  } else {
    for (unsigned long long m = dmask; m; m &= m - 1)
      atomicAdd(&s_send[src * a.R + __ffsll((long long)m) - 1], 1);
  }
}

// Rows of one tile of mask-bin tokens (DEDUP, TWO_HOP).  Every thread of the
// block calls it; `t` is the thread's token, `live` whether it has one.
template <int KM, int MODE, bool SEND>
__device__ __forceinline__ void rows_mask_tile(const LayoutArgs &a, const SmemPlan &P, int *sm,
                                               const TokenPicks<KM> &p, const Ballots &bl, int t,
                                               bool live, bool &over) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int *s_w = sm + P.w + warp * a.NBp;
  const int *s_woff = sm + P.woff + warp * a.NBp;
  const unsigned b0 = bl.b0, b1 = bl.b1;
  if (lane < a.R) s_w[lane] = b0;
  if (lane + 32 < a.R) s_w[lane + 32] = b1;
  if (MODE == MOE_LAYOUT_TWO_HOP) {
    if (lane < a.G) s_w[a.R + lane] = bl.g0;
    if (lane + 32 < a.G) s_w[a.R + lane + 32] = bl.g1;
  }
  if (SEND) add_send_counts(a, P, sm, p.dmask, bl, t, live);
  __syncthreads();
  int *s_base = sm + P.base;
  for (int b = tid; b < a.NB; b += kTile) {
    int run = s_base[b];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      sm[P.woff + w * a.NBp + b] = run;
      run += __popc((unsigned)sm[P.w + w * a.NBp + b]);
    }
    s_base[b] = run;
  }
  __syncthreads();

  const moe_layout &L = a.L;
  const unsigned lt = lanemask_lt();
  const size_t tk = (size_t)t * a.k;
  auto row_of = [&](int bin) { return s_woff[bin] + __popc((unsigned)s_w[bin] & lt); };
  if (MODE == MOE_LAYOUT_TWO_HOP) {
    int cg = 0;
    for (unsigned long long m = p.gmask; m; m &= m - 1, ++cg) {
      const int g = __ffsll((long long)m) - 1;
      const int row1 = row_of(a.R + g);
      if (row1 < L.capacity_hop1) {
        L.hop1_row_token[row1] = t;
        L.token_groups[tk + cg] = row1;
        const int nchild = __popcll(p.dmask & group_bits(g, a.rpg));
        for (int ci = nchild; ci < a.k; ++ci) L.hop1_children[(size_t)row1 * a.k + ci] = -1;
      } else {
        L.token_groups[tk + cg] = -1;
        over = true;
      }
    }
    if (live)
      for (int c = cg; c < a.k; ++c) L.token_groups[tk + c] = -1;
  }
  int c = 0;
  for (unsigned long long m = p.dmask; m; m &= m - 1, ++c) {
    const int r = __ffsll((long long)m) - 1;
    const int row = row_of(r);
    float coef = 0.0f;
#pragma unroll
    for (int j = 0; j < KM; ++j)
      if ((p.present >> j & 1u) && p.r[j] == r) coef += p.w[j];
    const bool fits = row < L.capacity;
    if (fits) {
      L.row_token[row] = t;
      L.row_coef[row] = coef;
      L.token_rows[tk + c] = row;
    } else {
      L.token_rows[tk + c] = -1;
      over = true;
    }
    if (MODE == MOE_LAYOUT_TWO_HOP) {
      const int g = r / a.rpg;
      int row1 = row_of(a.R + g);
      if (row1 >= L.capacity_hop1) row1 = -1;
      const int ci = __popcll(p.dmask & group_bits(g, a.rpg) & ((1ull << r) - 1ull));
      if (fits) L.hop2_src_row[row] = row1;
      if (row1 >= 0) L.hop1_children[(size_t)row1 * a.k + ci] = fits ? row : -1;
    }
  }
  if (live)
    for (int cc = c; cc < a.k; ++cc) L.token_rows[tk + cc] = -1;
  __syncthreads();  // s_w and s_woff are reused by the next tile
}

// Rows of one tile of PER_PICK tokens: rows (rank, expert, token).
template <int KM>
__device__ __forceinline__ void rows_pick_tile(const LayoutArgs &a, const SmemPlan &P, int *sm,
                                               const TokenPicks<KM> &p, int t, bool live, bool &over) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kWarps * a.NBp; i += kTile) sm[P.w + i] = 0;
  __syncthreads();
  int *s_w = sm + P.w + warp * a.NBp;
  int *s_send = sm + P.send;
  const int src = live ? t / a.tpr : 0;
  const int src0 = __shfl_sync(kFull, src, 0);
  const bool uniform = __all_sync(kFull, !live || src == src0);
  warp_merge<KM>(p, [&](uint32_t b, bool has, unsigned ball, int, uint32_t) {
    if (lane == 0) s_w[b & 1023u] = __popc(ball);
    if (!has) return;
    const unsigned peers = uniform ? ball : __match_any_sync(ball, src);
    if (lane == __ffs(peers) - 1) atomicAdd(&s_send[src * a.R + (int)(b >> 10)], __popc(peers));
  });
  __syncthreads();
  int *s_base = sm + P.base;
  for (int b = tid; b < a.NB; b += kTile) {
    int run = s_base[b];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int c = sm[P.w + w * a.NBp + b];
      sm[P.w + w * a.NBp + b] = run;
      run += c;
    }
    s_base[b] = run;
  }
  __syncthreads();
  const moe_layout &L = a.L;
  const unsigned lt = lanemask_lt();
  const size_t tk = (size_t)t * a.k;
  int cnt = 0;
  warp_merge<KM>(p, [&](uint32_t b, bool has, unsigned ball, int c, uint32_t matched) {
    if (!has) return;
    const int row = s_w[b & 1023u] + __popc(ball & lt);
    float coef = 0.0f;
#pragma unroll
    for (int j = 0; j < KM; ++j)
      if (matched >> j & 1u) coef += p.w[j];
    if (row < L.capacity) {
      L.row_token[row] = t;
      L.row_coef[row] = coef;
      L.token_rows[tk + c] = row;
    } else {
      L.token_rows[tk + c] = -1;
      over = true;
    }
    cnt = c + 1;
  });
  if (live)
    for (int c = cnt; c < a.k; ++c) L.token_rows[tk + c] = -1;
  __syncthreads();
}

// Phase 2 of the block's chunk [t0, t1) once the barrier has passed.  `pre`
// and `pre_bl`: the thread's picks (with weights) and its warp's ballots kept
// from phase 1 when the chunk is one tile, else null (loaded again, tile by
// tile).
template <int KM, int MODE, bool SEND>
__device__ __forceinline__ void rows_loop(const LayoutArgs &a, const SmemPlan &P, int *sm, int t0,
                                          int t1, DeviceCtx ctx, const TokenPicks<KM> *pre,
                                          const Ballots *pre_bl) {
  bool over = false, bad = false;
  const int lane = threadIdx.x & 31;
  for (int base = t0; base < t1; base += kTile) {
    const int t = base + (int)threadIdx.x;
    const bool live = t < t1;
    TokenPicks<KM> p;
    if (pre)
      p = *pre;
    else
      load_picks<KM, MODE>(a, sm + P.er, t, live, true, p, bad);
    if (MODE == MOE_LAYOUT_PER_PICK) {
      rows_pick_tile<KM>(a, P, sm, p, t, live, over);
    } else {
      const Ballots bl = pre_bl ? *pre_bl : mask_ballots<MODE>(a, p.dmask, p.gmask, live, lane);
      rows_mask_tile<KM, MODE, SEND>(a, P, sm, p, bl, t, live, over);
    }
  }
  if (over) set_status(ctx.status, MOE_ERR_CAPACITY);
  if (SEND) {  // the block's send counts (send_counts was cleared before the barrier)
    const int *s_send = sm + P.send;
    for (int i = threadIdx.x; i < a.R * a.R; i += kTile)
      if (s_send[i]) atomicAdd(&a.L.send_counts[i], s_send[i]);
  }
}

template <int KM, int MODE>
__device__ __forceinline__ void phase2(const LayoutArgs &a, const SmemPlan &P, int *sm, int t0,
                                       int t1, DeviceCtx ctx, const TokenPicks<KM> *pre,
                                       const Ballots *pre_bl) {
  gather_counts(a, P, sm);
  segment_offsets<MODE>(a, P, sm, ctx);
  rows_loop<KM, MODE, true>(a, P, sm, t0, t1, ctx, pre, pre_bl);
}

// Phase-1 epilogue: the block's counts into its table row; block 0 clears the
// send-count matrix (every block adds into it after the barrier).
__device__ __forceinline__ void publish_counts(const LayoutArgs &a, const SmemPlan &P, int *sm) {
  __syncthreads();
  for (int b = threadIdx.x; b < a.NBp; b += kTile)
    a.agg[(size_t)blockIdx.x * a.NBp + b] = b < a.NB ? sm[P.cnt + b] : 0;
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < a.R * a.R; i += kTile) a.L.send_counts[i] = 0;
}

// Clears the block's shared counters and loads the expert -> rank map (unless
// the caller has already put it in shared memory: `load_er` false).
__device__ __forceinline__ void smem_init(const LayoutArgs &a, const SmemPlan &P, int *sm,
                                          bool load_er = true) {
  if (load_er)
    for (int i = threadIdx.x; i < a.E; i += kTile) sm[P.er + i] = __ldcg(a.expert_rank + i);
  for (int i = threadIdx.x; i < a.NBp; i += kTile) sm[P.cnt + i] = 0;
  for (int i = threadIdx.x; i < a.R * a.R; i += kTile) sm[P.send + i] = 0;
  __syncthreads();
}

// Both layout phases over the block's chunk [t0, t1), after smem_init: phase
// 1 counts the chunk's rows per bin (a one-tile chunk keeps its picks and
// ballots), the grid barrier `round` publishes the count table, phase 2
// writes the rows.  Returns false when the barrier gave up.
template <int KM, int MODE>
__device__ __forceinline__ bool layout_phases(const LayoutArgs &a, const SmemPlan &P, int *sm, int t0,
                                              int t1, DeviceCtx ctx, int *s_flag, unsigned round) {
  const int lane = threadIdx.x & 31;
  const bool one_tile = t1 - t0 <= kTile;
  bool bad = false;
  int c[4] = {0, 0, 0, 0};
  TokenPicks<KM> p;
  Ballots bl{0u, 0u, 0u, 0u};
  for (int base = t0; base < t1; base += kTile) {
    const int t = base + (int)threadIdx.x;
    load_picks<KM, MODE>(a, sm + P.er, t, t < t1, one_tile, p, bad);
    count_tile<KM, MODE>(a, p, t < t1, lane, sm + P.cnt, c, bl);
  }
  flush_counts<MODE>(a, lane, sm + P.cnt, c);
  if (bad) set_status(ctx.status, MOE_ERR_BAD_INPUT);
  publish_counts(a, P, sm);
  if (!grid_barrier(a, ctx, s_flag, round)) return false;
  phase2<KM, MODE>(a, P, sm, t0, t1, ctx, one_tile ? &p : nullptr, one_tile ? &bl : nullptr);
  return true;
}

// ------------------------------------------------------------ one pass ----
// Small token sets (mask modes) skip the count table and its grid barrier:
// every block counts every token's rows per bin itself -- the bin totals and
// the rows before its own chunk -- and block 0 also counts the whole
// send-count matrix, walking the tokens in tiles of 256 with the next tile's
// picks loaded while this one is counted.  A tile costs each block about as
// much as the barrier and the count-table pass it replaces take in all
// (clock-stamped on the decode workloads: ~2.5k cycles a tile, against ~4.7 us
// for the two-phase route at 1024 tokens), so only one or two tiles go this way.
constexpr int kOnePassTokens = 2 * kTile;

// Whether a layout of T tokens takes the one-pass route.
__host__ __device__ inline bool single_pass(int T, int mode) {
  return mode != MOE_LAYOUT_PER_PICK && T <= kOnePassTokens;
}

// The layout over the block's chunk [t0, t1) in one pass (mask modes), after
// smem_init; the expert -> rank map is in shared memory.
template <int KM, int MODE>
__device__ __forceinline__ void layout_single_pass(const LayoutArgs &a, const SmemPlan &P, int *sm,
                                                   int t0, int t1, DeviceCtx ctx) {
  static_assert(MODE != MOE_LAYOUT_PER_PICK, "mask modes only");
  const int lane = threadIdx.x & 31;
  int *s_cnt = sm + P.cnt, *s_base = sm + P.base;
  const int *s_er = sm + P.er;
  for (int b = threadIdx.x; b < a.NBp; b += kTile) s_base[b] = 0;
  __syncthreads();
  auto fetch = [&](int t, int (&e)[KM]) {
#pragma unroll
    for (int j = 0; j < KM; ++j) e[j] = (j < a.k && t < a.T) ? a.idx[(size_t)t * a.k + j] : 0;
  };
  int nxt[KM];
  fetch((int)threadIdx.x, nxt);
  bool bad = false;
  int c[4] = {0, 0, 0, 0}, cp[4] = {0, 0, 0, 0};
#pragma unroll 1
  for (int base = 0; base < a.T; base += kTile) {
    int e[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j) e[j] = nxt[j];
    fetch(base + kTile + (int)threadIdx.x, nxt);  // the next tile, in flight meanwhile
    const int t = base + (int)threadIdx.x;
    const bool live = t < a.T;
    unsigned long long dmask = 0, gmask = 0;
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      if (j < a.k && live) {
        const int ex = e[j];
        const int r = (unsigned)ex < (unsigned)a.E ? s_er[ex] : -1;
        if ((unsigned)r < (unsigned)a.R) {
          dmask |= 1ull << r;
          gmask |= 1ull << (r / a.rpg);
        } else {
          bad = true;
        }
      }
    }
    const Ballots bl = mask_ballots<MODE>(a, dmask, gmask, live, lane);
    const unsigned before = __ballot_sync(kFull, live && t < t0);
    c[0] += __popc(bl.b0);
    c[1] += __popc(bl.b1);
    c[2] += __popc(bl.g0);
    c[3] += __popc(bl.g1);
    cp[0] += __popc(bl.b0 & before);
    cp[1] += __popc(bl.b1 & before);
    cp[2] += __popc(bl.g0 & before);
    cp[3] += __popc(bl.g1 & before);
    if (blockIdx.x == 0) add_send_counts(a, P, sm, dmask, bl, t, live);
  }
  flush_counts<MODE>(a, lane, s_cnt, c);
  flush_counts<MODE>(a, lane, s_base, cp);
  if (bad) set_status(ctx.status, MOE_ERR_BAD_INPUT);
  __syncthreads();
  segment_offsets<MODE>(a, P, sm, ctx);
  rows_loop<KM, MODE, false>(a, P, sm, t0, t1, ctx, nullptr, nullptr);
  if (blockIdx.x == 0) {
    __syncthreads();
    const int *s_send = sm + P.send;
    for (int i = threadIdx.x; i < a.R * a.R; i += kTile) a.L.send_counts[i] = s_send[i];
  }
}

// ---------------------------------------------------------------- host ----
inline int num_bins(int E, int R, int rpg, int mode) {
  if (mode == MOE_LAYOUT_PER_PICK) return E;
  if (mode == MOE_LAYOUT_TWO_HOP) return R + R / rpg;
  return R;
}

// Blocks and chunk of a launch: at most `max_blocks` blocks, chunks of a
// multiple of `granule` tokens (32 for the layout kernel, a thread per token;
// 8 for the fused front ends, whose routing phase gives each warp a token).
// The workspace holds a count-table row per 8 tokens, up to kMaxBlocks.
inline void split_tokens(int T, int max_blocks, int &nblk, int &chunk, int granule = 32) {
  if (max_blocks < 1) max_blocks = 1;
  if (max_blocks > kMaxBlocks) max_blocks = kMaxBlocks;
  chunk = (int)(((long)T + max_blocks - 1) / max_blocks);
  chunk = (chunk + granule - 1) / granule * granule;
  nblk = (int)(((long)T + chunk - 1) / chunk);
}

// Arguments of one layout over the caller's buffers and workspace.
LayoutArgs make_layout_args(const int *idx, const float *w, const int *expert_rank, int T,
                            int tokens_per_rank, int k, int E, int R, int rpg, int mode,
                            const moe_layout &L, void *ws);
// Outputs of an empty token set.
cudaError_t layout_empty(const moe_layout &L, int R, int rpg, int mode, cudaStream_t s);
// Largest co-resident grid of a kernel with this much dynamic shared memory.
cudaError_t max_resident_blocks(const void *kernel, size_t smem, const DeviceCtx &ctx, int &blocks);

}  // namespace layout
}  // namespace moe
