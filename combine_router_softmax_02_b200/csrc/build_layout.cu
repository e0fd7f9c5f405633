// Stable per-destination row layout: count kernel + decoupled-lookback scan.
//
// Rows are the destination chunks of an AllToAll(-v) ("METRO AllGather vs
// AllToAll for MoE decode" (fanout.sh), sections "Work the 8-GPU payload
// example" and "Distinguish METRO from backend names"):
//   PER_PICK  one row per (token, pick), ordered (rank, expert, token);
//   DEDUP     one row per (rank, token) in the token's destination set, the
//             single-send dispatcher of the arXiv:2610.09372 summary
//             (ainewsletter), section "Two locality techniques";
//   TWO_HOP   hop-1 rows (group, token) and hop-2 rows (rank, token), the
//             two-hop dispatch of the TerraceMoE editorial, "The core problem".
//
// "Bins" are the segments of the layout: ranks (DEDUP), experts (PER_PICK) or
// ranks followed by groups (TWO_HOP).  A row's id is
//   seg_off[bin] + (rows of bin in earlier tiles) + (rows of bin in earlier
//   warps of the tile) + (rows of bin in earlier lanes of the warp).
// Kernel 1 (count) builds the per-bin totals with block histograms and global
// atomics, and publishes each tile's per-bin aggregate as a look-back flag;
// its last block turns the totals into segment offsets.  Kernel 2 (place)
// takes tiles in ticket order, looks back over its predecessors' flags for the
// exclusive prefix (16 flags per round, bounded waits), publishes its
// inclusive prefix, and writes the rows.  Within a warp a bin's ballot over the lanes gives both its
// count and each lane's position in token order (stability).  Ranks and
// groups (at most 64 each) are 64-bit masks per token: one ballot per bin
// present in the warp, then each lane walks its own bits.  Experts (PER_PICK,
// up to 1024 bins) are merged instead: each round takes the smallest key
// (rank << 10 | expert) left in the warp with redux.sync.min.
#include "layout_common.cuh"

namespace moe {
namespace layout {
namespace {


// One token's picks as seen by one thread.
template <int KM>
struct TokenPicks {
  int e[KM];
  int r[KM];
  float w[KM];
  uint32_t present;      // picks with a valid expert and rank
  unsigned long long dmask;  // ranks of the token
  unsigned long long gmask;  // groups of the token (TWO_HOP)
};

template <int KM>
__device__ __forceinline__ void load_picks(const LayoutArgs &a, const int *s_er, int t,
                                           bool want_w, TokenPicks<KM> &p, bool &bad) {
  p.present = 0;
  p.dmask = 0;
  p.gmask = 0;
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    p.e[j] = 0;
    p.r[j] = 0;
    p.w[j] = 0.0f;
    if (j < a.k && t < a.T) {
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
}

enum Pass { kPassRank = 0, kPassGroup = 1, kPassPick = 2 };

template <int KM>
__device__ __forceinline__ uint32_t pick_key(const TokenPicks<KM> &p, int j, int pass, int rpg) {
  if (pass == kPassRank) return (uint32_t)p.r[j];
  if (pass == kPassGroup) return (uint32_t)(p.r[j] / rpg);
  return ((uint32_t)p.r[j] << 10) | (uint32_t)p.e[j];
}

template <int pass>
__device__ __forceinline__ int key_bin(uint32_t key, int R) {
  if (pass == kPassRank) return (int)key;
  if (pass == kPassGroup) return R + (int)key;
  return (int)(key & 1023u);
}

// Merge the lanes' distinct keys in ascending order.  For every key present
// in the warp, f(key, has, ball, c, matched) runs on all lanes: `has` says
// whether this lane's token has the key, `ball` which lanes do, `c` how many
// distinct keys this lane had before, `matched` its picks with the key.
template <int KM, int pass, class F>
__device__ __forceinline__ void warp_merge(const TokenPicks<KM> &p, int rpg, F &&f) {
  uint32_t key[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) key[j] = pick_key(p, j, pass, rpg);
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


// ---------------------------------------------------------------- count ----
template <int KM>
__global__ void __launch_bounds__(kTile) layout_count_kernel(LayoutArgs a, DeviceCtx ctx) {
  __shared__ int s_er[kMaxE];
  __shared__ int s_cnt[kMaxBins];
  __shared__ int s_send[kSendSmem];
  __shared__ int s_last;
  const int tile = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31;
  const int t = tile * kTile + tid;
  for (int i = tid; i < a.E; i += kTile) s_er[i] = a.expert_rank[i];
  for (int i = tid; i < a.NB; i += kTile) s_cnt[i] = 0;
  // source ranks are < R, so the block's send-count matrix fits R*R <= 4096 entries
  for (int i = tid; i < a.R * a.R; i += kTile) s_send[i] = 0;
  __syncthreads();

  TokenPicks<KM> p;
  bool bad = false;
  load_picks<KM>(a, s_er, t, false, p, bad);
  if (a.mode == MOE_LAYOUT_PER_PICK) {  // the row order needs distinct experts per token
#pragma unroll
    for (int i = 0; i < KM; ++i)
#pragma unroll
      for (int j = i + 1; j < KM; ++j)
        if ((p.present >> i & 1u) && (p.present >> j & 1u) && p.e[i] == p.e[j]) {
          bad = true;
          p.present &= ~(1u << j);
        }
  }
  const int src0 = __shfl_sync(kFull, (t < a.T) ? t / a.tpr : 0, 0);
  const int src = (t < a.T) ? t / a.tpr : src0;
  const bool src_uniform = __all_sync(kFull, src == src0);  // one source rank in the warp

  auto count_send = [&](int dst, bool has, unsigned ball) {
    if (!has) return;
    const unsigned peers = src_uniform ? ball : __match_any_sync(ball, src);
    if (lane == __ffs(peers) - 1) atomicAdd(&s_send[src * a.R + dst], __popc(peers));
  };
  if (a.mode == MOE_LAYOUT_PER_PICK) {
    warp_merge<KM, kPassPick>(p, a.rpg, [&](uint32_t b, bool has, unsigned ball, int, uint32_t) {
      if (lane == 0) atomicAdd(&s_cnt[key_bin<kPassPick>(b, a.R)], __popc(ball));
      count_send((int)(b >> 10), has, ball);
    });
  } else {
    warp_mask_bins(p.dmask, [&](int r, bool has, unsigned ball) {
      if (lane == 0) atomicAdd(&s_cnt[r], __popc(ball));
      count_send(r, has, ball);
    });
    if (a.mode == MOE_LAYOUT_TWO_HOP)
      warp_mask_bins(p.gmask, [&](int g, bool, unsigned ball) {
        if (lane == 0) atomicAdd(&s_cnt[a.R + g], __popc(ball));
      });
  }
  if (bad) set_status(ctx.status, MOE_ERR_BAD_INPUT);
  __syncthreads();
  // publish this tile's aggregates for the place kernel's look-back (the
  // first tile's is its inclusive prefix); a silent tile leaves its flags clear
  const bool silent = (tile == ctx.silent_tile);
  for (int i = tid; i < a.NB; i += kTile)
    a.state[(size_t)tile * a.NB + i] =
        silent ? 0ull : ((tile == 0 ? kFlagInc : kFlagAgg) | (unsigned)s_cnt[i]);
  for (int i = tid; i < a.NB; i += kTile)
    if (s_cnt[i]) atomicAdd(&a.totals[i], s_cnt[i]);
  for (int i = tid; i < a.R * a.R; i += kTile)
    if (s_send[i]) atomicAdd(&a.L.send_counts[i], s_send[i]);
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&a.counters[1], 1) == a.num_tiles - 1);
  __syncthreads();
  if (s_last) {
    __threadfence();
    finalize(a, s_er, s_cnt, ctx);  // s_cnt is free again after the flush
  }
}

// ---------------------------------------------------------------- place ----
__device__ __forceinline__ unsigned long long wait_published(const unsigned long long *word,
                                                             const DeviceCtx &ctx, bool &timed_out) {
  unsigned long long v = ld_acquire_u64(word);
  if (v >> 32) return v;
  const uint64_t t0 = global_ns();
  while (true) {
    __nanosleep(64);
    v = ld_acquire_u64(word);
    if (v >> 32) return v;
    if (global_ns() - t0 > ctx.wait_limit_ns || ld_volatile_i32(ctx.status) == MOE_ERR_TIMEOUT) {
      timed_out = true;
      return kFlagInc;  // treat as an inclusive zero so the chain ends
    }
  }
}

constexpr int kWindow = 16;

// Exclusive prefix of one bin before `tile`: the bin's flags of the earlier
// tiles are summed from tile - 1 backwards until an inclusive prefix is met,
// kWindow predecessors per round with all of their loads in flight.
__device__ __forceinline__ int look_back(const unsigned long long *col, int NB, int tile,
                                         const DeviceCtx &ctx, bool &timed_out) {
  int excl = 0;
  for (int q = tile - 1; q >= 0; q -= kWindow) {
    unsigned long long v[kWindow];
#pragma unroll
    for (int i = 0; i < kWindow; ++i)
      v[i] = (q - i >= 0) ? ld_acquire_u64(col + (size_t)(q - i) * NB) : 0ull;
#pragma unroll
    for (int i = 0; i < kWindow; ++i) {
      if (q - i < 0) return excl;
      unsigned long long w = v[i];
      if ((w >> 32) == 0ull) w = wait_published(col + (size_t)(q - i) * NB, ctx, timed_out);
      excl += (int)(unsigned)(w & 0xffffffffull);
      if ((w >> 32) == 2ull) return excl;
    }
  }
  return excl;
}

template <int KM>
__global__ void __launch_bounds__(kTile) layout_place_kernel(LayoutArgs a, DeviceCtx ctx) {
  __shared__ int s_er[kMaxE];
  __shared__ int s_wcnt[kWarps][kMaxBins];
  __shared__ int s_base[kMaxBins];
  __shared__ unsigned s_wball[kWarps][2 * kMaxR];  // mask bins: each warp's ballot per bin
  __shared__ int s_tile;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_tile = atomicAdd(&a.counters[0], 1);
  for (int i = tid; i < a.E; i += kTile) s_er[i] = a.expert_rank[i];
  for (int i = tid; i < a.NB; i += kTile)
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s_wcnt[w][i] = 0;
  __syncthreads();
  const int tile = s_tile;
  const int t = tile * kTile + tid;
  const moe_layout &L = a.L;

  TokenPicks<KM> p;
  bool bad = false;  // reported by the count kernel already
  load_picks<KM>(a, s_er, t, true, p, bad);
  if (a.mode == MOE_LAYOUT_PER_PICK) {
#pragma unroll
    for (int i = 0; i < KM; ++i)
#pragma unroll
      for (int j = i + 1; j < KM; ++j)
        if ((p.present >> i & 1u) && (p.present >> j & 1u) && p.e[i] == p.e[j]) p.present &= ~(1u << j);
  }

  // 1. per-warp counts of every bin
  auto note = [&](int bin, unsigned ball) {
    if (lane == 0) s_wcnt[warp][bin] = __popc(ball);
  };
  if (a.mode == MOE_LAYOUT_PER_PICK) {
    warp_merge<KM, kPassPick>(p, a.rpg, [&](uint32_t b, bool, unsigned ball, int, uint32_t) {
      note(key_bin<kPassPick>(b, a.R), ball);
    });
  } else {
    warp_mask_bins(p.dmask, [&](int r, bool, unsigned ball) {
      note(r, ball);
      if (lane == 0) s_wball[warp][r] = ball;
    });
    if (a.mode == MOE_LAYOUT_TWO_HOP)
      warp_mask_bins(p.gmask, [&](int g, bool, unsigned ball) {
        note(a.R + g, ball);
        if (lane == 0) s_wball[warp][a.R + g] = ball;
      });
  }
  __syncthreads();

  // 2. tile aggregate, publish, look back, publish the inclusive prefix
  bool timed_out = false;
  const bool silent = (tile == ctx.silent_tile);
  for (int b = tid; b < a.NB; b += kTile) {
    int agg = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int c = s_wcnt[w][b];
      s_wcnt[w][b] = agg;
      agg += c;
    }
    unsigned long long *mine = a.state + (size_t)tile * a.NB + b;
    int excl = 0;
    if (tile == 0) {
      if (!silent) st_release_u64(mine, kFlagInc | (unsigned)agg);
    } else {
      if (!silent) st_release_u64(mine, kFlagAgg | (unsigned)agg);
      excl = look_back(a.state + b, a.NB, tile, ctx, timed_out);
      if (!silent) st_release_u64(mine, kFlagInc | (unsigned)(excl + agg));
    }
    s_base[b] = __ldcg(a.seg_off + b) + excl;
  }
  if (timed_out) set_status(ctx.status, MOE_ERR_TIMEOUT);
  __syncthreads();

  // 3. rows (every lane takes part in the merges; lanes past T have no picks)
  bool over = false;
  const bool live = t < a.T;
  const unsigned lt = lanemask_lt();
  const size_t tk = (size_t)t * a.k;
  if (a.mode != MOE_LAYOUT_PER_PICK) {
    // mask bins: each lane walks its own ranks (and groups) in ascending order;
    // its position in a bin is the count of earlier lanes in the bin's ballot
    auto row_of = [&](int bin) {
      return s_base[bin] + s_wcnt[warp][bin] + __popc(s_wball[warp][bin] & lt);
    };
    if (a.mode == MOE_LAYOUT_TWO_HOP) {
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
      if (a.mode == MOE_LAYOUT_TWO_HOP) {
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
  } else if (a.mode == MOE_LAYOUT_PER_PICK) {
    int cnt = 0;
    auto write_row = [&](int bin, bool has, unsigned ball, int c, uint32_t matched) {
      if (!has) return;
      const int row = s_base[bin] + s_wcnt[warp][bin] + __popc(ball & lt);
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
    };
    warp_merge<KM, kPassPick>(p, a.rpg, [&](uint32_t b, bool has, unsigned ball, int c, uint32_t m) {
      write_row(key_bin<kPassPick>(b, a.R), has, ball, c, m);
    });
    if (live)
      for (int c = cnt; c < a.k; ++c) L.token_rows[tk + c] = -1;
  }
  if (over) set_status(ctx.status, MOE_ERR_CAPACITY);
}

template <int KM>
cudaError_t launch_count_place(const LayoutArgs &a, const DeviceCtx &ctx, cudaStream_t s) {
  layout_count_kernel<KM><<<a.num_tiles, kTile, 0, s>>>(a, ctx);
  cudaError_t err = count_launch(cudaGetLastError());
  if (err != cudaSuccess) return err;
  layout_place_kernel<KM><<<a.num_tiles, kTile, 0, s>>>(a, ctx);
  return count_launch(cudaGetLastError());
}

template <int KM>
cudaError_t launch_place(const LayoutArgs &a, const DeviceCtx &ctx, cudaStream_t s) {
  layout_place_kernel<KM><<<a.num_tiles, kTile, 0, s>>>(a, ctx);
  return count_launch(cudaGetLastError());
}

}  // namespace

LayoutArgs make_layout_args(const int *idx, const float *w, const int *expert_rank, int T,
                            int tokens_per_rank, int k, int E, int R, int rpg, int mode,
                            const moe_layout &L, void *ws) {
  LayoutArgs a;
  a.idx = idx;
  a.w = w;
  a.expert_rank = expert_rank;
  a.T = T;
  a.tpr = tokens_per_rank;
  a.k = k;
  a.E = E;
  a.R = R;
  a.rpg = (mode == MOE_LAYOUT_TWO_HOP) ? rpg : 1;
  a.G = (mode == MOE_LAYOUT_TWO_HOP) ? R / rpg : 0;
  a.mode = mode;
  a.NB = num_bins(E, R, a.rpg, mode);
  a.num_tiles = (T + kTile - 1) / kTile;
  char *base = static_cast<char *>(ws);
  a.counters = reinterpret_cast<int *>(base);
  a.totals = a.counters + 2;
  a.seg_off = a.totals + a.NB;
  a.state = reinterpret_cast<unsigned long long *>(base + align16(sizeof(int) * (2 + 2 * (size_t)a.NB)));
  a.L = L;
  return a;
}

cudaError_t layout_clear(const LayoutArgs &a, cudaStream_t s) {
  cudaError_t err = cudaMemsetAsync(a.counters, 0, sizeof(int) * (2 + (size_t)a.NB), s);
  if (err != cudaSuccess) return err;
  return cudaMemsetAsync(a.L.send_counts, 0, sizeof(int) * (size_t)a.R * a.R, s);
}

cudaError_t layout_empty(const moe_layout &L, int R, int rpg, int mode, cudaStream_t s) {
  cudaError_t err;
  if ((err = cudaMemsetAsync(L.rank_offsets, 0, sizeof(int) * (R + 1), s)) != cudaSuccess) return err;
  if ((err = cudaMemsetAsync(L.num_rows, 0, sizeof(int), s)) != cudaSuccess) return err;
  if ((err = cudaMemsetAsync(L.send_counts, 0, sizeof(int) * R * R, s)) != cudaSuccess) return err;
  if (mode == MOE_LAYOUT_TWO_HOP) {
    if ((err = cudaMemsetAsync(L.group_offsets, 0, sizeof(int) * (R / rpg + 1), s)) != cudaSuccess)
      return err;
    if ((err = cudaMemsetAsync(L.num_rows_hop1, 0, sizeof(int), s)) != cudaSuccess) return err;
  }
  return cudaSuccess;
}

cudaError_t launch_layout_place(const LayoutArgs &a, const DeviceCtx &ctx, cudaStream_t s) {
  if (a.k <= 2) return launch_place<2>(a, ctx, s);
  if (a.k <= 4) return launch_place<4>(a, ctx, s);
  if (a.k <= 8) return launch_place<8>(a, ctx, s);
  return launch_place<16>(a, ctx, s);
}

}  // namespace layout

size_t layout_workspace_bytes(int T, int k, int E, int R, int rpg, int mode) {
  (void)k;
  const int NB = layout::num_bins(E, R, rpg, mode);
  const size_t tiles = (size_t)((T + layout::kTile - 1) / layout::kTile);
  return layout::align16(sizeof(int) * (2 + 2 * (size_t)NB)) + tiles * NB * sizeof(unsigned long long);
}

cudaError_t launch_build_layout(const int *idx, const float *w, const int *expert_rank, int T,
                                int tokens_per_rank, int k, int E, int R, int rpg, int mode,
                                const moe_layout &L, void *ws, const DeviceCtx &ctx,
                                cudaStream_t s) {
  if (T == 0) return layout::layout_empty(L, R, rpg, mode, s);
  const layout::LayoutArgs a =
      layout::make_layout_args(idx, w, expert_rank, T, tokens_per_rank, k, E, R, rpg, mode, L, ws);
  cudaError_t err = layout::layout_clear(a, s);
  if (err != cudaSuccess) return err;
  if (k <= 2) return layout::launch_count_place<2>(a, ctx, s);
  if (k <= 4) return layout::launch_count_place<4>(a, ctx, s);
  if (k <= 8) return layout::launch_count_place<8>(a, ctx, s);
  return layout::launch_count_place<16>(a, ctx, s);
}

}  // namespace moe
