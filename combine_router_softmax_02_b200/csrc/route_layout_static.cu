// Fused routing and layout for placements with one replica per expert.
//
// With a single replica per expert, METRO's assignment ("METRO AllGather vs
// AllToAll for MoE decode" (fanout.sh), sections "changes the routing
// information" and "Add the expert-weight traffic term") has no choice to
// make: each active expert goes to its only replica.  The destination rank of
// every pick is then known as soon as the pick is, so one cooperative kernel
// routes each token of its chunk (route_common.cuh), counts the demand vector
// and the layout's bins while it does, and after the grid barrier runs the
// layout's second phase (layout_common.cuh) -- the work of route_topk,
// demand_hist, replica_assign and build_layout in one launch.  Every output
// equals that of the separate calls.
#include "layout_common.cuh"
#include "route_common.cuh"

namespace moe {
namespace {

using layout::LayoutArgs;
using layout::SmemPlan;
using layout::kTile;
using layout::kWarps;

struct RouteArgs {
  const float *logits;
  int n_groups, gpt, renorm;
  int *idx_out;      // [T][k] picks (phase 2 reads them back)
  float *w_out;      // [T][k] gate weights
  int *counts;       // [E] demand vector
  int *rank_active;  // [R] activated experts per rank, or null
};

template <int EPL, bool FULL, int KM>
__global__ void __launch_bounds__(kTile) route_layout_kernel(RouteArgs ra, LayoutArgs a, DeviceCtx ctx) {
  extern __shared__ int4 smem_raw[];
  int *sm = reinterpret_cast<int *>(smem_raw);
  __shared__ __align__(16) float s_cv[kWarps][32];
  __shared__ int s_ce[kWarps][32];
  __shared__ int s_flag;
  const SmemPlan P = layout::smem_plan(a.E, a.NBp, a.R, true);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int *s_er = sm + P.er, *s_cnt = sm + P.cnt, *s_hist = sm + P.hist;
  for (int i = tid; i < a.E; i += kTile) s_hist[i] = 0;
  layout::smem_init(a, P, sm);
  const int t0 = blockIdx.x * a.chunk, t1 = min(a.T, t0 + a.chunk);

  // phase 1: route the chunk, one warp per token, counting as it goes
  route::Lanes<EPL, FULL> L;
  L.init(lane, a.E, ra.n_groups, ra.gpt);
  bool bad = false;
  for (int t = t0 + warp; t < t1; t += kWarps) {
    int e;
    float w;
    route::route_token<EPL, FULL>(ra.logits + (size_t)t * a.E, a.E, a.k, ra.n_groups, ra.gpt,
                                  ra.renorm, L, s_cv[warp], s_ce[warp], lane, e, w, bad);
    int r = -1;
    if (lane < a.k) {
      ra.idx_out[(size_t)t * a.k + lane] = e;
      ra.w_out[(size_t)t * a.k + lane] = w;
      r = s_er[e];
      if ((unsigned)r >= (unsigned)a.R) {
        bad = true;
        r = -1;
      }
      if (r >= 0) atomicAdd(&s_hist[e], 1);
    }
    if (a.mode == MOE_LAYOUT_PER_PICK) {
      if (r >= 0) atomicAdd(&s_cnt[e], 1);  // top-k experts of a token are distinct
    } else {
      const unsigned long long dmask = layout::warp_or64(r >= 0 ? 1ull << r : 0ull);
      if (dmask >> lane & 1ull) atomicAdd(&s_cnt[lane], 1);
      if (dmask >> (lane + 32) & 1ull) atomicAdd(&s_cnt[lane + 32], 1);
      if (a.mode == MOE_LAYOUT_TWO_HOP) {
        const unsigned long long gmask = layout::warp_or64(r >= 0 ? 1ull << (r / a.rpg) : 0ull);
        if (gmask >> lane & 1ull) atomicAdd(&s_cnt[a.R + lane], 1);
        if (gmask >> (lane + 32) & 1ull) atomicAdd(&s_cnt[a.R + lane + 32], 1);
      }
    }
  }
  if (__any_sync(route::kFull, bad) && lane == 0) set_status(ctx.status, MOE_ERR_BAD_INPUT);
  layout::publish_counts(a, P, sm);
  if (blockIdx.x == 0)
    for (int i = tid; i < a.E; i += kTile) ra.counts[i] = 0;
  if (!layout::grid_barrier(a, ctx, &s_flag)) return;

  // phase 2: the layout's offsets and rows, then the demand vector
  using Picks = layout::TokenPicks<KM>;
  if (a.mode == MOE_LAYOUT_DEDUP)
    layout::phase2<KM, MOE_LAYOUT_DEDUP>(a, P, sm, t0, t1, ctx, (const Picks *)nullptr, nullptr);
  else if (a.mode == MOE_LAYOUT_TWO_HOP)
    layout::phase2<KM, MOE_LAYOUT_TWO_HOP>(a, P, sm, t0, t1, ctx, (const Picks *)nullptr, nullptr);
  else
    layout::phase2<KM, MOE_LAYOUT_PER_PICK>(a, P, sm, t0, t1, ctx, (const Picks *)nullptr, nullptr);
  for (int i = tid; i < a.E; i += kTile)
    if (s_hist[i]) atomicAdd(&ra.counts[i], s_hist[i]);
  if (!ra.rank_active) return;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_flag = (atomicAdd(&a.bar[1], 1u) == (unsigned)a.nblk - 1);
  __syncthreads();
  if (!s_flag) return;
  __threadfence();  // the last block: every count is in
  int *s_act = sm + P.send;
  for (int i = tid; i < a.R; i += kTile) s_act[i] = 0;
  __syncthreads();
  for (int i = tid; i < a.E; i += kTile) {
    const int r = s_er[i];
    if ((unsigned)r < (unsigned)a.R && __ldcg(ra.counts + i) > 0) atomicAdd(&s_act[r], 1);
  }
  __syncthreads();
  for (int i = tid; i < a.R; i += kTile) ra.rank_active[i] = s_act[i];
}

std::atomic<unsigned long long> g_smem_set[6][2][2];

template <int EPL, bool FULL, int KM>
cudaError_t launch_fused(const RouteArgs &ra0, const LayoutArgs &a0, int slot, const DeviceCtx &ctx,
                         cudaStream_t s) {
  RouteArgs ra = ra0;
  LayoutArgs a = a0;
  const size_t smem = sizeof(int) * (size_t)layout::smem_plan(a.E, a.NBp, a.R, true).total;
  auto kern = route_layout_kernel<EPL, FULL, KM>;
  cudaError_t err = set_smem_limit_once(kern, 200 * 1024, g_smem_set[slot][FULL][KM > 8]);
  if (err != cudaSuccess) return err;
  int resident = 0;
  if ((err = layout::max_resident_blocks((const void *)kern, smem, ctx, resident)) != cudaSuccess)
    return err;
  layout::split_tokens(a.T, resident, a.nblk, a.chunk, 8);
  if ((err = cudaMemsetAsync(a.bar, 0, sizeof(int) * 16, s)) != cudaSuccess) return err;
  void *args[] = {&ra, &a, const_cast<DeviceCtx *>(&ctx)};
  err = cudaLaunchCooperativeKernel((const void *)kern, dim3(a.nblk), dim3(kTile), args, smem, s);
  if (err != cudaSuccess) return err;
  return count_launch(cudaGetLastError());
}

template <int EPL>
cudaError_t launch_epl(const RouteArgs &ra, const LayoutArgs &a, int slot, const DeviceCtx &ctx,
                       cudaStream_t s) {
  const bool full = a.E == 32 * EPL;
  if (a.k <= 8)
    return full ? launch_fused<EPL, true, 8>(ra, a, slot, ctx, s)
                : launch_fused<EPL, false, 8>(ra, a, slot, ctx, s);
  return full ? launch_fused<EPL, true, 16>(ra, a, slot, ctx, s)
              : launch_fused<EPL, false, 16>(ra, a, slot, ctx, s);
}

}  // namespace

cudaError_t launch_route_layout_static(const float *logits, int T, int E, int k, int n_groups,
                                       int gpt, int renorm, const int *expert_rank,
                                       int tokens_per_rank, int R, int rpg, int mode, int *idx,
                                       float *w, int *counts, int *rank_active,
                                       const moe_layout &L, void *ws, const DeviceCtx &ctx,
                                       cudaStream_t s) {
  cudaError_t err;
  if (T == 0) {
    if ((err = cudaMemsetAsync(counts, 0, sizeof(int) * (size_t)E, s)) != cudaSuccess) return err;
    if (rank_active && (err = cudaMemsetAsync(rank_active, 0, sizeof(int) * (size_t)R, s)) != cudaSuccess)
      return err;
    return layout::layout_empty(L, R, rpg, mode, s);
  }
  const LayoutArgs a = layout::make_layout_args(idx, w, expert_rank, T, tokens_per_rank, k, E, R,
                                                rpg, mode, L, ws);
  RouteArgs ra{logits, n_groups, gpt, renorm, idx, w, counts, rank_active};
  const int epl = (E + 31) / 32;
  if (epl <= 1) return launch_epl<1>(ra, a, 0, ctx, s);
  if (epl <= 2) return launch_epl<2>(ra, a, 1, ctx, s);
  if (epl <= 4) return launch_epl<4>(ra, a, 2, ctx, s);
  if (epl <= 8) return launch_epl<8>(ra, a, 3, ctx, s);
  if (epl <= 16) return launch_epl<16>(ra, a, 4, ctx, s);
  return launch_epl<32>(ra, a, 5, ctx, s);
}

}  // namespace moe
