// Routing, demand histogram, METRO assignment and layout in one launch.
//
// "METRO AllGather vs AllToAll for MoE decode" (fanout.sh): at decode sizes the
// per-kernel launch cost is the price of the global routing information
// (section "changes the routing information"), so the whole front end runs
// as one cooperative kernel in three phases separated by grid barriers:
//   A. every block routes the tokens of its chunk (route_common.cuh), adds its
//      demand histogram into the workspace's demand scratch, and stages the
//      replica map in shared memory (assign_common.cuh; a small map's loads
//      are issued before the routing, so they complete behind it);
//   B. every block runs the METRO greedy over the complete demand vector into
//      its own shared memory (the greedy is deterministic, so every block gets
//      the same expert -> rank map and no block waits for another); block 0
//      writes expert_slot, expert_rank, rank_active and counts; then every
//      block counts its chunk's layout bins with that map;
//   C. after the layout's barrier every block writes its rows (layout_common.cuh);
//      small token sets (mask modes) skip that barrier: every block counts every
//      token's rows itself and writes its own.
// Every output equals that of moe_route_topk, moe_demand_hist,
// moe_replica_assign and moe_build_layout called one after the other.
#include "assign_common.cuh"
#include "layout_common.cuh"
#include "route_common.cuh"

namespace moe {
namespace {

using layout::LayoutArgs;
using layout::SmemPlan;
using layout::kTile;
using layout::kWarps;

struct FrontArgs {
  const float *logits;
  int n_groups, gpt, renorm;
  int *idx_out;      // [T][k] picks (phases C and D read them back)
  float *w_out;      // [T][k] gate weights
  int *counts;       // [E] demand vector
  const int *off, *slots, *slot_rank;  // replica map (CSR)
  int n_entries, S;
  int *expert_slot;  // [E]
  int *expert_rank;  // [E] (the layout phases read it back)
  int *rank_active;  // [R]
};

// METRO's shared memory starts after the expert -> rank map (the layout
// plan's first region), which the greedy fills and the layout phases read.
__host__ __device__ inline int front_smem_ints(int E, int NBp, int R, int n_entries) {
  const int E4 = (E + 3) & ~3;
  const int lay = layout::smem_plan(E, NBp, R, true).total, metro = E4 + metro_plan(E, n_entries, R).total;
  return lay > metro ? lay : metro;
}

template <int EPL, bool FULL, int KM>
__global__ void __launch_bounds__(kTile) route_assign_layout_kernel(FrontArgs f, LayoutArgs a, DeviceCtx ctx) {
  extern __shared__ int4 smem_raw[];
  int *sm = reinterpret_cast<int *>(smem_raw);
  __shared__ __align__(16) float s_cv[kWarps][32];
  __shared__ int s_ce[kWarps][32];
  __shared__ int s_flag;
  const SmemPlan P = layout::smem_plan(a.E, a.NBp, a.R, true);
  const MetroPlan M = metro_plan(a.E, f.n_entries, a.R);
  int *smm = sm + ((a.E + 3) & ~3);  // METRO's scratch (P.er is the first region)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  MetroPrefetch pf;  // the replica map's loads, in flight while the block routes
  pf.load(a.E, f.off, f.slots, f.n_entries, f.slot_rank, f.S);
  int *s_hist = sm + P.hist;
  for (int i = tid; i < a.E; i += kTile) s_hist[i] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * a.chunk, t1 = min(a.T, t0 + a.chunk);

  // A: route the chunk, one warp per token; demand histogram of every pick
  route::Lanes<EPL, FULL> L;
  L.init(lane, a.E, f.n_groups, f.gpt);
  bool bad = false;
  for (int t = t0 + warp; t < t1; t += kWarps) {
    int e;
    float w;
    route::route_token<EPL, FULL>(f.logits + (size_t)t * a.E, a.E, a.k, f.n_groups, f.gpt, f.renorm, L,
                                  s_cv[warp], s_ce[warp], lane, e, w, bad);
    if (lane < a.k) {
      f.idx_out[(size_t)t * a.k + lane] = e;
      f.w_out[(size_t)t * a.k + lane] = w;
      atomicAdd(&s_hist[e], 1);
    }
  }
  if (__any_sync(route::kFull, bad) && lane == 0) set_status(ctx.status, MOE_ERR_BAD_INPUT);
  __syncthreads();
  for (int i = tid; i < a.E; i += kTile)
    if (s_hist[i]) atomicAdd(&a.cnt[i], s_hist[i]);
  __syncthreads();  // s_hist is read out before the replica map reuses its memory
  if (pf.ok)
    metro_stage_prefetched(a.E, f.n_entries, f.S, a.R, pf, smm, M);
  else
    metro_stage(a.E, f.off, f.slots, f.n_entries, f.slot_rank, f.S, a.R, nullptr, smm, M);
  if (!layout::grid_barrier(a, ctx, &s_flag, 1)) return;

  // B: the greedy in every block, straight into the layout's expert -> rank map
  metro_solve(a.cnt, a.E, a.R, smm, M, sm + P.er, blockIdx.x == 0, f.expert_slot, f.expert_rank,
              f.rank_active, ctx);
  if (blockIdx.x == 0)
    for (int i = tid; i < a.E; i += kTile) f.counts[i] = __ldcg(a.cnt + i);

  // B + C: the layout with the assigned ranks
  layout::smem_init(a, P, sm, false);
  const bool one = layout::single_pass(a.T, a.mode);
  if (a.mode == MOE_LAYOUT_DEDUP) {
    if (one)
      layout::layout_single_pass<KM, MOE_LAYOUT_DEDUP>(a, P, sm, t0, t1, ctx);
    else
      layout::layout_phases<KM, MOE_LAYOUT_DEDUP>(a, P, sm, t0, t1, ctx, &s_flag, 2);
  } else if (a.mode == MOE_LAYOUT_TWO_HOP) {
    if (one)
      layout::layout_single_pass<KM, MOE_LAYOUT_TWO_HOP>(a, P, sm, t0, t1, ctx);
    else
      layout::layout_phases<KM, MOE_LAYOUT_TWO_HOP>(a, P, sm, t0, t1, ctx, &s_flag, 2);
  } else {
    layout::layout_phases<KM, MOE_LAYOUT_PER_PICK>(a, P, sm, t0, t1, ctx, &s_flag, 2);
  }
}

std::atomic<unsigned long long> g_smem_set[6][2][2];

template <int EPL, bool FULL, int KM>
cudaError_t launch_front(const FrontArgs &f0, const LayoutArgs &a0, int slot, const DeviceCtx &ctx,
                         cudaStream_t s) {
  FrontArgs f = f0;
  LayoutArgs a = a0;
  const size_t smem = sizeof(int) * (size_t)front_smem_ints(a.E, a.NBp, a.R, f.n_entries);
  auto kern = route_assign_layout_kernel<EPL, FULL, KM>;
  cudaError_t err = set_smem_limit_once(kern, kFrontSmemMax, g_smem_set[slot][FULL][KM > 8]);
  if (err != cudaSuccess) return err;
  int resident = 0;
  if ((err = layout::max_resident_blocks((const void *)kern, smem, ctx, resident)) != cudaSuccess) return err;
  layout::split_tokens(a.T, resident, a.nblk, a.chunk, 8);
  // barrier words and the demand scratch start at zero
  if ((err = cudaMemsetAsync(a.bar, 0, sizeof(int) * (16 + (size_t)a.E), s)) != cudaSuccess) return err;
  void *args[] = {&f, &a, const_cast<DeviceCtx *>(&ctx)};
  err = cudaLaunchCooperativeKernel((const void *)kern, dim3(a.nblk), dim3(kTile), args, smem, s);
  if (err != cudaSuccess) return err;
  return count_launch(cudaGetLastError());
}

template <int EPL>
cudaError_t launch_epl(const FrontArgs &f, const LayoutArgs &a, int slot, const DeviceCtx &ctx,
                       cudaStream_t s) {
  const bool full = a.E == 32 * EPL;
  if (a.k <= 8)
    return full ? launch_front<EPL, true, 8>(f, a, slot, ctx, s) : launch_front<EPL, false, 8>(f, a, slot, ctx, s);
  return full ? launch_front<EPL, true, 16>(f, a, slot, ctx, s) : launch_front<EPL, false, 16>(f, a, slot, ctx, s);
}

}  // namespace

size_t front_smem_bytes(int E, int k, int R, int rpg, int mode, int n_entries) {
  (void)k;
  const int NBp = (layout::num_bins(E, R, mode == MOE_LAYOUT_TWO_HOP ? rpg : 1, mode) + 3) & ~3;
  return sizeof(int) * (size_t)front_smem_ints(E, NBp, R, n_entries);
}

cudaError_t launch_route_assign_layout(const float *logits, int T, int E, int k, int n_groups, int gpt,
                                       int renorm, const int *off, const int *slots, int n_entries,
                                       const int *slot_rank, int S, int tokens_per_rank, int R,
                                       int rpg, int mode, int *idx, float *w, int *counts,
                                       int *expert_slot, int *expert_rank, int *rank_active,
                                       const moe_layout &L, void *ws, const DeviceCtx &ctx,
                                       cudaStream_t s) {
  cudaError_t err;
  if (T == 0) {  // no picks: every expert inactive
    if ((err = cudaMemsetAsync(counts, 0, sizeof(int) * (size_t)E, s)) != cudaSuccess) return err;
    if ((err = cudaMemsetAsync(expert_slot, 0xff, sizeof(int) * (size_t)E, s)) != cudaSuccess) return err;
    if ((err = cudaMemsetAsync(expert_rank, 0xff, sizeof(int) * (size_t)E, s)) != cudaSuccess) return err;
    if ((err = cudaMemsetAsync(rank_active, 0, sizeof(int) * (size_t)R, s)) != cudaSuccess) return err;
    return layout::layout_empty(L, R, rpg, mode, s);
  }
  const LayoutArgs a = layout::make_layout_args(idx, w, expert_rank, T, tokens_per_rank, k, E, R,
                                                rpg, mode, L, ws);
  FrontArgs f{logits, n_groups, gpt, renorm, idx, w, counts, off, slots, slot_rank, n_entries, S,
              expert_slot, expert_rank, rank_active};
  const int epl = (E + 31) / 32;
  if (epl <= 1) return launch_epl<1>(f, a, 0, ctx, s);
  if (epl <= 2) return launch_epl<2>(f, a, 1, ctx, s);
  if (epl <= 4) return launch_epl<4>(f, a, 2, ctx, s);
  if (epl <= 8) return launch_epl<8>(f, a, 3, ctx, s);
  if (epl <= 16) return launch_epl<16>(f, a, 4, ctx, s);
  return launch_epl<32>(f, a, 5, ctx, s);
}

}  // namespace moe
