// Fused routing and layout counting for placements with one replica per expert.
//
// With a single replica per expert, METRO's assignment ("METRO AllGather vs
// AllToAll for MoE decode" (fanout.sh), sections "changes the routing
// information" and "Add the expert-weight traffic term") has no choice to
// make: each active expert goes to its only replica.  The destination rank of
// every pick is then known as soon as the pick is, so one kernel routes each
// token (route_common.cuh), counts the demand vector, and counts the layout's
// bins and send matrix in the same pass -- the work of route_topk,
// demand_hist, replica_assign and the layout's count kernel.  Its last block
// scans the totals into segment offsets; the layout's place kernel then runs
// unchanged.  Every output equals that of the separate calls.
#include "layout_common.cuh"
#include "route_common.cuh"

namespace moe {
namespace {

using layout::LayoutArgs;

struct RouteArgs {
  const float *logits;
  int n_groups, gpt, renorm;
  int *idx_out;      // [T][k] picks (the layout reads them back in its place kernel)
  float *w_out;      // [T][k] gate weights
  int *counts;       // [E] demand vector (zeroed before the launch)
  int *rank_active;  // [R] activated experts per rank, or null
};

template <int EPL, bool FULL>
__global__ void __launch_bounds__(256) route_count_kernel(RouteArgs ra, LayoutArgs a, DeviceCtx ctx) {
  __shared__ uint32_t s_ck[8][32];
  __shared__ int s_ce[8][32];
  __shared__ int s_er[kMaxE];
  __shared__ int s_hist[kMaxE];
  __shared__ int s_cnt[layout::kMaxBins];
  __shared__ int s_send[layout::kSendSmem];
  __shared__ int s_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < a.E; i += blockDim.x) {
    s_er[i] = a.expert_rank[i];
    s_hist[i] = 0;
  }
  for (int i = tid; i < a.NB; i += blockDim.x) s_cnt[i] = 0;
  for (int i = tid; i < a.R * a.R; i += blockDim.x) s_send[i] = 0;
  // the place kernel's scan flags start clear
  const size_t nstate = (size_t)a.num_tiles * a.NB;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + tid; i < nstate; i += (size_t)gridDim.x * blockDim.x)
    a.state[i] = 0ull;
  __syncthreads();

  route::Lanes<EPL, FULL> L;
  L.init(lane, a.E, ra.n_groups, ra.gpt);
  // contiguous tokens per block, so each block touches few source ranks
  const int per = ((a.T + gridDim.x - 1) / gridDim.x + 7) & ~7;
  const int t0 = blockIdx.x * per, t1 = min(a.T, t0 + per);
  bool bad = false;
  for (int t = t0 + warp; t < t1; t += 8) {
    int e;
    float w;
    route::route_token<EPL, FULL>(ra.logits + (size_t)t * a.E, a.E, a.k, ra.n_groups, ra.gpt, ra.renorm, L,
                            s_ck[warp], s_ce[warp], lane, e, w, bad);
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
    const int src = t / a.tpr;
    if (a.mode == MOE_LAYOUT_PER_PICK) {
      if (r >= 0) {
        atomicAdd(&s_cnt[e], 1);
        atomicAdd(&s_send[src * a.R + r], 1);
      }
    } else {
      const unsigned long long dmask = layout::warp_or64(r >= 0 ? 1ull << r : 0ull);
      const unsigned long long gmask = layout::warp_or64(r >= 0 ? 1ull << (r / a.rpg) : 0ull);
      if (lane == 0) {
        for (unsigned long long m = dmask; m; m &= m - 1) {
          const int rr = __ffsll((long long)m) - 1;
          atomicAdd(&s_cnt[rr], 1);
          atomicAdd(&s_send[src * a.R + rr], 1);
        }
        if (a.mode == MOE_LAYOUT_TWO_HOP)
          for (unsigned long long m = gmask; m; m &= m - 1) atomicAdd(&s_cnt[a.R + __ffsll((long long)m) - 1], 1);
      }
    }
  }
  if (bad) set_status(ctx.status, MOE_ERR_BAD_INPUT);
  __syncthreads();
  for (int i = tid; i < a.E; i += blockDim.x)
    if (s_hist[i]) atomicAdd(&ra.counts[i], s_hist[i]);
  for (int i = tid; i < a.NB; i += blockDim.x)
    if (s_cnt[i]) atomicAdd(&a.totals[i], s_cnt[i]);
  for (int i = tid; i < a.R * a.R; i += blockDim.x)
    if (s_send[i]) atomicAdd(&a.L.send_counts[i], s_send[i]);
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&a.counters[1], 1) == (int)gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  layout::finalize(a, s_er, s_cnt, ctx);  // s_cnt is free again after the flush
  if (ra.rank_active) {
    __syncthreads();
    for (int i = tid; i < a.R; i += blockDim.x) s_send[i] = 0;
    __syncthreads();
    for (int i = tid; i < a.E; i += blockDim.x)
      if (__ldcg(ra.counts + i) > 0) atomicAdd(&s_send[s_er[i]], 1);
    __syncthreads();
    for (int i = tid; i < a.R; i += blockDim.x) ra.rank_active[i] = s_send[i];
  }
}

template <int EPL>
cudaError_t launch_epl(const RouteArgs &ra, const LayoutArgs &a, const DeviceCtx &ctx, cudaStream_t s) {
  long blocks = ((long)a.T + 63) / 64;  // >= 64 tokens per block
  const long cap = (long)ctx.num_sms * 4;
  if (blocks > cap) blocks = cap;
  if (a.E == 32 * EPL)
    route_count_kernel<EPL, true><<<(unsigned)blocks, 256, 0, s>>>(ra, a, ctx);
  else
    route_count_kernel<EPL, false><<<(unsigned)blocks, 256, 0, s>>>(ra, a, ctx);
  return count_launch(cudaGetLastError());
}

}  // namespace

cudaError_t launch_route_layout_static(const float *logits, int T, int E, int k, int n_groups,
                                       int gpt, int renorm, const int *expert_rank,
                                       int tokens_per_rank, int R, int rpg, int mode, int *idx,
                                       float *w, int *counts, int *rank_active,
                                       const moe_layout &L, void *ws, const DeviceCtx &ctx,
                                       cudaStream_t s) {
  cudaError_t err = cudaMemsetAsync(counts, 0, sizeof(int) * (size_t)E, s);
  if (err != cudaSuccess) return err;
  if (T == 0) {
    if (rank_active && (err = cudaMemsetAsync(rank_active, 0, sizeof(int) * (size_t)R, s)) != cudaSuccess)
      return err;
    return layout::layout_empty(L, R, rpg, mode, s);
  }
  const LayoutArgs a = layout::make_layout_args(idx, w, expert_rank, T, tokens_per_rank, k, E, R,
                                                rpg, mode, L, ws);
  if ((err = layout::layout_clear(a, s)) != cudaSuccess) return err;
  RouteArgs ra{logits, n_groups, gpt, renorm, idx, w, counts, rank_active};
  const int epl = (E + 31) / 32;
  if (epl <= 1) err = launch_epl<1>(ra, a, ctx, s);
  else if (epl <= 2) err = launch_epl<2>(ra, a, ctx, s);
  else if (epl <= 4) err = launch_epl<4>(ra, a, ctx, s);
  else if (epl <= 8) err = launch_epl<8>(ra, a, ctx, s);
  else if (epl <= 16) err = launch_epl<16>(ra, a, ctx, s);
  else err = launch_epl<32>(ra, a, ctx, s);
  if (err != cudaSuccess) return err;
  return layout::launch_layout_place(a, ctx, s);
}

}  // namespace moe
