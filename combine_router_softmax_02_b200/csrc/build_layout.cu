// Stable per-destination row layout in one cooperative launch.
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
// A row's id is seg_off[bin] + (rows of the bin in earlier blocks) + (rows of
// the bin in earlier tiles of the block) + (rows in earlier warps of the tile)
// + (rows in earlier lanes of the warp): the stable (token-order) prefix scan.
// Phase 1 counts every block's rows per bin, a grid barrier publishes the
// count table, phase 2 scans it and writes the rows (layout_common.cuh).
// Small token sets in the mask modes take one pass instead: every block counts
// every token itself, with no count table and no barrier.
// Ranks and groups (at most 64 each) are 64-bit masks per token, one ballot
// per bin per warp; experts (PER_PICK, up to 1024 bins) are merged in
// ascending (rank, expert) order with redux.sync.min.
#include "layout_common.cuh"

namespace moe {
namespace layout {
namespace {

template <int KM, int MODE>
__global__ void __launch_bounds__(kTile) layout_kernel(LayoutArgs a, DeviceCtx ctx) {
  extern __shared__ int4 smem_raw[];
  int *sm = reinterpret_cast<int *>(smem_raw);
  __shared__ int s_flag;
  const SmemPlan P = smem_plan(a.E, a.NBp, a.R, false);
  const int t0 = blockIdx.x * a.chunk, t1 = min(a.T, t0 + a.chunk);
  smem_init(a, P, sm);
  layout_phases<KM, MODE>(a, P, sm, t0, t1, ctx, &s_flag, 1);
}

// Small token sets in the mask modes: one pass, no count table, no barrier
// (a kernel of its own, so the two-phase kernel's code stays as it is).
template <int KM, int MODE>
__global__ void __launch_bounds__(kTile) layout_one_pass_kernel(LayoutArgs a, DeviceCtx ctx) {
  extern __shared__ int4 smem_raw[];
  int *sm = reinterpret_cast<int *>(smem_raw);
  const SmemPlan P = smem_plan(a.E, a.NBp, a.R, false);
  const int t0 = blockIdx.x * a.chunk, t1 = min(a.T, t0 + a.chunk);
  smem_init(a, P, sm);
  layout_single_pass<KM, MODE>(a, P, sm, t0, t1, ctx);
}

std::atomic<unsigned long long> g_smem_set[4][3][2];

template <int KM, int MODE>
cudaError_t launch_k(const LayoutArgs &a0, int kind, const DeviceCtx &ctx, cudaStream_t s) {
  LayoutArgs a = a0;
  const size_t smem = sizeof(int) * (size_t)smem_plan(a.E, a.NBp, a.R, false).total;
  const bool one = single_pass(a.T, MODE);
  auto kern = layout_kernel<KM, MODE>;
  if constexpr (MODE != MOE_LAYOUT_PER_PICK)
    if (one) kern = layout_one_pass_kernel<KM, MODE>;
  cudaError_t err = set_smem_limit_once(kern, 200 * 1024, g_smem_set[kind][MODE][one]);
  if (err != cudaSuccess) return err;
  int resident = 0;
  if ((err = max_resident_blocks((const void *)kern, smem, ctx, resident)) != cudaSuccess) return err;
  // blocks per SM: a sweep over 1-4 picked 2 for DEDUP on the 65536-token
  // workload (25.6 us against 28.8-29.0) and 1 for TWO_HOP on the two-hop one
  // (28.9 us against 32.1-32.5)
  const int bps = MODE == MOE_LAYOUT_TWO_HOP ? 1 : kBlocksPerSm;
  split_tokens(a.T, resident < bps * ctx.num_sms ? resident : bps * ctx.num_sms, a.nblk, a.chunk);
  if (!one)  // the barrier words start at zero
    if ((err = cudaMemsetAsync(a.bar, 0, sizeof(int) * 16, s)) != cudaSuccess) return err;
  void *args[] = {&a, const_cast<DeviceCtx *>(&ctx)};
  err = cudaLaunchCooperativeKernel((const void *)kern, dim3(a.nblk), dim3(kTile), args, smem, s);
  if (err != cudaSuccess) return err;
  return count_launch(cudaGetLastError());
}

template <int KM>
cudaError_t launch_km(const LayoutArgs &a, int kind, const DeviceCtx &ctx, cudaStream_t s) {
  if (a.mode == MOE_LAYOUT_PER_PICK) return launch_k<KM, MOE_LAYOUT_PER_PICK>(a, kind, ctx, s);
  if (a.mode == MOE_LAYOUT_TWO_HOP) return launch_k<KM, MOE_LAYOUT_TWO_HOP>(a, kind, ctx, s);
  return launch_k<KM, MOE_LAYOUT_DEDUP>(a, kind, ctx, s);
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
  a.NBp = (a.NB + 3) & ~3;
  a.nblk = 0;
  a.chunk = 0;
  a.bar = static_cast<unsigned *>(ws);
  a.cnt = static_cast<int *>(ws) + 16;
  a.agg = static_cast<int *>(ws) + kHeaderInts;
  a.L = L;
  return a;
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

cudaError_t max_resident_blocks(const void *kernel, size_t smem, const DeviceCtx &ctx, int &blocks) {
  int per_sm = 0;
  cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kTile, smem);
  if (err != cudaSuccess) return err;
  blocks = per_sm * ctx.num_sms;
  return blocks > 0 ? cudaSuccess : cudaErrorInvalidConfiguration;
}

}  // namespace layout

size_t layout_workspace_bytes(int T, int k, int E, int R, int rpg, int mode) {
  (void)k;
  const int NBp = (layout::num_bins(E, R, rpg, mode) + 3) & ~3;
  long rows = ((long)T + 7) / 8;  // chunks are multiples of 8 tokens
  if (rows > layout::kMaxBlocks) rows = layout::kMaxBlocks;
  if (rows < 1) rows = 1;
  return sizeof(int) * (layout::kHeaderInts + (size_t)rows * NBp);
}

cudaError_t launch_build_layout(const int *idx, const float *w, const int *expert_rank, int T,
                                int tokens_per_rank, int k, int E, int R, int rpg, int mode,
                                const moe_layout &L, void *ws, const DeviceCtx &ctx,
                                cudaStream_t s) {
  if (T == 0) return layout::layout_empty(L, R, rpg, mode, s);
  const layout::LayoutArgs a =
      layout::make_layout_args(idx, w, expert_rank, T, tokens_per_rank, k, E, R, rpg, mode, L, ws);
  if (k <= 2) return layout::launch_km<2>(a, 0, ctx, s);
  if (k <= 4) return layout::launch_km<4>(a, 1, ctx, s);
  if (k <= 8) return layout::launch_km<8>(a, 2, ctx, s);
  return layout::launch_km<16>(a, 3, ctx, s);
}

}  // namespace moe
