// Pieces of the layout shared by the layout kernels and the fused
// static-placement kernel: arguments, warp helpers, and the final scan of the
// per-bin totals into segment offsets (see build_layout.cu).
#pragma once

#include "moe_internal.cuh"

namespace moe {
namespace layout {

constexpr int kTile = 256;  // tokens per tile, one per thread
constexpr int kWarps = kTile / 32;
constexpr int kMaxBins = kMaxE;  // >= max(E, R + G)
constexpr int kSendSmem = kMaxR * kMaxR;
constexpr unsigned kFull = 0xffffffffu;
constexpr unsigned long long kFlagAgg = 1ull << 32;
constexpr unsigned long long kFlagInc = 2ull << 32;

struct LayoutArgs {
  const int *idx;
  const float *w;
  const int *expert_rank;
  int T, tpr, k, E, R, rpg, G, mode, NB, num_tiles;
  int *counters;  // [0] place-kernel ticket, [1] count-kernel blocks done
  int *totals;    // [NB]
  int *seg_off;   // [NB]
  unsigned long long *state;  // [num_tiles][NB]: flag << 32 | count
  moe_layout L;
};

__device__ __forceinline__ unsigned long long warp_or64(unsigned long long m) {
  const unsigned lo = __reduce_or_sync(kFull, (unsigned)m);
  const unsigned hi = __reduce_or_sync(kFull, (unsigned)(m >> 32));
  return ((unsigned long long)hi << 32) | lo;
}

// Bins given as 64-bit masks (ranks, or groups): for every bin present in the
// warp, f(bin, has, ball) runs on all lanes with the warp's ballot of the bin.
template <class F>
__device__ __forceinline__ void warp_mask_bins(unsigned long long mask, F &&f) {
  unsigned long long wm = warp_or64(mask);
  while (wm) {
    const int b = __ffsll((long long)wm) - 1;
    wm &= wm - 1;
    const bool has = (mask >> b) & 1ull;
    f(b, has, __ballot_sync(kFull, has));
  }
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ unsigned long long group_bits(int g, int rpg) {
  const unsigned long long ones = (rpg >= 64) ? ~0ull : ((1ull << rpg) - 1ull);
  return (rpg >= 64) ? ones : (ones << (g * rpg));
}

// ------------------------------------------------------------- finalize ----
// Runs in the last count block, all threads: the totals are loaded into
// shared memory in parallel (tot), then thread 0 scans them into segment
// offsets and the host-visible offsets.
__device__ __forceinline__ void finalize(const LayoutArgs &a, const int *s_er, int *tot, DeviceCtx ctx) {
  for (int i = threadIdx.x; i < a.NB; i += blockDim.x) tot[i] = __ldcg(a.totals + i);
  __syncthreads();
  if (threadIdx.x != 0) return;
  const moe_layout &L = a.L;
  if (a.mode == MOE_LAYOUT_PER_PICK) {
    int base[kMaxR + 1];
    for (int r = 0; r <= a.R; ++r) base[r] = 0;
    for (int e = 0; e < a.E; ++e) {
      const int r = s_er[e];
      if ((unsigned)r < (unsigned)a.R) base[r + 1] += tot[e];
    }
    for (int r = 0; r < a.R; ++r) base[r + 1] += base[r];
    for (int r = 0; r <= a.R; ++r) L.rank_offsets[r] = base[r];
    const int n = base[a.R];
    for (int e = 0; e < a.E; ++e) {
      const int r = s_er[e];
      if ((unsigned)r < (unsigned)a.R) {
        a.seg_off[e] = base[r];
        base[r] += tot[e];
      } else {
        a.seg_off[e] = 0;
      }
    }
    *L.num_rows = n;
    if (n > L.capacity) set_status(ctx.status, MOE_ERR_CAPACITY);
    return;
  }
  int run = 0;
  for (int r = 0; r < a.R; ++r) {
    a.seg_off[r] = run;
    L.rank_offsets[r] = run;
    run += tot[r];
  }
  L.rank_offsets[a.R] = run;
  *L.num_rows = run;
  if (run > L.capacity) set_status(ctx.status, MOE_ERR_CAPACITY);
  if (a.mode == MOE_LAYOUT_TWO_HOP) {
    int run1 = 0;
    for (int g = 0; g < a.G; ++g) {
      a.seg_off[a.R + g] = run1;
      L.group_offsets[g] = run1;
      run1 += tot[a.R + g];
    }
    L.group_offsets[a.G] = run1;
    *L.num_rows_hop1 = run1;
    if (run1 > L.capacity_hop1) set_status(ctx.status, MOE_ERR_CAPACITY);
  }
}

inline int num_bins(int E, int R, int rpg, int mode) {
  if (mode == MOE_LAYOUT_PER_PICK) return E;
  if (mode == MOE_LAYOUT_TWO_HOP) return R + R / rpg;
  return R;
}

inline size_t align16(size_t x) { return (x + 15) & ~(size_t)15; }

// Arguments of one layout over the caller's buffers and workspace.
LayoutArgs make_layout_args(const int *idx, const float *w, const int *expert_rank, int T,
                            int tokens_per_rank, int k, int E, int R, int rpg, int mode,
                            const moe_layout &L, void *ws);
// Clears the counters, totals and the send-count matrix (stream-ordered).
cudaError_t layout_clear(const LayoutArgs &a, cudaStream_t s);
// Outputs of an empty token set.
cudaError_t layout_empty(const moe_layout &L, int R, int rpg, int mode, cudaStream_t s);
// The place kernel, once the count phase (totals, segment offsets, cleared
// scan state) is complete.
cudaError_t launch_layout_place(const LayoutArgs &a, const DeviceCtx &ctx, cudaStream_t s);

}  // namespace layout
}  // namespace moe
