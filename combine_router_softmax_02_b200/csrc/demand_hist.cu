// Global per-expert demand vector: counts[e] = #(token, pick) with idx == e.
//
// "METRO AllGather vs AllToAll for MoE decode" (fanout.sh), section "changes
// the routing information": every rank computes the same global expert demand
// vector from the gathered token set.
//
// Block-then-global histogram: each block counts its share of the picks in
// shared memory (one atomic per group of equal ids in a warp, found with
// match.any), then adds its non-zero bins to the global vector.  Integer
// adds commute, so the result is exact and independent of scheduling.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kPer = 8;  // picks per thread per pass, all loaded before any is counted

__global__ void __launch_bounds__(256) demand_hist_kernel(const int *__restrict__ idx, long n,
                                                          int E, int *__restrict__ counts,
                                                          DeviceCtx ctx) {
  extern __shared__ int h[];
  for (int i = threadIdx.x; i < E; i += blockDim.x) h[i] = 0;
  __syncthreads();
  // a pass covers kPer warp-widths per warp: lane l of warp w takes picks
  // base + j * 32 + l, j < kPer (coalesced per j); every lane of a warp runs
  // the same passes, so the warp is converged at match.any
  const long per_block = (long)blockDim.x * kPer;
  const long stride = (long)gridDim.x * per_block;
  const int lane = threadIdx.x & 31;
  const long base0 = (long)blockIdx.x * per_block + (long)(threadIdx.x >> 5) * 32 * kPer;
  bool bad = false;
  for (long base = base0; base < n; base += stride) {
    int e[kPer];
    unsigned live = 0;  // which of this lane's slots hold a pick
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const long i = base + j * 32 + lane;
      e[j] = 0;
      if (i < n) {
        e[j] = __ldcs(idx + i);
        live |= 1u << j;
      }
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      int v = (live >> j & 1u) ? e[j] : -1;
      if ((live >> j & 1u) && (unsigned)v >= (unsigned)E) {
        bad = true;
        v = -1;
      }
      const unsigned peers = __match_any_sync(0xffffffffu, v);
      if (v >= 0 && lane == __ffs(peers) - 1) atomicAdd(&h[v], __popc(peers));
    }
  }
  if (bad) set_status(ctx.status, MOE_ERR_BAD_INPUT);
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x)
    if (h[i]) atomicAdd(&counts[i], h[i]);
}

}  // namespace

cudaError_t launch_demand_hist(const int *idx, int T, int k, int E, int *counts,
                               const DeviceCtx &ctx, cudaStream_t s) {
  cudaError_t err = cudaMemsetAsync(counts, 0, sizeof(int) * (size_t)E, s);
  if (err != cudaSuccess) return err;
  const long n = (long)T * k;
  if (n == 0) return cudaSuccess;
  long blocks = (n + 256 * kPer - 1) / (256 * kPer);
  const long cap = (long)ctx.num_sms * 2;
  if (blocks > cap) blocks = cap;
  demand_hist_kernel<<<(unsigned)blocks, 256, sizeof(int) * (size_t)E, s>>>(idx, n, E, counts, ctx);
  return count_launch(cudaGetLastError());
}

}  // namespace moe
