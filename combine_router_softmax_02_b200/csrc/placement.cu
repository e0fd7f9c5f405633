// Correlated expert placement: co-selection counts and a greedy placement.
//
// The ainewsletter summary of arXiv:2610.09372 ("Correlations in router
// choices", "Two locality techniques") places experts that the router often
// selects together on the same GPU, so that a single-send dispatcher sends
// fewer rows.  It gives no algorithm.  Here:
//   coselection_kernel   C[e][f] = tokens that picked both e and f (e != f),
//                        one warp per token, global atomics;
//   placement_kernel     one CTA grows the ranks one at a time, E/R experts
//                        each: seed = the unplaced expert of highest demand,
//                        then the unplaced expert with the most co-selections
//                        with the rank so far (ties: higher demand, then the
//                        lower id).  Each step is two block-wide argmax
//                        reductions over the experts.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kThreads = 1024;

__global__ void __launch_bounds__(256) coselection_kernel(const int *__restrict__ idx, int T, int k,
                                                          int E, int *__restrict__ C, DeviceCtx ctx) {
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  bool bad = false;
  for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += gridDim.x * wpb) {
    int e = -1;
    if (lane < k) {
      e = __ldcs(idx + (size_t)t * k + lane);
      if ((unsigned)e >= (unsigned)E) {
        bad = true;
        e = -1;
      }
    }
    for (int j = 0; j < k; ++j) {
      const int f = __shfl_sync(0xffffffffu, e, j);
      if (lane < k && lane != j && e >= 0 && f >= 0) atomicAdd(&C[(size_t)e * E + f], 1);
    }
  }
  if (bad) set_status(ctx.status, MOE_ERR_BAD_INPUT);
}

// Block-wide max of an unsigned 64-bit key; every thread gets the result.
__device__ unsigned long long block_max(unsigned long long v, unsigned long long *scratch) {
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, d));
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
  __syncthreads();
  unsigned long long r = scratch[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) r = max(r, scratch[w]);
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kThreads) placement_kernel(const int *__restrict__ C,
                                                             const int *__restrict__ counts, int E,
                                                             int R, int *__restrict__ expert_rank,
                                                             DeviceCtx ctx) {
  __shared__ long long s_aff[kMaxE];
  __shared__ int s_rank[kMaxE];
  __shared__ unsigned long long scratch[kThreads / 32];
  const int tid = threadIdx.x;
  const int cap = E / R;
  bool bad = false;
  for (int e = tid; e < E; e += blockDim.x) {
    s_rank[e] = -1;
    if (counts[e] < 0) bad = true;
  }
  __syncthreads();
  // (demand, -id) as a key: larger demand first, then the lower id
  auto demand_key = [&](int e) {
    return ((unsigned long long)(unsigned)max(counts[e], 0) << 32) | (unsigned)(kMaxE - e);
  };
  for (int r = 0; r < R; ++r) {
    unsigned long long best = 0;
    for (int e = tid; e < E; e += blockDim.x)
      if (s_rank[e] < 0) best = max(best, demand_key(e));
    int pick = kMaxE - (int)(block_max(best, scratch) & 0xffffffffu);
    for (int m = 0;; ++m) {
      if (tid == 0) s_rank[pick] = r;
      __syncthreads();
      if (m == cap - 1) break;
      for (int e = tid; e < E; e += blockDim.x) {
        const long long c = C[(size_t)pick * E + e];  // symmetric: row of the new member
        s_aff[e] = (m == 0 ? 0 : s_aff[e]) + c;
      }
      __syncthreads();
      long long amax = -1;
      for (int e = tid; e < E; e += blockDim.x)
        if (s_rank[e] < 0) amax = max(amax, s_aff[e]);
      amax = (long long)block_max((unsigned long long)(amax + 1), scratch) - 1;
      best = 0;
      for (int e = tid; e < E; e += blockDim.x)
        if (s_rank[e] < 0 && s_aff[e] == amax) best = max(best, demand_key(e));
      pick = kMaxE - (int)(block_max(best, scratch) & 0xffffffffu);
    }
  }
  for (int e = tid; e < E; e += blockDim.x) expert_rank[e] = s_rank[e];
  if (bad && tid == 0) set_status(ctx.status, MOE_ERR_BAD_INPUT);
}

}  // namespace

cudaError_t launch_coselection(const int *idx, int T, int k, int E, int *C, const DeviceCtx &ctx,
                               cudaStream_t s) {
  cudaError_t err = cudaMemsetAsync(C, 0, sizeof(int) * (size_t)E * E, s);
  if (err != cudaSuccess || T == 0) return err;
  long blocks = ((long)T + 7) / 8;
  const long cap = (long)ctx.num_sms * 16;
  if (blocks > cap) blocks = cap;
  coselection_kernel<<<(unsigned)blocks, 256, 0, s>>>(idx, T, k, E, C, ctx);
  return count_launch(cudaGetLastError());
}

cudaError_t launch_placement(const int *C, const int *counts, int E, int R, int *expert_rank,
                             const DeviceCtx &ctx, cudaStream_t s) {
  placement_kernel<<<1, kThreads, 0, s>>>(C, counts, E, R, expert_rank, ctx);
  return count_launch(cudaGetLastError());
}

}  // namespace moe
