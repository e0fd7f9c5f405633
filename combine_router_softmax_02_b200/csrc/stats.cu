// Workload statistics of one dispatch, and the token-balanced comparison policy.
//
// dispatch_stats: the gist.science summary of DODOCO ("Methodology") summarises
// the send-count matrix S by the per-expert max/mean ratio (routing skew,
// independent of the expert-to-rank map) and the Gini coefficient of per-rank
// load.  Per-rank load is read as the rows each destination rank receives
// (column sums of S).  All sums are exact 64-bit integers; the four ratios
// are formed in float64 at the end.
//
// token_balanced: the EPLB token-routing policy that "METRO AllGather vs
// AllToAll for MoE decode" compares METRO with ("Add the expert-weight
// traffic term", "Know what the paper actually measured"): each expert's
// tokens are dealt round-robin over its replicas in ascending slot id, and
// every replica that receives a token is activated.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;

// Block-wide reduction of a 64-bit value (sum or max), result on every thread.
template <bool kMax>
__device__ long long block_reduce(long long v, long long *scratch) {
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) {
    const long long o = __shfl_xor_sync(0xffffffffu, v, d);
    v = kMax ? max(v, o) : v + o;
  }
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) scratch[warp] = v;
  __syncthreads();
  long long r = scratch[0];
  for (int w = 1; w < kThreads / 32; ++w) r = kMax ? max(r, scratch[w]) : r + scratch[w];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kThreads) dispatch_stats_kernel(const int *__restrict__ counts,
                                                                  int E, const int *__restrict__ S,
                                                                  int R, double *__restrict__ out,
                                                                  DeviceCtx ctx) {
  __shared__ long long scratch[kThreads / 32];
  __shared__ long long s_load[kMaxR];
  const int tid = threadIdx.x;
  bool bad = false;
  long long cmax = 0, csum = 0;
  for (int e = tid; e < E; e += kThreads) {
    const int c = counts[e];
    if (c < 0) bad = true;
    cmax = max(cmax, (long long)c);
    csum += c;
  }
  cmax = block_reduce<true>(cmax, scratch);
  csum = block_reduce<false>(csum, scratch);
  long long diag = 0;
  for (int r = tid; r < R; r += kThreads) {
    long long l = 0;
    for (int s = 0; s < R; ++s) l += S[s * R + r];
    s_load[r] = l;
    diag += S[r * R + r];
  }
  __syncthreads();
  diag = block_reduce<false>(diag, scratch);
  long long lmax = 0, lsum = 0, gsum = 0;
  for (int r = tid; r < R; r += kThreads) {
    lmax = max(lmax, s_load[r]);
    lsum += s_load[r];
  }
  for (int p = tid; p < R * R; p += kThreads) {
    const long long d = s_load[p / R] - s_load[p % R];
    gsum += d < 0 ? -d : d;
  }
  lmax = block_reduce<true>(lmax, scratch);
  lsum = block_reduce<false>(lsum, scratch);
  gsum = block_reduce<false>(gsum, scratch);
  if (tid == 0) {
    out[0] = csum ? (double)cmax * E / (double)csum : 0.0;
    out[1] = lsum ? (double)gsum / (2.0 * R * (double)lsum) : 0.0;
    out[2] = lsum ? (double)lmax * R / (double)lsum : 0.0;
    out[3] = lsum ? (double)diag / (double)lsum : 0.0;
  }
  if (bad) set_status(ctx.status, MOE_ERR_BAD_INPUT);
}

__global__ void __launch_bounds__(kThreads) token_balanced_kernel(
    const int *__restrict__ counts, int E, const int *__restrict__ off,
    const int *__restrict__ slots, int n_entries, const int *__restrict__ slot_rank, int S, int R,
    int *__restrict__ slot_tokens, int *__restrict__ rank_active, DeviceCtx ctx) {
  __shared__ int s_act[kMaxR];
  const int tid = threadIdx.x;
  for (int s = tid; s < S; s += kThreads) slot_tokens[s] = 0;
  for (int r = tid; r < R; r += kThreads) s_act[r] = 0;
  __syncthreads();
  bool bad = false;
  for (int e = tid; e < E; e += kThreads) {
    const int c = counts[e];
    int lo = off[e], hi = off[e + 1];
    if (c < 0 || lo < 0 || hi > n_entries || lo > hi) {
      bad = true;
      continue;
    }
    if (c == 0) continue;
    int n = 0;
    for (int i = lo; i < hi; ++i) {
      const int s = slots[i];
      if ((unsigned)s < (unsigned)S && (unsigned)slot_rank[s] < (unsigned)R) ++n;
    }
    if (n == 0) {
      bad = true;  // active expert without a valid replica
      continue;
    }
    for (int i = lo; i < hi; ++i) {
      const int s = slots[i];
      if ((unsigned)s >= (unsigned)S || (unsigned)slot_rank[s] >= (unsigned)R) continue;
      int pos = 0;  // rank of this replica among the valid ones, by slot id
      for (int i2 = lo; i2 < hi; ++i2) {
        const int s2 = slots[i2];
        if ((unsigned)s2 < (unsigned)S && (unsigned)slot_rank[s2] < (unsigned)R && s2 < s) ++pos;
      }
      const int tok = c / n + (pos < c % n ? 1 : 0);
      slot_tokens[s] = tok;
      if (tok > 0) atomicAdd(&s_act[slot_rank[s]], 1);
    }
  }
  __syncthreads();
  for (int r = tid; r < R; r += kThreads) rank_active[r] = s_act[r];
  if (bad) set_status(ctx.status, MOE_ERR_BAD_INPUT);
}

}  // namespace

cudaError_t launch_dispatch_stats(const int *counts, int E, const int *send_counts, int R,
                                  double *stats, const DeviceCtx &ctx, cudaStream_t s) {
  dispatch_stats_kernel<<<1, kThreads, 0, s>>>(counts, E, send_counts, R, stats, ctx);
  return count_launch(cudaGetLastError());
}

cudaError_t launch_token_balanced(const int *counts, int E, const int *off, const int *slots,
                                  int n_entries, const int *slot_rank, int S, int R,
                                  int *slot_tokens, int *rank_active, const DeviceCtx &ctx,
                                  cudaStream_t s) {
  token_balanced_kernel<<<1, kThreads, 0, s>>>(counts, E, off, slots, n_entries, slot_rank, S, R,
                                               slot_tokens, rank_active, ctx);
  return count_launch(cudaGetLastError());
}

}  // namespace moe
