// METRO greedy replica assignment, one CTA.
//
// "METRO AllGather vs AllToAll for MoE decode" (fanout.sh), sections "changes
// the routing information" and "Add the expert-weight traffic term": each
// active expert goes to one of its replicas on the GPU with the fewest
// already-activated experts (a greedy, not the optimal min-max assignment).
// Experts are visited in ascending id; ties go to the lower rank, then to the
// lower slot id.
//
// The whole CTA stages the demand vector and the replica map in shared memory
// (each replica entry pre-packed as rank << 15 | slot); warp 0 then runs the
// serial greedy.  For each active expert the lanes form the key
// activated[rank] << 21 | rank << 15 | slot of its replicas and one
// redux.sync.min picks the winner, so the tie rules are the key's bit order.
#include "moe_internal.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) replica_assign_kernel(
    const int *__restrict__ counts, int E, const int *__restrict__ off,
    const int *__restrict__ slots, int n_entries, const int *__restrict__ slot_rank, int S, int R,
    int *__restrict__ expert_slot, int *__restrict__ expert_rank, int *__restrict__ rank_active,
    DeviceCtx ctx) {
  extern __shared__ int sm[];
  int *s_off = sm;              // E + 1
  int *s_cnt = s_off + E + 1;   // E
  int *s_key = s_cnt + E;       // n_entries: rank << 15 | slot, or -1 if invalid
  __shared__ int s_active[kMaxR];

  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_off[i] = off[i];
  for (int i = threadIdx.x; i < E; i += blockDim.x) s_cnt[i] = counts[i];
  for (int i = threadIdx.x; i < n_entries; i += blockDim.x) {
    const int sl = slots[i];
    int key = -1;
    if ((unsigned)sl < (unsigned)S) {
      const int r = slot_rank[sl];
      if ((unsigned)r < (unsigned)R) key = (r << 15) | sl;
    }
    s_key[i] = key;
  }
  for (int i = threadIdx.x; i < R; i += blockDim.x) s_active[i] = 0;
  __syncthreads();
  if (threadIdx.x >= 32) return;

  const int lane = threadIdx.x;
  bool bad = false;
  for (int e = 0; e < E; ++e) {
    const int c = s_cnt[e];
    int lo = s_off[e], hi = s_off[e + 1];
    if (c < 0) bad = true;
    if (lo < 0 || hi > n_entries || lo > hi) {
      bad = true;
      lo = hi = 0;
    }
    unsigned best = 0xffffffffu;
    if (c > 0) {
      for (int i = lo + lane; i < hi; i += 32) {
        const int kb = s_key[i];
        if (kb >= 0) best = min(best, ((unsigned)s_active[kb >> 15] << 21) | (unsigned)kb);
      }
      best = __reduce_min_sync(0xffffffffu, best);
    }
    if (lane == 0) {
      if (c > 0 && best != 0xffffffffu) {
        const int r = (best >> 15) & 63;
        expert_slot[e] = best & 0x7fff;
        expert_rank[e] = r;
        s_active[r] += 1;
      } else {
        if (c > 0) bad = true;  // active expert without a valid replica
        expert_slot[e] = -1;
        expert_rank[e] = -1;
      }
    }
    __syncwarp();
  }
  if (bad) set_status(ctx.status, MOE_ERR_BAD_INPUT);
  for (int r = lane; r < R; r += 32) rank_active[r] = s_active[r];
}

}  // namespace

cudaError_t launch_replica_assign(const int *counts, int E, const int *off, const int *slots,
                                  int n_entries, const int *slot_rank, int S, int R,
                                  int *expert_slot, int *expert_rank, int *rank_active,
                                  const DeviceCtx &ctx, cudaStream_t s) {
  const size_t smem = sizeof(int) * ((size_t)2 * E + 1 + n_entries);
  static std::atomic<unsigned long long> done{0};
  cudaError_t err = set_smem_limit_once(replica_assign_kernel,
                                        (int)(sizeof(int) * (2 * kMaxE + 1 + kMaxSlots)), done);
  if (err != cudaSuccess) return err;
  replica_assign_kernel<<<1, 256, smem, s>>>(counts, E, off, slots, n_entries, slot_rank, S, R,
                                             expert_slot, expert_rank, rank_active, ctx);
  return count_launch(cudaGetLastError());
}

}  // namespace moe
