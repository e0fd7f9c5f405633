// METRO greedy replica assignment by one block (shared by the assignment
// kernel and the fused single-launch front end).
//
// "METRO AllGather vs AllToAll for MoE decode" (fanout.sh), sections "changes
// the routing information" and "Add the expert-weight traffic term": each
// active expert goes to one of its replicas on the GPU with the fewest
// already-activated experts (a greedy, not the optimal min-max assignment).
// Experts are visited in ascending id; ties go to the lower rank, then to the
// lower slot id.
//
// The whole block stages the demand vector and the replica map in shared
// memory (each replica entry pre-packed as rank << 15 | slot).  Warp 0 then
// walks the experts 32 at a time.  An expert with one valid replica has no
// choice: its rank only gains one activated expert, so the forced experts
// between two experts with a choice are applied together with shared-memory
// atomics.  For an expert with a choice the lanes form the key
// activated[rank] << 21 | rank << 15 | slot of its replicas and one
// redux.sync.min picks the winner, so the tie rules are the key's bit order.
// The serial chain is only as long as the number of experts with a choice.
#pragma once

#include "moe_internal.cuh"

namespace moe {

// Shared memory metro_assign uses, in ints (besides s_active[kMaxR]).
__host__ __device__ inline int assign_smem_ints(int E, int n_entries) { return 2 * E + 1 + n_entries; }

// Every thread of the block calls it; `sm` holds assign_smem_ints() ints.
// counts are read through L2 (they may have been written by other blocks of
// the same launch).  Returns after a __syncthreads, with every output written.
__device__ __forceinline__ void metro_assign(const int *counts, int E, const int *__restrict__ off,
                                             const int *__restrict__ slots, int n_entries,
                                             const int *__restrict__ slot_rank, int S, int R,
                                             int *expert_slot, int *expert_rank, int *rank_active,
                                             int *sm, int *s_active, const DeviceCtx &ctx) {
  constexpr unsigned kFull = 0xffffffffu;
  int *s_off = sm;              // E + 1
  int *s_cnt = s_off + E + 1;   // E
  int *s_key = s_cnt + E;       // n_entries: rank << 15 | slot, or -1 if invalid
  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_off[i] = off[i];
  for (int i = threadIdx.x; i < E; i += blockDim.x) s_cnt[i] = __ldcg(counts + i);
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
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    bool bad = false;
    for (int base = 0; base < E; base += 32) {
      // classify this lane's expert: inactive, forced (one valid replica), or a choice
      const int e = base + lane;
      int kind = 0;        // 0 inactive / out of range, 1 forced, 2 choice
      int fkey = -1;       // the forced expert's key
      int lo = 0, hi = 0;
      if (e < E) {
        const int c = s_cnt[e];
        lo = s_off[e];
        hi = s_off[e + 1];
        if (c < 0 || lo < 0 || hi > n_entries || lo > hi) {
          bad = true;
          lo = hi = 0;
        }
        if (c > 0) {
          int nvalid = 0;
          for (int i = lo; i < hi && nvalid < 2; ++i)
            if (s_key[i] >= 0) {
              ++nvalid;
              fkey = s_key[i];
            }
          if (nvalid == 0) bad = true;  // active expert without a valid replica
          kind = (nvalid == 0) ? 0 : (nvalid == 1 ? 1 : 2);
        }
      }
      unsigned choice = __ballot_sync(kFull, kind == 2);
      int done_below = 0;  // forced lanes below this index are already applied
      while (true) {
        const int m = choice ? __ffs(choice) - 1 : 32;
        if (kind == 1 && lane >= done_below && lane < m) atomicAdd(&s_active[fkey >> 15], 1);
        __syncwarp();
        if (m == 32) break;
        // expert base + m has a choice: evaluate its replicas against the counts so far
        const int me = base + m;
        const int mlo = __shfl_sync(kFull, lo, m), mhi = __shfl_sync(kFull, hi, m);
        unsigned best = 0xffffffffu;
        for (int i = mlo + lane; i < mhi; i += 32) {
          const int kb = s_key[i];
          if (kb >= 0) best = min(best, ((unsigned)s_active[kb >> 15] << 21) | (unsigned)kb);
        }
        best = __reduce_min_sync(kFull, best);
        if (lane == 0) {
          const int r = (best >> 15) & 63;
          expert_slot[me] = best & 0x7fff;
          expert_rank[me] = r;
          s_active[r] += 1;
        }
        __syncwarp();
        done_below = m + 1;
        choice &= choice - 1;
      }
      if (e < E && kind != 2) {
        expert_slot[e] = (kind == 1) ? (fkey & 0x7fff) : -1;
        expert_rank[e] = (kind == 1) ? (fkey >> 15) : -1;
      }
    }
    if (__any_sync(kFull, bad) && lane == 0) set_status(ctx.status, MOE_ERR_BAD_INPUT);
    __syncwarp();
    for (int r = lane; r < R; r += 32) rank_active[r] = s_active[r];
  }
  __syncthreads();
}

}  // namespace moe
