// METRO greedy replica assignment, one CTA: the kernel around metro_stage and
// metro_solve
// (assign_common.cuh, which states the algorithm and its sources).
#include "assign_common.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) replica_assign_kernel(
    const int *__restrict__ counts, int E, const int *__restrict__ off,
    const int *__restrict__ slots, int n_entries, const int *__restrict__ slot_rank, int S, int R,
    int *__restrict__ expert_slot, int *__restrict__ expert_rank, int *__restrict__ rank_active,
    DeviceCtx ctx) {
  wait_prior_grids();
  extern __shared__ int4 sm_raw[];  // 16-byte aligned
  int *sm = reinterpret_cast<int *>(sm_raw);
  const MetroPlan P = metro_plan(E, n_entries, R);
  metro_stage(E, off, slots, n_entries, slot_rank, S, R, counts, sm, P);
  metro_solve(nullptr, E, R, sm, P, sm + P.total, true, expert_slot, expert_rank, rank_active, ctx);
}

}  // namespace

cudaError_t launch_replica_assign(const int *counts, int E, const int *off, const int *slots,
                                  int n_entries, const int *slot_rank, int S, int R,
                                  int *expert_slot, int *expert_rank, int *rank_active,
                                  const DeviceCtx &ctx, cudaStream_t s) {
  // the plan, then the expert -> rank map the walk leaves in shared memory
  const size_t smem = sizeof(int) * ((size_t)assign_smem_ints(E, n_entries, R) + E);
  static std::atomic<unsigned long long> done{0};
  cudaError_t err = set_smem_limit_once(
      replica_assign_kernel, (int)(sizeof(int) * (assign_smem_ints(kMaxE, kMaxSlots, kMaxR) + kMaxE)), done);
  if (err != cudaSuccess) return err;
  err = launch_after_prior(replica_assign_kernel, dim3(1), dim3(256), smem, s, counts, E, off, slots,
                           n_entries, slot_rank, S, R, expert_slot, expert_rank, rank_active, ctx);
  if (err != cudaSuccess) return err;
  return count_launch(cudaGetLastError());
}

}  // namespace moe
