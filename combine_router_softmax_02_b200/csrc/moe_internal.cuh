// Internal declarations shared by the kernels of libmoe.so (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/moe.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libmoe targets sm_100a only"
#endif

namespace moe {

constexpr int kMaxE = 1024;
constexpr int kMaxK = 16;
constexpr int kMaxR = 64;
constexpr int kMaxGroups = 32;
constexpr int kMaxSlots = 32768;

// Settings every launch receives by value.
struct DeviceCtx {
  int *status;            // per-device status word (first error wins)
  uint64_t wait_limit_ns; // limit of every bounded wait
  int silent_tile;        // layout block that never arrives at its barrier (-1: none)
  int num_sms;
  int smem_per_sm;        // shared memory per SM, bytes
};

// ---------------------------------------------------------------- device ----
__device__ __forceinline__ void set_status(int *status, int code) {
  atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Lanes below this one in the warp.
__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ int ld_volatile_i32(const int *p) {
  int v;
  asm volatile("ld.volatile.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// 16-byte streaming load (read-only path, no L1 allocation).
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_v4(void *p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// Programmatic dependent launch: a kernel launched with launch_after_prior()
// may be scheduled while the kernel before it in the stream is finishing; it
// waits here, before its first global access, until that kernel has completed
// and its writes are visible.  Launched any other way, this returns at once.
__device__ __forceinline__ void wait_prior_grids() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------------ host ----
// Launches `kern` so that its blocks may be scheduled before the previous
// kernel in the stream has completed (the kernel calls wait_prior_grids()
// before touching memory): the launch latency overlaps the previous kernel's
// tail.  Captured into a CUDA graph it becomes a programmatic edge.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_after_prior(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                      cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Raises a kernel's dynamic shared-memory limit once per device.
template <class Kern>
inline cudaError_t set_smem_limit_once(Kern kern, int bytes, std::atomic<unsigned long long> &done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Column slices per row for the one-warp-per-row copy kernels: few rows (the
// decode regime) would leave most SMs idle and each warp walking its whole row
// one dependent round trip after another, so a row is split into slices of
// whole warp-widths (32 16-byte vectors each) until there are about
// `warps_per_sm` warps per SM; many rows keep one slice each.
inline void row_slices(long rows, int nvec, int num_sms, int &slices, int &svec, int warps_per_sm = 32) {
  const long want = (long)num_sms * warps_per_sm;
  long s = rows > 0 ? (want + rows - 1) / rows : 1;
  const long cap = nvec / 32 > 0 ? nvec / 32 : 1;
  if (s > cap) s = cap;
  if (s < 1) s = 1;
  svec = (int)((((long)nvec + s - 1) / s + 31) / 32 * 32);
  if (svec < 1) svec = 1;
  slices = (nvec + svec - 1) / svec;
  if (slices < 1) slices = 1;
}

// Host-side count of kernel launches (moe_kernel_launches); each launch site
// calls count_launch() after a launch that cudaGetLastError() accepted.
extern std::atomic<unsigned long long> g_kernel_launches;
inline cudaError_t count_launch(cudaError_t e) {
  if (e == cudaSuccess) g_kernel_launches.fetch_add(1, std::memory_order_relaxed);
  return e;
}

// Kernel launchers (defined next to their kernels).  Each returns a
// cudaError_t from cudaGetLastError() after the launch.
cudaError_t launch_route_topk(const float *logits, int T, int E, int k, int n_groups, int gpt,
                              int renorm, int *idx, float *w, const DeviceCtx &ctx,
                              cudaStream_t s);
cudaError_t launch_demand_hist(const int *idx, int T, int k, int E, int *counts,
                               const DeviceCtx &ctx, cudaStream_t s);
cudaError_t launch_replica_assign(const int *counts, int E, const int *off, const int *slots,
                                  int n_entries, const int *slot_rank, int S, int R,
                                  int *expert_slot, int *expert_rank, int *rank_active,
                                  const DeviceCtx &ctx, cudaStream_t s);
size_t layout_workspace_bytes(int T, int k, int E, int R, int rpg, int mode);
cudaError_t launch_build_layout(const int *idx, const float *w, const int *expert_rank, int T,
                                int tokens_per_rank, int k, int E, int R, int rpg, int mode,
                                const moe_layout &L, void *ws, const DeviceCtx &ctx,
                                cudaStream_t s);
cudaError_t launch_pack(const void *x, int elem_bytes, int H, const moe_layout &L, void *packed,
                        void *packed_hop1, const DeviceCtx &ctx, cudaStream_t s);
cudaError_t launch_route_layout_static(const float *logits, int T, int E, int k, int n_groups,
                                       int gpt, int renorm, const int *expert_rank,
                                       int tokens_per_rank, int R, int rpg, int mode, int *idx,
                                       float *w, int *counts, int *rank_active,
                                       const moe_layout &L, void *ws, const DeviceCtx &ctx,
                                       cudaStream_t s);
// The single-launch front end for any replica map (route_assign_layout.cu):
// shared memory it needs for these sizes, and the largest it may take.
constexpr int kFrontSmemMax = 200 * 1024;
size_t front_smem_bytes(int E, int k, int R, int rpg, int mode, int n_entries);
cudaError_t launch_route_assign_layout(const float *logits, int T, int E, int k, int n_groups, int gpt,
                                       int renorm, const int *off, const int *slots, int n_entries,
                                       const int *slot_rank, int S, int tokens_per_rank, int R,
                                       int rpg, int mode, int *idx, float *w, int *counts,
                                       int *expert_slot, int *expert_rank, int *rank_active,
                                       const moe_layout &L, void *ws, const DeviceCtx &ctx,
                                       cudaStream_t s);
cudaError_t launch_coselection(const int *idx, int T, int k, int E, int *C, const DeviceCtx &ctx,
                               cudaStream_t s);
cudaError_t launch_placement(const int *C, const int *counts, int E, int R, int *expert_rank,
                             const DeviceCtx &ctx, cudaStream_t s);
cudaError_t launch_dispatch_stats(const int *counts, int E, const int *send_counts, int R,
                                  double *stats, const DeviceCtx &ctx, cudaStream_t s);
cudaError_t launch_token_balanced(const int *counts, int E, const int *off, const int *slots,
                                  int n_entries, const int *slot_rank, int S, int R,
                                  int *slot_tokens, int *rank_active, const DeviceCtx &ctx,
                                  cudaStream_t s);
cudaError_t launch_combine(const void *y, int dtype, int H, const moe_layout &L,
                           const float *row_coef, void *out, int out_dtype, void *hop1_buf,
                           const DeviceCtx &ctx, cudaStream_t s);

}  // namespace moe
