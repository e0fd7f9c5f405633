// C ABI of libmoe.so: argument checks, the per-device status word, launches.
// The operations and their sources are documented in include/moe.h.
#include <atomic>
#include <mutex>

#include "moe_internal.cuh"

namespace moe {
std::atomic<unsigned long long> g_kernel_launches{0};
}

namespace {

__device__ int g_status;      // first device-side error since the last moe_get_status
__device__ int g_status_out;  // where the exchange kernel leaves the old value

__global__ void status_exchange_kernel(int *status, int *out) { *out = atomicExch(status, 0); }

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultWaitNs = 1000000000ull;  // one second

struct PerDevice {
  std::atomic<int *> status{nullptr};
  int *status_out = nullptr;
  int num_sms = 0;
  int smem_per_sm = 0;
};
PerDevice g_dev[kMaxDevices];
std::mutex g_init_mu;
std::atomic<uint64_t> g_wait_limit_ns{kDefaultWaitNs};
std::atomic<int> g_silent_tile{-1};

int get_ctx(moe::DeviceCtx *ctx) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  PerDevice &d = g_dev[dev];
  int *st = d.status.load(std::memory_order_acquire);
  if (!st) {
    std::lock_guard<std::mutex> lk(g_init_mu);
    st = d.status.load(std::memory_order_relaxed);
    if (!st) {
      void *p = nullptr, *q = nullptr;
      int sms = 0, smem = 0;
      if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return MOE_ERR_CUDA;
      if (cudaGetSymbolAddress(&q, g_status_out) != cudaSuccess) return MOE_ERR_CUDA;
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return MOE_ERR_CUDA;
      if (cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess)
        return MOE_ERR_CUDA;
      d.status_out = static_cast<int *>(q);
      d.num_sms = sms;
      d.smem_per_sm = smem;
      st = static_cast<int *>(p);
      d.status.store(st, std::memory_order_release);
    }
  }
  ctx->status = st;
  ctx->num_sms = d.num_sms;
  ctx->smem_per_sm = d.smem_per_sm;
  ctx->wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  ctx->silent_tile = g_silent_tile.load(std::memory_order_relaxed);
  return MOE_OK;
}

inline int launched(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int elem_bytes(int dt) { return dt == MOE_F32 ? 4 : 2; }
inline bool valid_dtype(int dt) { return dt == MOE_F16 || dt == MOE_BF16 || dt == MOE_F32; }

bool valid_ekr(int E, int k) {
  return E >= 1 && E <= moe::kMaxE && k >= 1 && k <= moe::kMaxK && k <= E;
}

}  // namespace

extern "C" {

uint64_t moe_kernel_launches(void) { return moe::g_kernel_launches.load(); }

const char *moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_BOUNDS: return "MOE_ERR_BOUNDS";
    case MOE_ERR_BAD_INPUT: return "MOE_ERR_BAD_INPUT";
    case MOE_ERR_CAPACITY: return "MOE_ERR_CAPACITY";
    default: return "MOE_ERR_UNKNOWN";
  }
}

int moe_debug_set_wait(uint64_t wait_limit_ns, int32_t layout_silent_tile) {
  if (layout_silent_tile < -1) return MOE_ERR_INVALID_ARG;
  g_wait_limit_ns.store(wait_limit_ns ? wait_limit_ns : kDefaultWaitNs);
  g_silent_tile.store(layout_silent_tile);
  return MOE_OK;
}

int moe_get_status(moe_stream_t stream) {
  moe::DeviceCtx ctx;
  int rc = get_ctx(&ctx);
  if (rc) return rc;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  status_exchange_kernel<<<1, 1, 0, s>>>(ctx.status, g_dev[dev].status_out);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  int host = 0;
  if (cudaMemcpyAsync(&host, g_dev[dev].status_out, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  return host;
}

int moe_route_topk(const float *logits, int32_t T, int32_t E, int32_t k, int32_t n_groups,
                   int32_t groups_per_token, int32_t renormalize, int32_t *topk_idx,
                   float *topk_w, moe_stream_t stream) {
  if (T < 0 || !valid_ekr(E, k)) return MOE_ERR_INVALID_ARG;
  if ((int64_t)T * k >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
  if (T > 0 && (!logits || !topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
  if (renormalize != 0 && renormalize != 1) return MOE_ERR_INVALID_ARG;
  if (n_groups != 0 || groups_per_token != 0) {
    if (n_groups < 1 || n_groups > moe::kMaxGroups || E % n_groups != 0) return MOE_ERR_INVALID_ARG;
    if (groups_per_token < 1 || groups_per_token > n_groups) return MOE_ERR_INVALID_ARG;
    if ((int64_t)groups_per_token * (E / n_groups) < k) return MOE_ERR_INVALID_ARG;
  }
  moe::DeviceCtx ctx;
  int rc = get_ctx(&ctx);
  if (rc) return rc;
  return launched(moe::launch_route_topk(logits, T, E, k, n_groups, groups_per_token, renormalize,
                                         topk_idx, topk_w, ctx, reinterpret_cast<cudaStream_t>(stream)));
}

int moe_demand_hist(const int32_t *topk_idx, int32_t T, int32_t k, int32_t E, int32_t *counts,
                    moe_stream_t stream) {
  if (T < 0 || !valid_ekr(E, k) || !counts || (T > 0 && !topk_idx)) return MOE_ERR_INVALID_ARG;
  if ((int64_t)T * k >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
  moe::DeviceCtx ctx;
  int rc = get_ctx(&ctx);
  if (rc) return rc;
  return launched(moe::launch_demand_hist(topk_idx, T, k, E, counts, ctx,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

int moe_replica_assign(const int32_t *counts, int32_t E, const int32_t *replica_offsets,
                       const int32_t *replica_slots, int32_t n_replica_entries,
                       const int32_t *slot_rank, int32_t S, int32_t R, int32_t *expert_slot,
                       int32_t *expert_rank, int32_t *rank_active, moe_stream_t stream) {
  if (E < 1 || E > moe::kMaxE || R < 1 || R > moe::kMaxR) return MOE_ERR_INVALID_ARG;
  if (S < 1 || S > moe::kMaxSlots || n_replica_entries < 0 || n_replica_entries > moe::kMaxSlots)
    return MOE_ERR_INVALID_ARG;
  if (!counts || !replica_offsets || !slot_rank || !expert_slot || !expert_rank || !rank_active)
    return MOE_ERR_INVALID_ARG;
  if (n_replica_entries > 0 && !replica_slots) return MOE_ERR_INVALID_ARG;
  moe::DeviceCtx ctx;
  int rc = get_ctx(&ctx);
  if (rc) return rc;
  return launched(moe::launch_replica_assign(counts, E, replica_offsets, replica_slots,
                                             n_replica_entries, slot_rank, S, R, expert_slot,
                                             expert_rank, rank_active, ctx,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_layout_workspace_size(int32_t T, int32_t k, int32_t E, int32_t R,
                                 int32_t ranks_per_group, int32_t mode) {
  if (T < 0 || !valid_ekr(E, k) || R < 1 || R > moe::kMaxR) return 0;
  if (mode < MOE_LAYOUT_PER_PICK || mode > MOE_LAYOUT_TWO_HOP) return 0;
  if (mode == MOE_LAYOUT_TWO_HOP && (ranks_per_group < 1 || R % ranks_per_group != 0)) return 0;
  return moe::layout_workspace_bytes(T, k, E, R, ranks_per_group, mode);
}

int moe_build_layout(const int32_t *topk_idx, const float *topk_w, const int32_t *expert_rank,
                     int32_t T, int32_t tokens_per_rank, int32_t k, int32_t E, int32_t R,
                     int32_t ranks_per_group, int32_t mode, moe_layout *layout, void *workspace,
                     size_t workspace_bytes, moe_stream_t stream) {
  if (!layout || T < 0 || !valid_ekr(E, k) || R < 1 || R > moe::kMaxR) return MOE_ERR_INVALID_ARG;
  if (mode < MOE_LAYOUT_PER_PICK || mode > MOE_LAYOUT_TWO_HOP) return MOE_ERR_INVALID_ARG;
  if ((int64_t)T * k >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
  if (tokens_per_rank < 1 || (int64_t)tokens_per_rank * R < T) return MOE_ERR_INVALID_ARG;
  if (mode == MOE_LAYOUT_TWO_HOP && (ranks_per_group < 1 || ranks_per_group > R || R % ranks_per_group))
    return MOE_ERR_INVALID_ARG;
  moe_layout &L = *layout;
  if (!L.rank_offsets || !L.send_counts || !L.num_rows || L.capacity < 0) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_idx || !topk_w || !expert_rank || !L.token_rows)) return MOE_ERR_INVALID_ARG;
  if (L.capacity > 0 && (!L.row_token || !L.row_coef)) return MOE_ERR_INVALID_ARG;
  if (mode == MOE_LAYOUT_TWO_HOP) {
    if (!L.group_offsets || !L.num_rows_hop1 || L.capacity_hop1 < 0) return MOE_ERR_INVALID_ARG;
    if (T > 0 && !L.token_groups) return MOE_ERR_INVALID_ARG;
    if (L.capacity > 0 && !L.hop2_src_row) return MOE_ERR_INVALID_ARG;
    if (L.capacity_hop1 > 0 && (!L.hop1_row_token || !L.hop1_children)) return MOE_ERR_INVALID_ARG;
  }
  const size_t need = moe::layout_workspace_bytes(T, k, E, R, ranks_per_group, mode);
  if (T > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return MOE_ERR_INVALID_ARG;
  moe::DeviceCtx ctx;
  int rc = get_ctx(&ctx);
  if (rc) return rc;
  L.T = T;
  L.k = k;
  L.R = R;
  L.E = E;
  L.ranks_per_group = (mode == MOE_LAYOUT_TWO_HOP) ? ranks_per_group : 1;
  L.mode = mode;
  return launched(moe::launch_build_layout(topk_idx, topk_w, expert_rank, T, tokens_per_rank, k, E,
                                           R, ranks_per_group, mode, L, workspace, ctx,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

static int check_layout_shape(const moe_layout *L) {
  if (!L) return MOE_ERR_INVALID_ARG;
  if (L->T < 0 || !valid_ekr(L->E, L->k) || L->R < 1 || L->R > moe::kMaxR) return MOE_ERR_INVALID_ARG;
  if (L->mode < MOE_LAYOUT_PER_PICK || L->mode > MOE_LAYOUT_TWO_HOP) return MOE_ERR_INVALID_ARG;
  if (L->T > 0 && !L->token_rows) return MOE_ERR_INVALID_ARG;
  if (L->mode == MOE_LAYOUT_TWO_HOP && (L->T > 0 && !L->token_groups)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

int moe_pack(const void *x, int32_t dtype, int32_t H, const moe_layout *layout, void *packed,
             void *packed_hop1, moe_stream_t stream) {
  int rc = check_layout_shape(layout);
  if (rc) return rc;
  if (!valid_dtype(dtype) || H < 1) return MOE_ERR_INVALID_ARG;
  const size_t rb = (size_t)H * elem_bytes(dtype);
  if (rb % 16 != 0) return MOE_ERR_UNSUPPORTED;
  if (rb > ((size_t)1 << 30)) return MOE_ERR_UNSUPPORTED;
  if (layout->T > 0 && (!x || !aligned16(x))) return MOE_ERR_INVALID_ARG;
  if (layout->capacity > 0 && (!packed || !aligned16(packed))) return MOE_ERR_INVALID_ARG;
  if (layout->mode == MOE_LAYOUT_TWO_HOP && layout->capacity_hop1 > 0 &&
      (!packed_hop1 || !aligned16(packed_hop1)))
    return MOE_ERR_INVALID_ARG;
  moe::DeviceCtx ctx;
  rc = get_ctx(&ctx);
  if (rc) return rc;
  return launched(moe::launch_pack(x, elem_bytes(dtype), H, *layout, packed, packed_hop1, ctx,
                                   reinterpret_cast<cudaStream_t>(stream)));
}

int moe_combine(const void *y, int32_t dtype, int32_t H, const moe_layout *layout,
                const float *row_coef, void *out, int32_t out_dtype, void *hop1_buf,
                moe_stream_t stream) {
  int rc = check_layout_shape(layout);
  if (rc) return rc;
  if (!valid_dtype(dtype) || !valid_dtype(out_dtype) || H < 1) return MOE_ERR_INVALID_ARG;
  if (((size_t)H * elem_bytes(dtype)) % 16 != 0) return MOE_ERR_UNSUPPORTED;
  if (layout->T > 0 && (!out || !aligned16(out))) return MOE_ERR_INVALID_ARG;
  if (layout->capacity > 0 && (!y || !aligned16(y))) return MOE_ERR_INVALID_ARG;
  if (!row_coef && layout->capacity > 0 && !layout->row_coef) return MOE_ERR_INVALID_ARG;
  if (layout->mode == MOE_LAYOUT_TWO_HOP) {
    if (hop1_buf && !aligned16(hop1_buf)) return MOE_ERR_INVALID_ARG;
    if (layout->capacity > 0 && !layout->hop2_src_row) return MOE_ERR_INVALID_ARG;
  }
  moe::DeviceCtx ctx;
  rc = get_ctx(&ctx);
  if (rc) return rc;
  return launched(moe::launch_combine(y, dtype, H, *layout, row_coef, out, out_dtype, hop1_buf, ctx,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

extern "C" {

int moe_dispatch_stats(const int32_t *counts, int32_t E, const int32_t *send_counts, int32_t R,
                       double *stats, moe_stream_t stream) {
  if (E < 1 || E > moe::kMaxE || R < 1 || R > moe::kMaxR) return MOE_ERR_INVALID_ARG;
  if (!counts || !send_counts || !stats) return MOE_ERR_INVALID_ARG;
  moe::DeviceCtx ctx;
  int rc = get_ctx(&ctx);
  if (rc) return rc;
  return launched(moe::launch_dispatch_stats(counts, E, send_counts, R, stats, ctx,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

int moe_token_balanced_assign(const int32_t *counts, int32_t E, const int32_t *replica_offsets,
                              const int32_t *replica_slots, int32_t n_replica_entries,
                              const int32_t *slot_rank, int32_t S, int32_t R, int32_t *slot_tokens,
                              int32_t *rank_active, moe_stream_t stream) {
  if (E < 1 || E > moe::kMaxE || R < 1 || R > moe::kMaxR) return MOE_ERR_INVALID_ARG;
  if (S < 1 || S > moe::kMaxSlots || n_replica_entries < 0 || n_replica_entries > moe::kMaxSlots)
    return MOE_ERR_INVALID_ARG;
  if (!counts || !replica_offsets || !slot_rank || !slot_tokens || !rank_active) return MOE_ERR_INVALID_ARG;
  if (n_replica_entries > 0 && !replica_slots) return MOE_ERR_INVALID_ARG;
  moe::DeviceCtx ctx;
  int rc = get_ctx(&ctx);
  if (rc) return rc;
  return launched(moe::launch_token_balanced(counts, E, replica_offsets, replica_slots,
                                             n_replica_entries, slot_rank, S, R, slot_tokens,
                                             rank_active, ctx, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// The checks of moe_route_topk and moe_build_layout for the fused front ends
// (launch-free).
int check_front(const float *logits, int32_t T, int32_t E, int32_t k, int32_t n_groups,
                int32_t groups_per_token, int32_t renormalize, int32_t tokens_per_rank, int32_t R,
                int32_t ranks_per_group, int32_t mode, const int32_t *topk_idx, const float *topk_w,
                const int32_t *counts, const moe_layout *layout, const void *workspace,
                size_t workspace_bytes) {
  if (!layout || T < 0 || !valid_ekr(E, k) || R < 1 || R > moe::kMaxR) return MOE_ERR_INVALID_ARG;
  if ((int64_t)T * k >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
  if (!counts) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!logits || !topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
  if (renormalize != 0 && renormalize != 1) return MOE_ERR_INVALID_ARG;
  if (n_groups != 0 || groups_per_token != 0) {
    if (n_groups < 1 || n_groups > moe::kMaxGroups || E % n_groups != 0) return MOE_ERR_INVALID_ARG;
    if (groups_per_token < 1 || groups_per_token > n_groups) return MOE_ERR_INVALID_ARG;
    if ((int64_t)groups_per_token * (E / n_groups) < k) return MOE_ERR_INVALID_ARG;
  }
  if (mode < MOE_LAYOUT_PER_PICK || mode > MOE_LAYOUT_TWO_HOP) return MOE_ERR_INVALID_ARG;
  if (tokens_per_rank < 1 || (int64_t)tokens_per_rank * R < T) return MOE_ERR_INVALID_ARG;
  if (mode == MOE_LAYOUT_TWO_HOP && (ranks_per_group < 1 || ranks_per_group > R || R % ranks_per_group))
    return MOE_ERR_INVALID_ARG;
  const moe_layout &L = *layout;
  if (!L.rank_offsets || !L.send_counts || !L.num_rows || L.capacity < 0) return MOE_ERR_INVALID_ARG;
  if (T > 0 && !L.token_rows) return MOE_ERR_INVALID_ARG;
  if (L.capacity > 0 && (!L.row_token || !L.row_coef)) return MOE_ERR_INVALID_ARG;
  if (mode == MOE_LAYOUT_TWO_HOP) {
    if (!L.group_offsets || !L.num_rows_hop1 || L.capacity_hop1 < 0) return MOE_ERR_INVALID_ARG;
    if (T > 0 && !L.token_groups) return MOE_ERR_INVALID_ARG;
    if (L.capacity > 0 && !L.hop2_src_row) return MOE_ERR_INVALID_ARG;
    if (L.capacity_hop1 > 0 && (!L.hop1_row_token || !L.hop1_children)) return MOE_ERR_INVALID_ARG;
  }
  const size_t need = moe::layout_workspace_bytes(T, k, E, R, ranks_per_group, mode);
  if (T > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

void fill_layout_shape(moe_layout &L, int32_t T, int32_t k, int32_t E, int32_t R,
                       int32_t ranks_per_group, int32_t mode) {
  L.T = T;
  L.k = k;
  L.R = R;
  L.E = E;
  L.ranks_per_group = (mode == MOE_LAYOUT_TWO_HOP) ? ranks_per_group : 1;
  L.mode = mode;
}

}  // namespace

extern "C" int moe_route_layout_single_replica(
    const float *logits, int32_t T, int32_t E, int32_t k, int32_t n_groups,
    int32_t groups_per_token, int32_t renormalize, const int32_t *expert_rank,
    int32_t tokens_per_rank, int32_t R, int32_t ranks_per_group, int32_t mode, int32_t *topk_idx,
    float *topk_w, int32_t *counts, int32_t *rank_active, moe_layout *layout, void *workspace,
    size_t workspace_bytes, moe_stream_t stream) {
  int rc = check_front(logits, T, E, k, n_groups, groups_per_token, renormalize, tokens_per_rank, R,
                       ranks_per_group, mode, topk_idx, topk_w, counts, layout, workspace,
                       workspace_bytes);
  if (rc) return rc;
  if (!expert_rank) return MOE_ERR_INVALID_ARG;
  moe::DeviceCtx ctx;
  rc = get_ctx(&ctx);
  if (rc) return rc;
  moe_layout &L = *layout;
  fill_layout_shape(L, T, k, E, R, ranks_per_group, mode);
  return launched(moe::launch_route_layout_static(
      logits, T, E, k, n_groups, groups_per_token, renormalize, expert_rank, tokens_per_rank, R,
      ranks_per_group, mode, topk_idx, topk_w, counts, rank_active, L, workspace, ctx,
      reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" int moe_route_assign_layout(
    const float *logits, int32_t T, int32_t E, int32_t k, int32_t n_groups, int32_t groups_per_token,
    int32_t renormalize, const int32_t *replica_offsets, const int32_t *replica_slots,
    int32_t n_replica_entries, const int32_t *slot_rank, int32_t S, int32_t tokens_per_rank, int32_t R,
    int32_t ranks_per_group, int32_t mode, int32_t *topk_idx, float *topk_w, int32_t *counts,
    int32_t *expert_slot, int32_t *expert_rank, int32_t *rank_active, moe_layout *layout,
    void *workspace, size_t workspace_bytes, moe_stream_t stream) {
  int rc = check_front(logits, T, E, k, n_groups, groups_per_token, renormalize, tokens_per_rank, R,
                       ranks_per_group, mode, topk_idx, topk_w, counts, layout, workspace,
                       workspace_bytes);
  if (rc) return rc;
  // the checks of moe_replica_assign
  if (S < 1 || S > moe::kMaxSlots || n_replica_entries < 0 || n_replica_entries > moe::kMaxSlots)
    return MOE_ERR_INVALID_ARG;
  if (!replica_offsets || !slot_rank || !expert_slot || !expert_rank || !rank_active)
    return MOE_ERR_INVALID_ARG;
  if (n_replica_entries > 0 && !replica_slots) return MOE_ERR_INVALID_ARG;
  if (moe::front_smem_bytes(E, k, R, ranks_per_group, mode, n_replica_entries) > (size_t)moe::kFrontSmemMax)
    return MOE_ERR_UNSUPPORTED;
  moe::DeviceCtx ctx;
  rc = get_ctx(&ctx);
  if (rc) return rc;
  moe_layout &L = *layout;
  fill_layout_shape(L, T, k, E, R, ranks_per_group, mode);
  return launched(moe::launch_route_assign_layout(
      logits, T, E, k, n_groups, groups_per_token, renormalize, replica_offsets, replica_slots,
      n_replica_entries, slot_rank, S, tokens_per_rank, R, ranks_per_group, mode, topk_idx, topk_w,
      counts, expert_slot, expert_rank, rank_active, L, workspace, ctx,
      reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" {

int moe_coselection_hist(const int32_t *topk_idx, int32_t T, int32_t k, int32_t E, int32_t *cosel,
                         moe_stream_t stream) {
  if (T < 0 || !valid_ekr(E, k) || !cosel || (T > 0 && !topk_idx)) return MOE_ERR_INVALID_ARG;
  if ((int64_t)T * k >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
  moe::DeviceCtx ctx;
  int rc = get_ctx(&ctx);
  if (rc) return rc;
  return launched(moe::launch_coselection(topk_idx, T, k, E, cosel, ctx,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

int moe_correlated_placement(const int32_t *cosel, const int32_t *counts, int32_t E, int32_t R,
                             int32_t *expert_rank, moe_stream_t stream) {
  if (E < 1 || E > moe::kMaxE || R < 1 || R > moe::kMaxR || E % R != 0) return MOE_ERR_INVALID_ARG;
  if (!cosel || !counts || !expert_rank) return MOE_ERR_INVALID_ARG;
  moe::DeviceCtx ctx;
  int rc = get_ctx(&ctx);
  if (rc) return rc;
  return launched(moe::launch_placement(cosel, counts, E, R, expert_rank, ctx,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
