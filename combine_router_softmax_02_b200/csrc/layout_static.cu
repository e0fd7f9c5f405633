// moe_build_layout_static: the layout entry point for callers that cannot
// allocate device memory.  Its scratch lives in a file-scope device array of
// a fixed size instead of a caller-supplied workspace.  See include/moe.h.
#include <mutex>

#include "moe_internal.cuh"

namespace {

// The scratch every call shares.  Each GPU that loads the library holds it
// until the process exits.
static __device__ __align__(256) unsigned char g_layout_scratch[MOE_LAYOUT_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_layout_scratch on the current device.  In host code the
// array's name is only a stand-in, so the address comes from the runtime,
// once per device, with that device current.  The lookup is not a stream
// operation and may load the module, so it is refused while `stream` is being
// captured: the first call on a device must come before any capture.
int scratch_address(cudaStream_t stream, void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return MOE_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return MOE_ERR_UNSUPPORTED;
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_layout_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" int moe_build_layout_static(const int32_t *topk_idx, const float *topk_w,
                                       const int32_t *expert_rank, int32_t T,
                                       int32_t tokens_per_rank, int32_t k, int32_t E, int32_t R,
                                       int32_t ranks_per_group, int32_t mode, moe_layout *layout,
                                       moe_stream_t stream) {
  const size_t need = moe_layout_workspace_size(T, k, E, R, ranks_per_group, mode);
  if (need == 0 && T > 0) return MOE_ERR_INVALID_ARG;
  if (need > MOE_LAYOUT_STATIC_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  const int rc = scratch_address(reinterpret_cast<cudaStream_t>(stream), &scratch);
  if (rc != MOE_OK) return rc;
  // Same checks and kernels as moe_build_layout; the launch clears the parts
  // of the scratch that must start at zero.
  return moe_build_layout(topk_idx, topk_w, expert_rank, T, tokens_per_rank, k, E, R,
                          ranks_per_group, mode, layout, scratch, MOE_LAYOUT_STATIC_SCRATCH_BYTES,
                          stream);
}
