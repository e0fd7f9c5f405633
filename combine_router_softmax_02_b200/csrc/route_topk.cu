// Router softmax + top-k kernel: one warp per token (see route_common.cuh).
#include "route_common.cuh"

namespace moe {
namespace {

template <int EPL, bool FULL>
__global__ void __launch_bounds__(256) route_topk_kernel(const float *__restrict__ logits, int T,
                                                         int E, int k, int n_groups, int gpt,
                                                         int renorm, int *__restrict__ idx_out,
                                                         float *__restrict__ w_out, DeviceCtx ctx) {
  wait_prior_grids();
  __shared__ __align__(16) float s_cv[8][32];  // per-warp candidate logits
  __shared__ int s_ce[8][32];       // and their experts
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int wpb = blockDim.x >> 5;
  route::Lanes<EPL, FULL> L;
  L.init(lane, E, n_groups, gpt);
  for (int t = blockIdx.x * wpb + warp; t < T; t += gridDim.x * wpb) {
    int my_e;
    float my_w;
    bool bad = false;
    route::route_token<EPL, FULL>(logits + (size_t)t * E, E, k, n_groups, gpt, renorm, L, s_cv[warp],
                            s_ce[warp], lane, my_e, my_w, bad);
    if (__any_sync(route::kFull, bad) && lane == 0) set_status(ctx.status, MOE_ERR_BAD_INPUT);
    if (lane < k) {
      idx_out[(size_t)t * k + lane] = my_e;
      w_out[(size_t)t * k + lane] = my_w;
    }
  }
}

template <int EPL>
cudaError_t launch_epl(const float *logits, int T, int E, int k, int n_groups, int gpt, int renorm,
                       int *idx, float *w, const DeviceCtx &ctx, cudaStream_t s) {
  const int wpb = 8;
  long blocks = (T + wpb - 1) / wpb;
  const long cap = (long)ctx.num_sms * 16;
  if (blocks > cap) blocks = cap;
  auto kern = E == 32 * EPL ? route_topk_kernel<EPL, true> : route_topk_kernel<EPL, false>;
  cudaError_t err = launch_after_prior(kern, dim3((unsigned)blocks), dim3(wpb * 32), 0, s, logits, T, E, k,
                                       n_groups, gpt, renorm, idx, w, ctx);
  if (err != cudaSuccess) return err;
  return count_launch(cudaGetLastError());
}

}  // namespace

cudaError_t launch_route_topk(const float *logits, int T, int E, int k, int n_groups, int gpt,
                              int renorm, int *idx, float *w, const DeviceCtx &ctx,
                              cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int epl = (E + 31) / 32;
  if (epl <= 1) return launch_epl<1>(logits, T, E, k, n_groups, gpt, renorm, idx, w, ctx, s);
  if (epl <= 2) return launch_epl<2>(logits, T, E, k, n_groups, gpt, renorm, idx, w, ctx, s);
  if (epl <= 4) return launch_epl<4>(logits, T, E, k, n_groups, gpt, renorm, idx, w, ctx, s);
  if (epl <= 8) return launch_epl<8>(logits, T, E, k, n_groups, gpt, renorm, idx, w, ctx, s);
  if (epl <= 16) return launch_epl<16>(logits, T, E, k, n_groups, gpt, renorm, idx, w, ctx, s);
  return launch_epl<32>(logits, T, E, k, n_groups, gpt, renorm, idx, w, ctx, s);
}

}  // namespace moe
