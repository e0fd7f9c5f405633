// Router softmax + top-k, one warp per token.
//
// "METRO AllGather vs AllToAll for MoE decode" (fanout.sh), section "changes
// the routing information": every rank computes the top-k expert choices of
// the whole gathered token set.  Group-limited routing follows the TerraceMoE
// editorial (lyndhub), section "The core problem".
//
// Lane l holds experts l, l+32, l+64, ... of its token (coalesced 128-byte
// loads).  Softmax max and sum are butterfly reductions, so every lane ends
// with bit-identical values.  Selection works on an order-preserving u32 key
// of each logit.  The k-th largest of the 32 lane maxima is a lower bound on
// the k-th largest key, so only the few elements at or above it can be picked;
// they are compacted one per lane through shared memory and k rounds of two
// redux.sync instructions pick the winners: the largest key, and among equal
// keys the smallest expert id (ties to the lower index).  When more than 32
// elements tie at the bound, every element is scanned each round instead.
// The gate weights are computed at the end, one pick per lane.
#include <math.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr unsigned kFull = 0xffffffffu;

// Monotone map float -> uint32 (larger float, larger key); -0 and +0 map to
// the same key so they tie like the floats compare.  Finite values never map
// to 0, which marks "no candidate".
__device__ __forceinline__ uint32_t order_key(float v) {
  uint32_t u = (v == 0.0f) ? 0u : __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inverse of order_key (a zero key comes back as +0).
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, d));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(kFull, v, d);
  return v;
}

template <int EPL>  // experts per lane = ceil(E / 32)
__global__ void __launch_bounds__(256) route_topk_kernel(const float *__restrict__ logits, int T,
                                                         int E, int k, int n_groups, int gpt,
                                                         int renorm, int *__restrict__ idx_out,
                                                         float *__restrict__ w_out, DeviceCtx ctx) {
  __shared__ uint32_t s_ck[8][32];  // per-warp candidate keys
  __shared__ int s_ce[8][32];       // and their experts
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int wpb = blockDim.x >> 5;
  const bool limit = gpt > 0 && gpt < n_groups;
  const int gsize = limit ? E / n_groups : E;

  uint32_t valid = 0;   // which of the lane's slots hold an expert
  int gid[EPL];         // group of each slot (only read when limited)
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = lane + 32 * j;
    if (e < E) valid |= 1u << j;
    gid[j] = limit ? (e < E ? e / gsize : 0) : 0;
  }

  for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += gridDim.x * wpb) {
    const float *row = logits + (size_t)t * E;
    float v[EPL];
    uint32_t key[EPL];
    bool bad = false;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      v[j] = (valid >> j & 1u) ? __ldcs(row + lane + 32 * j) : 0.0f;
      bad |= (valid >> j & 1u) && !isfinite(v[j]);
      key[j] = order_key(v[j]);
    }
    if (__any_sync(kFull, bad) && lane == 0) set_status(ctx.status, MOE_ERR_BAD_INPUT);

    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (valid >> j & 1u) m = fmaxf(m, v[j]);
    m = warp_max(m);
    float s = 0.0f;
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (valid >> j & 1u) s += expf(v[j] - m);
    s = warp_sum(s);

    uint32_t avail = valid;
    if (limit) {
      // group score = largest logit in the group; lane g holds group g's key
      uint32_t gkey = 0;
      for (int g = 0; g < n_groups; ++g) {
        uint32_t best = 0;
#pragma unroll
        for (int j = 0; j < EPL; ++j)
          if ((valid >> j & 1u) && gid[j] == g) best = max(best, key[j]);
        best = __reduce_max_sync(kFull, best);
        if (lane == g) gkey = best;
      }
      uint32_t keep = 0;
      for (int r = 0; r < gpt; ++r) {
        const uint32_t kmax = __reduce_max_sync(kFull, gkey);
        const int g = (int)__reduce_min_sync(kFull, (gkey == kmax && kmax != 0) ? (unsigned)lane : 32u);
        keep |= 1u << g;
        if (lane == g) gkey = 0;
      }
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        if (!(keep >> gid[j] & 1u)) avail &= ~(1u << j);
    }

#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (!(avail >> j & 1u)) key[j] = 0;  // 0 = not a candidate

    // Candidates.  tau = the k-th largest of the 32 lane maxima: k distinct
    // elements reach it, so every top-k element has key >= tau.
    uint32_t lm = 0;
#pragma unroll
    for (int j = 0; j < EPL; ++j) lm = max(lm, key[j]);
    uint32_t tau = 0;
    for (int r = 0; r < k; ++r) {
      tau = __reduce_max_sync(kFull, lm);
      const unsigned lw = __reduce_min_sync(kFull, lm == tau ? (unsigned)lane : 32u);
      if (lane == (int)lw) lm = 0;
    }
    int cnt = 0;
#pragma unroll
    for (int j = 0; j < EPL; ++j) cnt += (key[j] >= tau) ? 1 : 0;
    const unsigned total = __reduce_add_sync(kFull, (unsigned)cnt);

    int my_e = 0;
    uint32_t my_k = 0;
    if (total <= 32) {
      // one candidate per lane, through shared memory, then k rounds of
      // (largest key, then smallest expert id among equal keys)
      int pos = cnt;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int n = __shfl_up_sync(kFull, pos, d);
        if (lane >= d) pos += n;
      }
      pos -= cnt;
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        if (key[j] >= tau) {
          s_ck[warp][pos] = key[j];
          s_ce[warp][pos] = lane + 32 * j;
          ++pos;
        }
      __syncwarp();
      uint32_t ck = lane < (int)total ? s_ck[warp][lane] : 0u;
      const unsigned ce = lane < (int)total ? (unsigned)s_ce[warp][lane] : 0x7fffffffu;
      __syncwarp();
      for (int r = 0; r < k; ++r) {
        const uint32_t kmax = __reduce_max_sync(kFull, ck);
        const unsigned ewin = __reduce_min_sync(kFull, ck == kmax ? ce : 0x7fffffffu);
        if (ce == ewin) ck = 0;
        if (lane == r) {
          my_e = (int)ewin;
          my_k = kmax;
        }
      }
    } else {
      // many ties at tau: scan every element each round
      for (int r = 0; r < k; ++r) {
        uint32_t bk = 0;
        int be = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < EPL; ++j)
          if (key[j] > bk) {  // strict: the lowest slot wins ties
            bk = key[j];
            be = lane + 32 * j;
          }
        const uint32_t kmax = __reduce_max_sync(kFull, bk);
        const int ewin = (int)__reduce_min_sync(kFull, (bk == kmax) ? (unsigned)be : 0x7fffffffu);
        if (lane == (ewin & 31)) {
#pragma unroll
          for (int j = 0; j < EPL; ++j)
            if (j == (ewin >> 5)) key[j] = 0;
        }
        if (lane == r) {
          my_e = ewin;
          my_k = kmax;
        }
      }
    }
    // gate weights, one per lane: softmax probability of the pick
    float my_w = (lane < k) ? expf(key_value(my_k) - m) / s : 0.0f;
    if (renorm) {
      const float tot = warp_sum(lane < k ? my_w : 0.0f);
      my_w = my_w / tot;
    }
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
  route_topk_kernel<EPL><<<(unsigned)blocks, wpb * 32, 0, s>>>(logits, T, E, k, n_groups, gpt,
                                                               renorm, idx, w, ctx);
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
