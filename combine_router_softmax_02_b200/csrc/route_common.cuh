// Router softmax + top-k of one token by one warp (shared by the router
// kernel and the fused static-placement kernel).
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
#pragma once

#include <math.h>

#include "moe_internal.cuh"

namespace moe {
namespace route {

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

// Per-lane constants of a routing warp.
template <int EPL>  // experts per lane = ceil(E / 32)
struct Lanes {
  uint32_t valid;  // which of the lane's slots hold an expert
  int gid[EPL];    // group of each slot (read only when limited)
  bool limit;

  __device__ __forceinline__ void init(int lane, int E, int n_groups, int gpt) {
    limit = gpt > 0 && gpt < n_groups;
    const int gsize = limit ? E / n_groups : E;
    valid = 0;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      if (e < E) valid |= 1u << j;
      gid[j] = limit ? (e < E ? e / gsize : 0) : 0;
    }
  }
};

// Routes the token whose logits start at `row`.  Lanes r < k return pick r in
// (my_e, my_w); `bad` is set on lanes that saw a non-finite logit.  s_ck and
// s_ce are this warp's 32-entry shared-memory candidate buffers.
template <int EPL>
__device__ __forceinline__ void route_token(const float *row, int E, int k, int n_groups, int gpt,
                                            int renorm, const Lanes<EPL> &L, uint32_t *s_ck,
                                            int *s_ce, int lane, int &my_e, float &my_w,
                                            bool &bad) {
  float v[EPL];
  uint32_t key[EPL];
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    v[j] = (L.valid >> j & 1u) ? __ldcs(row + lane + 32 * j) : 0.0f;
    bad |= (L.valid >> j & 1u) && !isfinite(v[j]);
    key[j] = order_key(v[j]);
  }

  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < EPL; ++j)
    if (L.valid >> j & 1u) m = fmaxf(m, v[j]);
  m = warp_max(m);
  float s = 0.0f;
#pragma unroll
  for (int j = 0; j < EPL; ++j)
    if (L.valid >> j & 1u) s += expf(v[j] - m);
  s = warp_sum(s);

  uint32_t avail = L.valid;
  if (L.limit) {
    // group score = largest logit in the group; lane g holds group g's key
    uint32_t gkey = 0;
    for (int g = 0; g < n_groups; ++g) {
      uint32_t best = 0;
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        if ((L.valid >> j & 1u) && L.gid[j] == g) best = max(best, key[j]);
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
      if (!(keep >> L.gid[j] & 1u)) avail &= ~(1u << j);
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

  my_e = 0;
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
        s_ck[pos] = key[j];
        s_ce[pos] = lane + 32 * j;
        ++pos;
      }
    __syncwarp();
    uint32_t ck = lane < (int)total ? s_ck[lane] : 0u;
    const unsigned ce = lane < (int)total ? (unsigned)s_ce[lane] : 0x7fffffffu;
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
  my_w = (lane < k) ? expf(key_value(my_k) - m) / s : 0.0f;
  if (renorm) {
    const float tot = warp_sum(lane < k ? my_w : 0.0f);
    my_w = my_w / tot;
  }
}

}  // namespace route
}  // namespace moe
