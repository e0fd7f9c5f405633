// Router softmax + top-k of one token by one warp (shared by the router
// kernel and the fused static-placement kernel).
//
// "METRO AllGather vs AllToAll for MoE decode" (fanout.sh), section "changes
// the routing information": every rank computes the top-k expert choices of
// the whole gathered token set.  Group-limited routing follows the TerraceMoE
// editorial (lyndhub), section "The core problem".
//
// Lane l holds experts l, l+32, l+64, ... of its token (coalesced 128-byte
// loads).  Each lane's largest logit becomes an order-preserving u32 key, so
// the softmax maximum is one integer warp reduction; the softmax sum is a
// butterfly reduction, so every lane ends with bit-identical values.
//
// Selection: the k-th largest of the 32 lane maxima (tau) is a lower bound on
// the k-th largest key, so only the few elements at or above it can be picked.
// They are compacted through shared memory in ascending expert order (one
// ballot per slot), and each candidate counts the candidates that beat it --
// a larger key, or an equal key at a lower position, i.e. a lower expert id
// (ties go to the lower index).  That count is its rank; the candidates of rank
// < k are scattered so lane r holds pick r.  When more than 32 elements tie at
// the bound, every element is scanned in each of k rounds instead.  The gate
// weights are computed at the end, one pick per lane.
#pragma once

#include <math.h>

#include "moe_internal.cuh"

namespace moe {
namespace route {

constexpr unsigned kFull = 0xffffffffu;

// Monotone map float -> uint32 (larger float, larger key): negative values
// have all bits flipped, the others their sign bit set.  Adding +0 first turns
// -0 into +0, so the two zeros tie like the floats compare.  Finite values map
// into [0x00800000, 0xff800000); -inf, +inf and NaNs land outside that range.
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t u = __float_as_uint(v + 0.0f);
  return u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
}

// Inverse of order_key (a zero key comes back as +0).
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// e^x computed as 2^(x log2 e) with exp2f (documented within 2 ulp): a
// multiply and the exponent unit instead of expf's range reduction.  The
// product's rounding adds |x| units of roundoff to the relative error.
constexpr float kLog2e = 1.44269504088896341f;
__device__ __forceinline__ float exp_via_exp2(float x) { return exp2f(x * kLog2e); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(kFull, v, d);
  return v;
}

// Per-lane constants of a routing warp.  FULL: E == 32 * EPL, every slot
// holds an expert.
template <int EPL, bool FULL>
struct Lanes {
  uint32_t valid;  // which of the lane's slots hold an expert
  bool limit;      // group-limited routing
  int gsize;       // experts per group
  uint32_t magic;  // e / gsize == umulhi(e, magic) for e < 2^16, gsize >= 2

  __device__ __forceinline__ void init(int lane, int E, int n_groups, int gpt) {
    limit = gpt > 0 && gpt < n_groups;
    gsize = limit ? E / n_groups : E;
    magic = gsize >= 2 ? 0xffffffffu / (uint32_t)gsize + 1u : 0u;
    valid = 0;
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (lane + 32 * j < E) valid |= 1u << j;
  }
  __device__ __forceinline__ bool ok(int j) const { return FULL || (valid >> j & 1u); }
  __device__ __forceinline__ int group(int e) const {
    return gsize >= 2 ? (int)__umulhi((uint32_t)e, magic) : e;
  }
};

// Routes the token whose logits start at `row`.  Lanes r < k return pick r in
// (my_e, my_w); `bad` is set on lanes that saw a non-finite logit.  s_cv and
// s_ce are this warp's 32-entry shared-memory candidate buffers (s_cv
// 16-byte aligned).
template <int EPL, bool FULL>
__device__ __forceinline__ void route_token(const float *row, int E, int k, int n_groups, int gpt,
                                            int renorm, const Lanes<EPL, FULL> &L, float *s_cv,
                                            int *s_ce, int lane, int &my_e, float &my_w,
                                            bool &bad) {
  constexpr float kNoCand = -INFINITY;  // an empty slot, or an expert ruled out by its group
  float v[EPL];
#pragma unroll
  for (int j = 0; j < EPL; ++j) v[j] = L.ok(j) ? __ldcs(row + lane + 32 * j) : kNoCand;
  // x * 0 is +-0 for finite x and NaN for an infinity or a NaN
  float z = 0.0f, lmf = kNoCand;
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    if (L.ok(j)) z = fmaf(v[j], 0.0f, z);
    lmf = fmaxf(lmf, v[j]);
  }
  bad |= !(z == 0.0f);

  // softmax maximum and sum over all experts; only the lane maxima need keys
  uint32_t lm = lmf == kNoCand ? 0u : order_key(lmf);  // this lane's largest selectable key
  const uint32_t top = __reduce_max_sync(kFull, lm);
  const float m = key_value(top);
  float s = 0.0f;
#pragma unroll
  for (int j = 0; j < EPL; ++j)
    if (L.ok(j)) s += exp_via_exp2(v[j] - m);
  s = warp_sum(s);

  bool fresh = true;  // lm is still the lane maximum (then the warp max is `top`)
  if (L.limit) {
    // group score = largest logit in the group; lane g holds group g's key
    uint32_t gkey = 0;
    for (int g = 0; g < n_groups; ++g) {
      float bf = kNoCand;
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        if (L.ok(j) && L.group(lane + 32 * j) == g) bf = fmaxf(bf, v[j]);
      const uint32_t best = __reduce_max_sync(kFull, bf == kNoCand ? 0u : order_key(bf));
      if (lane == g) gkey = best;
    }
    uint32_t keep = 0;
    for (int r = 0; r < gpt; ++r) {
      const uint32_t gm = __reduce_max_sync(kFull, gkey);
      const unsigned b = __ballot_sync(kFull, gkey == gm && gm != 0);
      const int g = b ? __ffs(b) - 1 : 0;
      keep |= 1u << g;
      if (lane == g) gkey = 0;
    }
    lmf = kNoCand;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      if (!(keep >> L.group(lane + 32 * j) & 1u)) v[j] = kNoCand;
      lmf = fmaxf(lmf, v[j]);
    }
    lm = lmf == kNoCand ? 0u : order_key(lmf);
    fresh = false;
  }

  // Candidates.  tau = the k-th largest of the 32 lane maxima: k distinct
  // elements reach it, so every top-k element has a logit >= tau (tau == 0:
  // fewer than k lanes hold a selectable expert; every slot is a candidate).
  uint32_t tau = 0;
  for (int r = 0; r < k; ++r) {
    tau = (r == 0 && fresh) ? top : __reduce_max_sync(kFull, lm);
    const unsigned b = __ballot_sync(kFull, lm == tau);
    if (lane == 31 - __clz(b)) lm = 0;  // any one lane holding the value
  }
  const float tau_v = key_value(tau);

  // compaction in ascending expert order: slot j of lane l is expert l + 32 j
  const unsigned below = lanemask_lt();
  unsigned total = 0;
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const bool c = L.ok(j) && (tau == 0u || v[j] >= tau_v);
    const unsigned b = __ballot_sync(kFull, c);
    const unsigned pos = total + __popc(b & below);
    if (c && pos < 32) {
      s_cv[pos] = v[j];
      s_ce[pos] = lane + 32 * j;
    }
    total += __popc(b);
  }

  my_e = 0;
  float my_v = 0.0f;
  if (total <= 32) {
    // -inf pads the candidates to a multiple of 4: a pad beats no candidate
    if (lane >= (int)total && lane < (int)((total + 3) & ~3u)) s_cv[lane] = kNoCand;
    __syncwarp();
    const float cv = lane < (int)total ? s_cv[lane] : 0.0f;
    const int ce = lane < (int)total ? s_ce[lane] : 0;
    // rank = candidates with a larger logit, or an equal one at a lower
    // position (a lower expert id); -0 and +0 compare equal
    int rank = 0;
    for (int j = 0; j < (int)total; j += 4) {
      const float4 q = *reinterpret_cast<const float4 *>(s_cv + j);  // broadcast
      rank += (q.x > cv || (q.x == cv && j < lane)) ? 1 : 0;
      rank += (q.y > cv || (q.y == cv && j + 1 < lane)) ? 1 : 0;
      rank += (q.z > cv || (q.z == cv && j + 2 < lane)) ? 1 : 0;
      rank += (q.w > cv || (q.w == cv && j + 3 < lane)) ? 1 : 0;
    }
    __syncwarp();
    if (lane < (int)total && rank < k) {
      s_cv[rank] = cv;
      s_ce[rank] = ce;
    }
    __syncwarp();
    if (lane < k) {
      my_v = s_cv[lane];
      my_e = s_ce[lane];
    }
    __syncwarp();
  } else {
    // many ties at tau: scan every element each round
    for (int r = 0; r < k; ++r) {
      float bf = kNoCand;
      int be = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        if (v[j] > bf) {  // strict: the lowest slot wins ties
          bf = v[j];
          be = lane + 32 * j;
        }
      const uint32_t bk = be != 0x7fffffff ? order_key(bf) : 0u;
      const uint32_t kmx = __reduce_max_sync(kFull, bk);
      const int ewin = (int)__reduce_min_sync(kFull, (bk == kmx) ? (unsigned)be : 0x7fffffffu);
      if (lane == (ewin & 31)) {
#pragma unroll
        for (int j = 0; j < EPL; ++j)
          if (j == (ewin >> 5)) v[j] = kNoCand;
      }
      if (lane == r) {
        my_e = ewin;
        my_v = key_value(kmx);
      }
    }
  }
  // gate weights, one per lane: softmax probability of the pick
  my_w = (lane < k) ? exp_via_exp2(my_v - m) / s : 0.0f;
  if (renorm) {
    const float tot = warp_sum(lane < k ? my_w : 0.0f);
    my_w = my_w / tot;
  }
}

}  // namespace route
}  // namespace moe
