// Router softmax + top-k kernels.
//
// The general kernel gives each token a warp (route_common.cuh).  Its warp
// collectives (the maximum, the butterfly sum, the k rounds for the candidate
// bound, the compaction ballots) cost about 600 warp instructions a token, so
// on a large token set it runs at the issue limit, far below the memory bound.
// For the common shapes (E = 64, 128 or 256 experts, k <= 8, no group limit
// or groups of whole sixteenths of the experts) a second kernel gives each
// token a thread instead: a warp streams 32 tokens' logit rows through shared
// memory and every lane routes its own token with plain per-thread
// arithmetic, well under half the instructions.  Its results are
// bit-identical to the warp kernel's: the same maximum, the softmax sum added
// in the same order (lane l's running sum over experts l, l + 32, ... and the
// butterfly's pairing of the 32 partial sums, reproduced in registers), the
// same exact top-k order (larger logit first, the lower expert id on ties)
// and the same weight formula.
#include "route_common.cuh"

namespace moe {
namespace {

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
               "l"(gmem)
               : "memory");
}

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

// ------------------------------------------------- one thread per token ----
constexpr int kRowTokens = 32;  // tokens per block (one warp)

// The sum of a[0..31] in the order of a 32-lane butterfly (lane l adds lane
// l ^ d for d = 16, 8, 4, 2, 1; every lane ends with lane 0's value, which is
// this): the warp kernel's softmax sum, bit for bit.
__device__ __forceinline__ float butterfly_sum(float (&a)[32]) {
#pragma unroll
  for (int d = 16; d > 0; d >>= 1)
#pragma unroll
    for (int l = 0; l < d; ++l) a[l] = a[l] + a[l + d];
  return a[0];
}

// One stage of a bitonic sort of 16 values into descending order: pairs
// (i, i + D) inside blocks of SIZE, descending where i & SIZE is clear.
template <int SIZE, int D>
__device__ __forceinline__ void bitonic_stage(float (&x)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i)
    if (!(i & D)) {
      const float hi = fmaxf(x[i], x[i | D]), lo = fminf(x[i], x[i | D]);
      const bool desc = !(i & SIZE) || SIZE == 16;
      x[i] = desc ? hi : lo;
      x[i | D] = desc ? lo : hi;
    }
}

// Routes the T tokens, 32 to a block (one warp).  The block streams its
// tokens' logits through shared memory in 32-expert columns (32 tokens x 32
// experts, 4 KB), three columns in flight (cp.async), the row stride padded to
// 36 floats so that the eight 16-byte reads a quarter-warp makes at the same
// column of eight rows fall in distinct banks; the small tiles leave room for
// many resident warps.  The columns go by twice (the second time mostly from
// L2), and lane l routes token t0 + l:
//   1. first pass: the non-finite check, the maximum m and the maxima of 16
//      chunks of E/16 experts.  Under a group limit (groups of whole chunks)
//      a group's score is the largest of its chunks' maxima, and the token keeps
//      its best groups_per_token groups (gpt rounds of a scan in chunk order,
//      ties to the lower group); tau = the k-th largest maximum of the kept
//      chunks (a sorting network) bounds the k-th largest kept logit from below
//      (k kept chunks hold an element >= tau; -inf when fewer than k are kept);
//   2. second pass: expert e adds e^(v - m) to partial sum e % 32 (the warp
//      kernel's lane e % 32; the softmax is over every expert) and, when it is
//      kept and v >= tau, is a candidate; each column's
//      candidates go, in ascending expert order, through an insertion network
//      that keeps the k best order keys: a candidate goes in before the first
//      entry with a strictly smaller key and every entry after it shifts down
//      one, so equal keys stay in ascending expert order and the last of them
//      is the one dropped;
//   3. the weights of the picks from m and the butterfly-ordered sum (a pick's
//      logit comes back from its order key; only a -0 turns into +0, which
//      gives the same e^(v - m)).
constexpr int kColStride = 36;  // floats per token row of a column tile
constexpr int kColTiles = 3;    // column tiles in flight

template <int E, int KM>
__global__ void __launch_bounds__(kRowTokens, 16) route_rows_kernel(const float *__restrict__ logits, int T,
                                                                int k, int n_groups, int gpt, int renorm,
                                                                int *__restrict__ idx_out,
                                                                float *__restrict__ w_out, DeviceCtx ctx) {
  static_assert(E % 32 == 0 && E <= 256 && KM <= 8, "the per-thread router's shapes");
  constexpr int NC = E / 32;    // columns
  constexpr int NCH = 16;       // chunks of the bound
  constexpr int CH = E / NCH;   // experts per chunk
  constexpr int CPC = 32 / CH;  // chunks per column
  __shared__ __align__(16) float s_col[kColTiles][kRowTokens * kColStride];
  wait_prior_grids();
  const int lane = threadIdx.x;
  const long t0 = (long)blockIdx.x * kRowTokens;
  const int nt = (int)min((long)kRowTokens, (long)T - t0);
  const float *src = logits + t0 * E;
  // column step % NC of the tile (the first pass, then the second) into tile step % kColTiles
  auto load = [&](int step) {
    const int col = step % NC;
    float *dst = s_col[step % kColTiles];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = u * 32 + lane, r = i >> 3, c = i & 7;
      if (r < nt) cp_async16(dst + r * kColStride + c * 4, src + (size_t)r * E + col * 32 + c * 4);
    }
  };
#pragma unroll
  for (int st = 0; st < kColTiles - 1; ++st) {
    load(st);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }

  float z = 0.0f, cm[NCH], m = 0.0f, tau = 0.0f;
  uint32_t keep = (1u << NCH) - 1;  // chunks kept by the group limit
#pragma unroll
  for (int c = 0; c < NCH; ++c) cm[c] = -INFINITY;
  float acc[32];
#pragma unroll
  for (int l = 0; l < 32; ++l) acc[l] = 0.0f;
  uint32_t key[KM];
  int ex[KM];
#pragma unroll
  for (int i = 0; i < KM; ++i) {
    key[i] = 0u;  // below every logit's key
    ex[i] = 0;
  }
#pragma unroll 1
  for (int step = 0; step < 2 * NC; ++step) {
    if (step + kColTiles - 1 < 2 * NC) load(step + kColTiles - 1);
    asm volatile("cp.async.commit_group;" ::: "memory");  // possibly empty: one group per step
    asm volatile("cp.async.wait_group %0;" ::"n"(kColTiles - 1) : "memory");
    __syncwarp();
    const float *tile = s_col[step % kColTiles] + lane * kColStride;
    const float4 *tile4 = reinterpret_cast<const float4 *>(tile);
    if (step < NC) {
      // 1: non-finite check and the chunk maxima of this column
      float cmax[CPC];
#pragma unroll
      for (int j = 0; j < CPC; ++j) cmax[j] = -INFINITY;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 x = tile4[q];
        z = fmaf(x.x, 0.0f, z);
        z = fmaf(x.y, 0.0f, z);
        z = fmaf(x.z, 0.0f, z);
        z = fmaf(x.w, 0.0f, z);
        cmax[4 * q / CH] = fmaxf(cmax[4 * q / CH], fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w)));
      }
#pragma unroll
      for (int i = 0; i < NCH; ++i) cm[i] = (i / CPC == step) ? cmax[i % CPC] : cm[i];
      if (step == NC - 1) {
        if (lane < nt && !(z == 0.0f)) set_status(ctx.status, MOE_ERR_BAD_INPUT);
        float mx = cm[0];
#pragma unroll
        for (int c = 1; c < NCH; ++c) mx = fmaxf(mx, cm[c]);
        // the warp kernel's maximum: the largest order key of the lane
        // maxima, a lane whose maximum is -inf counting as key 0
        m = route::key_value(mx == -INFINITY ? 0u : route::order_key(mx));
        if (gpt > 0 && gpt < n_groups) {  // n_groups divides 16: groups of whole chunks
          const int cpg = NCH / n_groups;
          float gm[NCH];  // each chunk's group score
#pragma unroll
          for (int i = 0; i < NCH; ++i) gm[i] = cm[i];
#pragma unroll
          for (int ld = 0; ld < 4; ++ld) {  // NCH = 2^4
            const int d = 1 << ld;
            if (d < cpg)
#pragma unroll
              for (int i = 0; i < NCH; ++i)
                if (!(i & d)) {
                  const float g2 = fmaxf(gm[i], gm[i | d]);
                  gm[i] = g2;
                  gm[i | d] = g2;
                }
          }
          keep = 0;
#pragma unroll 1
          for (int r = 0; r < gpt; ++r) {  // the best group left; ties to the lower one
            float best = -INFINITY;
            int bi = -1;
#pragma unroll
            for (int i = 0; i < NCH; ++i) {
              const bool take = !(keep >> i & 1u) && (bi < 0 || gm[i] > best);
              best = take ? gm[i] : best;
              bi = take ? i : bi;
            }
            keep |= ((1u << cpg) - 1u) << (bi & ~(cpg - 1));
          }
        }
        // tau: the k-th largest kept chunk maximum (bitonic sort, descending)
        float x[NCH];
#pragma unroll
        for (int i = 0; i < NCH; ++i) x[i] = (keep >> i & 1u) ? cm[i] : -INFINITY;
        bitonic_stage<2, 1>(x);
        bitonic_stage<4, 2>(x);
        bitonic_stage<4, 1>(x);
        bitonic_stage<8, 4>(x);
        bitonic_stage<8, 2>(x);
        bitonic_stage<8, 1>(x);
        bitonic_stage<16, 8>(x);
        bitonic_stage<16, 4>(x);
        bitonic_stage<16, 2>(x);
        bitonic_stage<16, 1>(x);
        tau = x[0];  // x[k - 1], as the minimum of the first k (no indexed read)
#pragma unroll
        for (int r = 1; r < KM; ++r) tau = r < k ? fminf(tau, x[r]) : tau;
      }
    } else {
      // 2: partial sums in lane order, candidates through the insertion network
      const int col = step - NC;
      uint32_t colkeep = 0;  // this column's experts in kept chunks
#pragma unroll
      for (int c = 0; c < CPC; ++c)
        colkeep |= ((keep >> (col * CPC + c)) & 1u) ? ((1u << CH) - 1u) << (c * CH) : 0u;
      uint32_t cand = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 x = tile4[q];
        acc[4 * q + 0] += route::exp_via_exp2(x.x - m);
        acc[4 * q + 1] += route::exp_via_exp2(x.y - m);
        acc[4 * q + 2] += route::exp_via_exp2(x.z - m);
        acc[4 * q + 3] += route::exp_via_exp2(x.w - m);
        cand |= (x.x >= tau ? 1u : 0u) << (4 * q) | (x.y >= tau ? 2u : 0u) << (4 * q) |
                (x.z >= tau ? 4u : 0u) << (4 * q) | (x.w >= tau ? 8u : 0u) << (4 * q);
      }
      cand &= colkeep;
      while (cand) {
        const int l = __ffs(cand) - 1;
        cand &= cand - 1;
        uint32_t kc = route::order_key(tile[l]);
        int ec = col * 32 + l;
        bool moved = false;  // after the first move every later entry shifts down one
#pragma unroll
        for (int i = 0; i < KM; ++i) {
          const bool up = moved || kc > key[i];
          moved = up;
          const uint32_t kt = key[i];
          const int et = ex[i];
          key[i] = up ? kc : kt;
          ex[i] = up ? ec : et;
          kc = up ? kt : kc;
          ec = up ? et : ec;
        }
      }
    }
    __syncwarp();  // the tile is read before a later step's copy reuses it
  }
  if (lane >= nt) return;
  const float s = butterfly_sum(acc);

  // 3: gate weights (renormalised over the picks in the butterfly's order)
  float w[KM];
#pragma unroll
  for (int r = 0; r < KM; ++r) w[r] = r < k ? route::exp_via_exp2(route::key_value(key[r]) - m) / s : 0.0f;
  if (renorm) {
    float p[32];
#pragma unroll
    for (int l = 0; l < 32; ++l) p[l] = l < KM ? w[l < KM ? l : 0] : 0.0f;
    const float tot = butterfly_sum(p);
#pragma unroll
    for (int r = 0; r < KM; ++r) w[r] = w[r] / tot;
  }
  const size_t o = (size_t)(t0 + lane) * k;
#pragma unroll
  for (int r = 0; r < KM; ++r)
    if (r < k) {
      idx_out[o + r] = ex[r];
      w_out[o + r] = w[r];
    }
}

// The per-thread router when it applies: E = 64, 128 or 256, k <= 8, no group
// limit or groups of whole chunks (n_groups dividing 16), 16-byte aligned
// logits, and tokens for at least 4 warps on every SM (18944 on 148 SMs).
// With fewer, too few warps share an SM to hide each other's latency: on the
// 8192-token training workload (E = 64, under 2 warps per SM) an earlier
// version took 11.4 us against the warp kernel's 10.7.  On the 32768-token
// two-hop workload (E = 128, 8 groups, 7 warps per SM) it takes 23.0 us against
// 31.8, on the 65536-token prefill workload (E = 256) 36.0 against 47.4.
constexpr int kRowMinWarpsPerSm = 4;

template <int E>
cudaError_t launch_rows(const float *logits, int T, int k, int n_groups, int gpt, int renorm, int *idx,
                        float *w, const DeviceCtx &ctx, cudaStream_t s) {
  const long blocks = ((long)T + kRowTokens - 1) / kRowTokens;
  cudaError_t err = launch_after_prior(route_rows_kernel<E, 8>, dim3((unsigned)blocks), dim3(kRowTokens), 0,
                                       s, logits, T, k, n_groups, gpt, renorm, idx, w, ctx);
  if (err != cudaSuccess) return err;
  return count_launch(cudaGetLastError());
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
  const bool limit = gpt > 0 && gpt < n_groups;
  if ((long)T >= (long)kRowMinWarpsPerSm * kRowTokens * ctx.num_sms && k <= 8 &&
      (!limit || 16 % n_groups == 0) && ((uintptr_t)logits & 15u) == 0) {
    if (E == 64) return launch_rows<64>(logits, T, k, n_groups, gpt, renorm, idx, w, ctx, s);
    if (E == 128) return launch_rows<128>(logits, T, k, n_groups, gpt, renorm, idx, w, ctx, s);
    if (E == 256) return launch_rows<256>(logits, T, k, n_groups, gpt, renorm, idx, w, ctx, s);
  }
  const int epl = (E + 31) / 32;
  if (epl <= 1) return launch_epl<1>(logits, T, E, k, n_groups, gpt, renorm, idx, w, ctx, s);
  if (epl <= 2) return launch_epl<2>(logits, T, E, k, n_groups, gpt, renorm, idx, w, ctx, s);
  if (epl <= 4) return launch_epl<4>(logits, T, E, k, n_groups, gpt, renorm, idx, w, ctx, s);
  if (epl <= 8) return launch_epl<8>(logits, T, E, k, n_groups, gpt, renorm, idx, w, ctx, s);
  if (epl <= 16) return launch_epl<16>(logits, T, E, k, n_groups, gpt, renorm, idx, w, ctx, s);
  return launch_epl<32>(logits, T, E, k, n_groups, gpt, renorm, idx, w, ctx, s);
}

}  // namespace moe
