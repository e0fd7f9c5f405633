// Combine: weighted sum of each token's rows back into token order.
//
// The combine after the experts ("METRO AllGather vs AllToAll for MoE decode"
// (fanout.sh), section "changes the routing information"): out[t] = sum over
// t's rows i, in ascending row order, of coef[i] * y[i], accumulated in
// float32 and rounded to nearest-even into the output dtype.
//
// Generic fan-in, one warp per output row (or column slice of it): the item's
// (<= k) source rows and coefficients go to a per-warp table, then each lane
// walks 16-byte column vectors, with the item's rows copied into shared memory
// two vectors ahead (cp.async, two stages, so the loads overlap the
// arithmetic and the store), multiply-adds them in row order and writes the
// result once.  No atomics: the result does not depend on scheduling.
// Items are tokens and lists token_rows.  The two-hop reverse has its own
// kernel below (both hops in one pass per token).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr unsigned kFull = 0xffffffffu;

struct FaninArgs {
  const uint8_t *y;
  uint32_t rb_in;           // input row bytes
  uint8_t *out;
  uint32_t rb_out;          // output row bytes
  int n_items;              // >= 0: item count; < 0: read *n_items_dev
  const int *n_items_dev;
  int cap_items;
  const int *lists;         // [items][k]
  int k;
  const float *coef;        // per source row; nullptr = 1
  int src_cap;              // rows in y
  int nvec;                 // 16-byte input vectors per row
  int slices;               // warps per item, each a column slice of the row
  int svec;                 // 16-byte input vectors per slice
};

template <typename T>
struct Elem;
template <>
struct Elem<float> {
  static constexpr int kPerVec = 4;
  __device__ static float get(const uint4 &v, int i) { return __uint_as_float((&v.x)[i]); }
};
template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kPerVec = 8;
  __device__ static float get(const uint4 &v, int i) {
    const uint32_t w = (&v.x)[i >> 1];
    return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
  }
};
template <>
struct Elem<__half> {
  static constexpr int kPerVec = 8;
  __device__ static float get(const uint4 &v, int i) {
    const uint32_t w = (&v.x)[i >> 1];
    return __half2float(__ushort_as_half((unsigned short)((i & 1) ? (w >> 16) : (w & 0xffffu))));
  }
};

template <typename T>
__device__ __forceinline__ uint32_t to_bits16(float f);
template <>
__device__ __forceinline__ uint32_t to_bits16<__nv_bfloat16>(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
template <>
__device__ __forceinline__ uint32_t to_bits16<__half>(float f) {
  return __half_as_ushort(__float2half_rn(f));
}

// Store N floats as Tout at p (N * sizeof(Tout) bytes, aligned to that size).
template <typename Tout, int N>
__device__ __forceinline__ void store_out(uint8_t *p, const float (&acc)[N]) {
  if constexpr (sizeof(Tout) == 4) {
#pragma unroll
    for (int c = 0; c < N; c += 4)
      st_v4(p + c * 4, make_uint4(__float_as_uint(acc[c]), __float_as_uint(acc[c + 1]),
                                  __float_as_uint(acc[c + 2]), __float_as_uint(acc[c + 3])));
  } else {
    uint32_t w[N / 2];
#pragma unroll
    for (int c = 0; c < N / 2; ++c)
      w[c] = to_bits16<Tout>(acc[2 * c]) | (to_bits16<Tout>(acc[2 * c + 1]) << 16);
    if constexpr (N == 8) {
      st_v4(p, make_uint4(w[0], w[1], w[2], w[3]));
    } else {
      asm volatile("st.global.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(w[0]), "r"(w[1]) : "memory");
    }
  }
}

// One source row of the warp's current item: its byte address (0 = none) and
// coefficient.  The table lives in shared memory and is re-read (volatile, a
// broadcast load) on every column vector, so the row addresses do not hold
// registers: that keeps the kernel at 3-4 resident blocks per SM, i.e. more
// loads in flight per SM.
struct SrcEntry {
  unsigned long long addr;
  float coef;
  int aux;  // two-hop: hop-1 row of the source row (-1 = none)
};

constexpr int kFaninWarps = 8;
// Few output rows (decode) are split into column slices until about this many
// warps per SM (row_slices): a sweep of 8, 12, 16, 24 and 32 on the 1024-token
// decode step put combine at 20.5, 20.5, 20.2, 22.6 and 22.5 us -- longer
// slices keep each warp's two-stage cp.async pipeline full -- while the
// 256-token step did not move.  Pack keeps 32 (it has no such pipeline).
constexpr int kSliceWarpsPerSm = 16;

__device__ __forceinline__ SrcEntry read_entry(const SrcEntry *e) {
  uint4 v;
  asm volatile("ld.volatile.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"((uint32_t)__cvta_generic_to_shared(e)));
  SrcEntry r;
  r.addr = ((unsigned long long)v.y << 32) | v.x;
  r.coef = __uint_as_float(v.z);
  r.aux = (int)v.w;
  return r;
}

// 16-byte asynchronous copy global -> shared (L2 only), and its group fences.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <typename Tin, typename Tout, int KM>
__global__ void __launch_bounds__(kFaninWarps * 32, KM <= 8 ? 3 : 1)
    fanin_kernel(FaninArgs a, DeviceCtx ctx) {
  wait_prior_grids();
  constexpr int VE = Elem<Tin>::kPerVec;
  extern __shared__ uint4 s_stage[];  // [warp][stage 2][KM][32 lanes]
  __shared__ __align__(16) SrcEntry s_tab[kFaninWarps][KM];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  SrcEntry *tab = s_tab[warp];
  uint4 *stage = s_stage + (size_t)warp * 2 * KM * 32 + lane;  // slot (st, j): stage[(st * KM + j) * 32]
  int n = a.n_items;
  if (n < 0) n = min(max(*a.n_items_dev, 0), a.cap_items);
  const int n_work = n * a.slices;  // < 2^31: slices > 1 only for few rows
  bool bounds = false;
  for (unsigned wk = blockIdx.x * kFaninWarps + warp; wk < (unsigned)n_work; wk += gridDim.x * kFaninWarps) {
    const int item = (int)(wk / (unsigned)a.slices);
    const int vbeg = (int)(wk % (unsigned)a.slices) * a.svec;
    const int vend = min(a.nvec, vbeg + a.svec);
    int my_r = -1;
    float my_c = 0.0f;
    if (lane < a.k) {
      my_r = __ldcs(a.lists + (size_t)item * a.k + lane);
      if (my_r >= a.src_cap || my_r < -1) {
        bounds = true;
        my_r = -1;
      }
      if (my_r >= 0) my_c = a.coef ? __ldg(a.coef + my_r) : 1.0f;
    }
    const unsigned vmask = __ballot_sync(kFull, my_r >= 0);
    __syncwarp();  // the previous item's readers are done
    if (lane < KM) {
      SrcEntry e;
      e.addr = my_r >= 0 ? (unsigned long long)(a.y + (size_t)my_r * a.rb_in) : 0ull;
      e.coef = my_c;
      e.aux = -1;
      tab[lane] = e;
    }
    __syncwarp();
    auto issue = [&](int v, int st) {
#pragma unroll
      for (int j = 0; j < KM; ++j)
        if (vmask >> j & 1u)
          cp_async16(stage + (st * KM + j) * 32, (const uint8_t *)read_entry(tab + j).addr + (size_t)v * 16);
      cp_async_commit();
    };
    uint8_t *orow = a.out + (size_t)item * a.rb_out;
    int st = 0;
    if (vbeg + lane < vend) issue(vbeg + lane, 0);
    for (int v = vbeg + lane; v < vend; v += 32, st ^= 1) {
      if (v + 32 < vend) {
        issue(v + 32, st ^ 1);
        cp_async_wait<1>();  // this vector's group is in
      } else {
        cp_async_wait<0>();
      }
      float acc[VE];
#pragma unroll
      for (int e = 0; e < VE; ++e) acc[e] = 0.0f;
#pragma unroll
      for (int j = 0; j < KM; ++j)
        if (vmask >> j & 1u) {
          const uint4 d = stage[(st * KM + j) * 32];
          const float c = read_entry(tab + j).coef;
#pragma unroll
          for (int e = 0; e < VE; ++e) acc[e] = fmaf(c, Elem<Tin>::get(d, e), acc[e]);
        }
      store_out<Tout, VE>(orow + (size_t)v * VE * sizeof(Tout), acc);
    }
  }
  if (bounds) set_status(ctx.status, MOE_ERR_BOUNDS);
}

// Rounds a float32 value to the activation dtype and back (the wire format).
template <typename T>
__device__ __forceinline__ float round_wire(float x);
template <>
__device__ __forceinline__ float round_wire<float>(float x) { return x; }
template <>
__device__ __forceinline__ float round_wire<__nv_bfloat16>(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}
template <>
__device__ __forceinline__ float round_wire<__half>(float x) {
  return __half2float(__float2half_rn(x));
}

struct TwoHopArgs {
  const uint8_t *y;         // hop-2 (rank) rows
  uint32_t rb_in;
  uint8_t *out;             // [T][H] of the output dtype
  uint32_t rb_out;
  uint8_t *hop1;            // group partials [rows1][H] in the input dtype, or null
  int T, k;
  const int *token_rows;    // [T][k] hop-2 rows of each token, ascending (grouped by group)
  const int *hop2_src_row;  // hop-1 row of each hop-2 row
  const float *coef;
  int cap, cap1;
  int nvec;
  int slices, svec;         // column slices per token, vectors per slice
};

// TWO_HOP reverse in one pass per token, one warp per token (or column slice):
// the token's rank rows are summed group by group in float32 (ascending rows),
// each group partial is rounded to the activation dtype (the slow-fabric wire
// format), stored to its hop-1 row when a buffer is given, and the rounded
// partials are summed in ascending group order into the token.  Bit-identical
// to running the two reverse hops one after the other, without re-reading the
// partials.
//
// The rows' column vectors go through shared memory in two stages with
// cp.async: while a lane works on vector v, its copies of vector v + 32 are in
// flight, so the loads overlap the arithmetic and the stores without holding
// registers.  Each lane reads back only the slots it copied itself, so the
// per-thread wait_group is the only fence needed.
template <typename Tin, typename Tout, int KM>
__global__ void __launch_bounds__(kFaninWarps * 32, KM <= 8 ? 3 : 1)
    two_hop_fanin_kernel(TwoHopArgs a, DeviceCtx ctx) {
  wait_prior_grids();
  constexpr int VE = Elem<Tin>::kPerVec;
  extern __shared__ uint4 s_stage[];  // [warp][stage 2][KM][32 lanes]
  __shared__ __align__(16) SrcEntry s_tab[kFaninWarps][KM];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  SrcEntry *tab = s_tab[warp];
  uint4 *stage = s_stage + (size_t)warp * 2 * KM * 32 + lane;  // slot (st, j): stage[(st * KM + j) * 32]
  bool bounds = false;
  const int n_work = a.T * a.slices;  // < 2^31: slices > 1 only for few rows
  for (unsigned wk = blockIdx.x * kFaninWarps + warp; wk < (unsigned)n_work; wk += gridDim.x * kFaninWarps) {
    const int t = (int)(wk / (unsigned)a.slices);
    const int vbeg = (int)(wk % (unsigned)a.slices) * a.svec;
    const int vend = min(a.nvec, vbeg + a.svec);
    int my_r = -1, my_s = -1;
    float my_c = 0.0f;
    if (lane < a.k) {
      my_r = __ldcs(a.token_rows + (size_t)t * a.k + lane);
      if (my_r >= a.cap || my_r < -1) {
        bounds = true;
        my_r = -1;
      }
      if (my_r >= 0) {
        my_c = __ldg(a.coef + my_r);
        my_s = __ldg(a.hop2_src_row + my_r);
        if (my_s >= a.cap1 || my_s < -1) {
          bounds = true;
          my_s = -1;
        }
      }
    }
    const unsigned vmask = __ballot_sync(kFull, my_r >= 0);
    const int next_s = __shfl_down_sync(kFull, my_s, 1);
    // a row closes its group when the next row belongs to another hop-1 row
    const bool closes = my_r >= 0 && (!(vmask >> (lane + 1) & 1u) || lane == 31 || next_s != my_s);
    const unsigned lastmask = __ballot_sync(kFull, closes);
    __syncwarp();  // the previous token's readers are done
    if (lane < KM) {
      SrcEntry e;
      e.addr = my_r >= 0 ? (unsigned long long)(a.y + (size_t)my_r * a.rb_in) : 0ull;
      e.coef = my_c;
      e.aux = my_s;
      tab[lane] = e;
    }
    __syncwarp();
    auto issue = [&](int v, int st) {
#pragma unroll
      for (int j = 0; j < KM; ++j)
        if (vmask >> j & 1u)
          cp_async16(stage + (st * KM + j) * 32, (const uint8_t *)read_entry(tab + j).addr + (size_t)v * 16);
      cp_async_commit();
    };
    uint8_t *orow = a.out + (size_t)t * a.rb_out;
    int st = 0;
    if (vbeg + lane < vend) issue(vbeg + lane, 0);
    for (int v = vbeg + lane; v < vend; v += 32, st ^= 1) {
      if (v + 32 < vend) {
        issue(v + 32, st ^ 1);
        cp_async_wait<1>();  // this vector's group is in
      } else {
        cp_async_wait<0>();
      }
      float acc_g[VE], acc_o[VE];
#pragma unroll
      for (int e = 0; e < VE; ++e) acc_g[e] = acc_o[e] = 0.0f;
#pragma unroll
      for (int j = 0; j < KM; ++j) {
        if (vmask >> j & 1u) {
          const uint4 d = stage[(st * KM + j) * 32];
          const float c = read_entry(tab + j).coef;
#pragma unroll
          for (int e = 0; e < VE; ++e) acc_g[e] = fmaf(c, Elem<Tin>::get(d, e), acc_g[e]);
        }
        if (lastmask >> j & 1u) {
#pragma unroll
          for (int e = 0; e < VE; ++e) acc_g[e] = round_wire<Tin>(acc_g[e]);
          const int src = read_entry(tab + j).aux;
          if (a.hop1 && src >= 0)
            store_out<Tin, VE>(a.hop1 + (size_t)src * a.rb_in + (size_t)v * 16, acc_g);
#pragma unroll
          for (int e = 0; e < VE; ++e) {
            acc_o[e] += acc_g[e];
            acc_g[e] = 0.0f;
          }
        }
      }
      store_out<Tout, VE>(orow + (size_t)v * VE * sizeof(Tout), acc_o);
    }
  }
  if (bounds) set_status(ctx.status, MOE_ERR_BOUNDS);
}

template <typename Tin, typename Tout, int KM>
cudaError_t launch_two_hop3(const TwoHopArgs &a, const DeviceCtx &ctx, cudaStream_t s) {
  const long blocks = ((long)a.T * a.slices + kFaninWarps - 1) / kFaninWarps;  // uncapped, as in pack
  constexpr int smem = kFaninWarps * 2 * KM * 32 * 16;  // two stages of 16-byte slots per lane and row
  static std::atomic<unsigned long long> smem_set{0};
  cudaError_t err = set_smem_limit_once(two_hop_fanin_kernel<Tin, Tout, KM>, smem, smem_set);
  if (err != cudaSuccess) return err;
  cudaError_t lerr = launch_after_prior(two_hop_fanin_kernel<Tin, Tout, KM>, dim3((unsigned)blocks),
                                        dim3(kFaninWarps * 32), (size_t)smem, s, a, ctx);
  if (lerr != cudaSuccess) return lerr;
  return count_launch(cudaGetLastError());
}

template <typename Tin, typename Tout>
cudaError_t launch_two_hop2(const TwoHopArgs &a, const DeviceCtx &ctx, cudaStream_t s) {
  if (a.k <= 2) return launch_two_hop3<Tin, Tout, 2>(a, ctx, s);
  if (a.k <= 4) return launch_two_hop3<Tin, Tout, 4>(a, ctx, s);
  if (a.k <= 8) return launch_two_hop3<Tin, Tout, 8>(a, ctx, s);
  return launch_two_hop3<Tin, Tout, 16>(a, ctx, s);
}

template <typename Tin>
cudaError_t launch_two_hop1(const TwoHopArgs &a, int out_dtype, const DeviceCtx &ctx, cudaStream_t s) {
  if (out_dtype == MOE_F16) return launch_two_hop2<Tin, __half>(a, ctx, s);
  if (out_dtype == MOE_BF16) return launch_two_hop2<Tin, __nv_bfloat16>(a, ctx, s);
  return launch_two_hop2<Tin, float>(a, ctx, s);
}

template <typename Tin, typename Tout, int KM>
cudaError_t launch3(const FaninArgs &a, const DeviceCtx &ctx, cudaStream_t s) {
  // one block per 8 items, uncapped (resident blocks read and write one
  // advancing window); a device-side item count gets a grid-stride grid
  long blocks = (a.n_items >= 0) ? ((long)a.n_items * a.slices + kFaninWarps - 1) / kFaninWarps
                                 : (long)ctx.num_sms * 8;
  if (blocks <= 0) return cudaSuccess;
  // a grid of a few waves leaves the last one part-empty: one persistent wave
  // (grid-stride) instead.  8192 tokens (2.3 waves): 87.3 -> 85.2 us; the
  // 65536-token grid (18 waves) stays uncapped (capped: 1213 -> 1312 us,
  // the resident blocks no longer advance one window together).
  constexpr long kResident = KM <= 8 ? 3 : 1;  // blocks per SM (launch bounds, shared memory)
  if (blocks > kResident * ctx.num_sms && blocks <= 4 * kResident * ctx.num_sms)
    blocks = kResident * ctx.num_sms;
  constexpr int smem = kFaninWarps * 2 * KM * 32 * 16;  // two stages of 16-byte slots per lane and row
  static std::atomic<unsigned long long> smem_set{0};
  cudaError_t err = set_smem_limit_once(fanin_kernel<Tin, Tout, KM>, smem, smem_set);
  if (err != cudaSuccess) return err;
  cudaError_t lerr = launch_after_prior(fanin_kernel<Tin, Tout, KM>, dim3((unsigned)blocks),
                                        dim3(kFaninWarps * 32), (size_t)smem, s, a, ctx);
  if (lerr != cudaSuccess) return lerr;
  return count_launch(cudaGetLastError());
}

template <typename Tin, typename Tout>
cudaError_t launch2(const FaninArgs &a, const DeviceCtx &ctx, cudaStream_t s) {
  if (a.k <= 2) return launch3<Tin, Tout, 2>(a, ctx, s);
  if (a.k <= 4) return launch3<Tin, Tout, 4>(a, ctx, s);
  if (a.k <= 8) return launch3<Tin, Tout, 8>(a, ctx, s);
  return launch3<Tin, Tout, 16>(a, ctx, s);
}

template <typename Tin>
cudaError_t launch1(const FaninArgs &a, int out_dtype, const DeviceCtx &ctx, cudaStream_t s) {
  if (out_dtype == MOE_F16) return launch2<Tin, __half>(a, ctx, s);
  if (out_dtype == MOE_BF16) return launch2<Tin, __nv_bfloat16>(a, ctx, s);
  return launch2<Tin, float>(a, ctx, s);
}

cudaError_t launch_fanin(const FaninArgs &a, int in_dtype, int out_dtype, const DeviceCtx &ctx,
                         cudaStream_t s) {
  if (a.n_items == 0) return cudaSuccess;
  if (in_dtype == MOE_F16) return launch1<__half>(a, out_dtype, ctx, s);
  if (in_dtype == MOE_BF16) return launch1<__nv_bfloat16>(a, out_dtype, ctx, s);
  return launch1<float>(a, out_dtype, ctx, s);
}

int elem_size(int dt) { return dt == MOE_F32 ? 4 : 2; }

}  // namespace

cudaError_t launch_combine(const void *y, int dtype, int H, const moe_layout &L,
                           const float *row_coef, void *out, int out_dtype, void *hop1_buf,
                           const DeviceCtx &ctx, cudaStream_t s) {
  const float *coef = row_coef ? row_coef : L.row_coef;
  FaninArgs a;
  a.k = L.k;
  a.n_items_dev = nullptr;
  a.cap_items = 0;
  if (L.mode != MOE_LAYOUT_TWO_HOP) {
    a.y = static_cast<const uint8_t *>(y);
    a.rb_in = (uint32_t)((size_t)H * elem_size(dtype));
    a.out = static_cast<uint8_t *>(out);
    a.rb_out = (uint32_t)((size_t)H * elem_size(out_dtype));
    a.n_items = L.T;
    a.lists = L.token_rows;
    a.coef = coef;
    a.src_cap = L.capacity;
    a.nvec = (int)(a.rb_in / 16);
    row_slices(a.n_items, a.nvec, ctx.num_sms, a.slices, a.svec, kSliceWarpsPerSm);
    // One to four rows per resident warp: each warp takes whole rows in turns,
    // so the last turn runs part-empty (8192 rows over 3552 warps: 3 turns for
    // 2.3 rows' work).  Half rows halve that loss: 84.5 -> 82.0 us on the
    // 8192-token training workload (thirds: 83.8).
    const long warps = (a.k <= 8 ? 3L : 1L) * kFaninWarps * ctx.num_sms;  // resident (launch3)
    if (a.slices == 1 && a.n_items > warps && a.n_items <= 4 * warps) {
      a.svec = ((a.nvec + 1) / 2 + 31) / 32 * 32;
      a.slices = (a.nvec + a.svec - 1) / a.svec;
    }
    return launch_fanin(a, dtype, out_dtype, ctx, s);
  }
  // both reverse hops in one pass per token
  TwoHopArgs b;
  b.y = static_cast<const uint8_t *>(y);
  b.rb_in = (uint32_t)((size_t)H * elem_size(dtype));
  b.out = static_cast<uint8_t *>(out);
  b.rb_out = (uint32_t)((size_t)H * elem_size(out_dtype));
  b.hop1 = static_cast<uint8_t *>(hop1_buf);
  b.T = L.T;
  b.k = L.k;
  b.token_rows = L.token_rows;
  b.hop2_src_row = L.hop2_src_row;
  b.coef = coef;
  b.cap = L.capacity;
  b.cap1 = L.capacity_hop1;
  b.nvec = (int)(b.rb_in / 16);
  if (b.T == 0) return cudaSuccess;
  row_slices(b.T, b.nvec, ctx.num_sms, b.slices, b.svec, kSliceWarpsPerSm);
  if (dtype == MOE_F16) return launch_two_hop1<__half>(b, out_dtype, ctx, s);
  if (dtype == MOE_BF16) return launch_two_hop1<__nv_bfloat16>(b, out_dtype, ctx, s);
  return launch_two_hop1<float>(b, out_dtype, ctx, s);
}

}  // namespace moe
