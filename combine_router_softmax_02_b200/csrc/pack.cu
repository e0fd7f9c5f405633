// Pack: token rows into contiguous per-destination send buffers.
//
// The local half of the AllToAll dispatch ("METRO AllGather vs AllToAll for
// MoE decode" (fanout.sh), section "Work the 8-GPU payload example": AllToAll
// splits each rank's input into per-destination chunks).
//
// Generic fan-out: token t's row (src + t * rb) is copied to every row listed
// in its destination lists (-1 padded): token_rows for the one-hop layouts;
// token_groups (into the hop-1 buffer) and token_rows (into the hop-2 buffer)
// for TWO_HOP, whose two hops thus run from one read of the token -- the
// forwarded hop-2 rows are bit-identical to the group rows they come from.
// Each source row is read from HBM once and each destination row written
// once: the algorithmic minimum (tokens + rows) * rb bytes.
//
// One warp per CTA, one CTA per SM.  Lane 0 drives 1-D TMA bulk copies (no
// tensor map, no multicast): the row goes global -> shared on an mbarrier,
// then one bulk shared -> global store per destination, one bulk group per
// item.  S shared-memory stages; loads run D items ahead; a stage is reloaded
// once the stores of the item that used it have finished reading it
// (cp.async.bulk.wait_group.read).  The other lanes prefetch the destination
// lists of the next 32 items.
#include "moe_internal.cuh"

// Launch shape: CTAs per SM, and loads in flight as a fraction D/S of the stages.
#ifndef MOE_PACK_CTAS_PER_SM
#define MOE_PACK_CTAS_PER_SM 1
#endif
#ifndef MOE_PACK_D_NUM
#define MOE_PACK_D_NUM 1
#endif
#ifndef MOE_PACK_D_DEN
#define MOE_PACK_D_DEN 2
#endif
#ifndef MOE_PACK_STORE_EVICT_FIRST
#define MOE_PACK_STORE_EVICT_FIRST 1
#endif

namespace moe {
namespace {

constexpr unsigned kFull = 0xffffffffu;

struct FanoutArgs {
  const uint8_t *src;       // item i's source row: src + i * rb
  uint32_t rb;              // row bytes, multiple of 16
  int n_items;
  int k;
  // up to two destination lists per item: lists[l][i * k + j] is a row of dst[l]
  const int *lists[2];
  uint8_t *dst[2];
  int dst_cap[2];           // rows in dst[l]
};

template <int KM, int NL>
__device__ __forceinline__ void load_lists(const FanoutArgs &a, int item, int i_end, int (&r)[NL * KM]) {
#pragma unroll
  for (int l = 0; l < NL; ++l)
#pragma unroll
    for (int j = 0; j < KM; ++j)
      r[l * KM + j] = (item < i_end && j < a.k) ? __ldcs(a.lists[l] + (size_t)item * a.k + j) : -1;
}

template <int S, int D, int KM, int NL>
__global__ void __launch_bounds__(32, 1) fanout_kernel(FanoutArgs a, DeviceCtx ctx) {
  static_assert(D >= 1 && D < S, "pipeline depth");
  constexpr int W = NL * KM;  // destination slots per item
  extern __shared__ __align__(128) uint8_t stages[];
  __shared__ __align__(8) uint64_t bars[S];
  __shared__ int s_list[2][32][W];
  const int lane = threadIdx.x;

  const int n = a.n_items;
  const int per = (n + gridDim.x - 1) / gridDim.x;
  const int i0 = blockIdx.x * per;
  const int i1 = min(n, i0 + per);
  const int nq = i1 - i0;
  if (nq <= 0) return;

  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < S; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  {
    int r[W];
    load_lists<KM, NL>(a, i0 + lane, i1, r);
#pragma unroll
    for (int j = 0; j < W; ++j) s_list[0][lane][j] = r[j];
  }
  __syncwarp();
  int pre[W];
  load_lists<KM, NL>(a, i0 + 32 + lane, i1, pre);

  const uint64_t pol_ld = policy_evict_first();
  const uint64_t pol_st = MOE_PACK_STORE_EVICT_FIRST ? policy_evict_first() : policy_evict_normal();
  if (lane == 0) {
    for (int q = 0; q < D && q < nq; ++q) {
      mbar_arrive_expect_tx(&bars[q % S], a.rb);
      bulk_g2s(stages + (size_t)(q % S) * a.rb, a.src + (size_t)(i0 + q) * a.rb, a.rb, &bars[q % S], pol_ld);
    }
  }

  bool bounds = false;
  int aborted = 0;
  int issued = min(D, nq);  // loads issued so far
  for (int q = 0; q < nq; ++q) {
    const int qi = q & 31, buf = (q >> 5) & 1;
    if (lane == 0) {
      if (q + D < nq) {
        // stage (q+D)%S was last used by item q+D-S, whose store group is
        // followed by S-D-1 newer groups
        bulk_wait_read<S - D - 1>();
        const int s2 = (q + D) % S;
        mbar_arrive_expect_tx(&bars[s2], a.rb);
        bulk_g2s(stages + (size_t)s2 * a.rb, a.src + (size_t)(i0 + q + D) * a.rb, a.rb, &bars[s2], pol_ld);
        ++issued;
      }
      const int s = q % S;
      if (mbar_wait_bounded(&bars[s], (uint32_t)((q / S) & 1), ctx.wait_limit_ns)) {
        fence_proxy_async_smem();
        const uint8_t *row = stages + (size_t)s * a.rb;
#pragma unroll
        for (int j = 0; j < W; ++j) {
          const int l = j / KM;
          const int r = s_list[buf][qi][j];
          if (r >= 0) {
            if (r < a.dst_cap[l])
              bulk_s2g(a.dst[l] + (size_t)r * a.rb, row, a.rb, pol_st);
            else
              bounds = true;
          } else if (r < -1) {
            bounds = true;
          }
        }
        bulk_commit();
      } else {
        // a load never landed: drain the ones still in flight, then stop
        set_status(ctx.status, MOE_ERR_TIMEOUT);
        for (int q2 = q + 1; q2 < issued; ++q2)
          (void)mbar_wait_bounded(&bars[q2 % S], (uint32_t)((q2 / S) & 1), ctx.wait_limit_ns);
        aborted = 1;
      }
    }
    if (__shfl_sync(kFull, aborted, 0)) break;
    if (qi == 31) {
      __syncwarp();
#pragma unroll
      for (int j = 0; j < W; ++j) s_list[buf ^ 1][lane][j] = pre[j];
      __syncwarp();
      load_lists<KM, NL>(a, i0 + q + 33 + lane, i1, pre);
    }
  }
  if (lane == 0) bulk_wait_all();
  if (bounds) set_status(ctx.status, MOE_ERR_BOUNDS);
}

// bytes of shared memory for stages, per CTA
constexpr size_t kStageBudget = 200 * 1024 / MOE_PACK_CTAS_PER_SM;

template <int S, int KM, int NL>
cudaError_t launch_sk(const FanoutArgs &a, int grid, cudaStream_t s, const DeviceCtx &ctx) {
  constexpr int D0 = S * MOE_PACK_D_NUM / MOE_PACK_D_DEN;
  constexpr int D = D0 < 1 ? 1 : (D0 >= S ? S - 1 : D0);
  auto kern = fanout_kernel<S, D, KM, NL>;
  const size_t smem = (size_t)S * a.rb;  // <= kStageBudget by the choice of S
  static std::atomic<unsigned long long> done{0};
  cudaError_t err = set_smem_limit_once(kern, (int)kStageBudget, done);
  if (err != cudaSuccess) return err;
  kern<<<grid, 32, smem, s>>>(a, ctx);
  return count_launch(cudaGetLastError());
}

template <int KM, int NL>
cudaError_t launch_km(const FanoutArgs &a, int grid, cudaStream_t s, const DeviceCtx &ctx) {
  const size_t fit = kStageBudget / a.rb;
  if (fit >= 24) return launch_sk<24, KM, NL>(a, grid, s, ctx);
  if (fit >= 16) return launch_sk<16, KM, NL>(a, grid, s, ctx);
  if (fit >= 12) return launch_sk<12, KM, NL>(a, grid, s, ctx);
  if (fit >= 8) return launch_sk<8, KM, NL>(a, grid, s, ctx);
  if (fit >= 6) return launch_sk<6, KM, NL>(a, grid, s, ctx);
  return launch_sk<4, KM, NL>(a, grid, s, ctx);
}

template <int NL>
cudaError_t launch_nl(const FanoutArgs &a, int grid, const DeviceCtx &ctx, cudaStream_t s) {
  if (a.k <= 2) return launch_km<2, NL>(a, grid, s, ctx);
  if (a.k <= 4) return launch_km<4, NL>(a, grid, s, ctx);
  if (a.k <= 8) return launch_km<8, NL>(a, grid, s, ctx);
  return launch_km<16, NL>(a, grid, s, ctx);
}

cudaError_t launch_fanout(const FanoutArgs &a, const DeviceCtx &ctx, cudaStream_t s) {
  if (a.n_items <= 0) return cudaSuccess;
  const int grid = min(ctx.num_sms * MOE_PACK_CTAS_PER_SM, a.n_items);
  return a.lists[1] ? launch_nl<2>(a, grid, ctx, s) : launch_nl<1>(a, grid, ctx, s);
}

}  // namespace

size_t fanout_max_row_bytes() { return kStageBudget / 4; }

cudaError_t launch_pack(const void *x, int elem_bytes, int H, const moe_layout &L, void *packed,
                        void *packed_hop1, const DeviceCtx &ctx, cudaStream_t s) {
  FanoutArgs a;
  a.src = static_cast<const uint8_t *>(x);
  a.rb = (uint32_t)((size_t)H * elem_bytes);
  a.n_items = L.T;
  a.k = L.k;
  if (L.mode != MOE_LAYOUT_TWO_HOP) {
    a.lists[0] = L.token_rows;
    a.dst[0] = static_cast<uint8_t *>(packed);
    a.dst_cap[0] = L.capacity;
    a.lists[1] = nullptr;
    a.dst[1] = nullptr;
    a.dst_cap[1] = 0;
    return launch_fanout(a, ctx, s);
  }
  // both hops from one read of the token: its group rows (hop 1) and its rank
  // rows (hop 2, bit-identical to forwarding the group rows)
  a.lists[0] = L.token_groups;
  a.dst[0] = static_cast<uint8_t *>(packed_hop1);
  a.dst_cap[0] = L.capacity_hop1;
  a.lists[1] = L.token_rows;
  a.dst[1] = static_cast<uint8_t *>(packed);
  a.dst_cap[1] = L.capacity;
  return launch_fanout(a, ctx, s);
}

}  // namespace moe
