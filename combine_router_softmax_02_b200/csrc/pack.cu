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
// One warp per token.  Lanes 0..W-1 fetch the destination rows and broadcast
// them; each lane then walks the row in 16-byte column vectors, kU at a time:
// streaming loads into registers (ld.global.nc.L1::no_allocate), then one
// st.global.v4 per destination, so every warp store writes 512 contiguous
// bytes.  Pack traffic is ~90% writes.  On B200 the register store path
// writes faster than the bulk-copy (TMA) store engine: a write-only probe gave
// 6.7 TB/s for st.global.v4 against 6.3 TB/s for cp.async.bulk stores, and a
// TMA version of this kernel (row to shared memory on an mbarrier, one bulk
// store per destination) reached 5.7 TB/s where this one reaches 6.1 TB/s.
#include "moe_internal.cuh"

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
  int slices;               // warps per item, each a column slice of the row
  int svec;                 // 16-byte vectors per slice
  int hold = 0;             // sliced rows that still take the residency hold
};

// Column vectors per lane per iteration (a sweep over 1-4 on both benchmark
// workloads picked 2).  The grid is one block per 8 tokens, uncapped: resident
// blocks then work on consecutive tokens, so the writes of every destination
// segment advance as one window.  Capping it at 16 blocks per SM with a
// grid-stride loop split the resident tokens into disjoint windows and cost
// 2.5% on the 65536-token workload (a write probe shows the same: a sliding
// window of stores runs at 7.1 TB/s, scattered windows at 6.2-6.9); a
// persistent grid of 2 blocks per SM cost 11%.
//
// Residency: fewer concurrent warps write fewer rows at a time, and the DRAM
// then serves the writes faster.  A launch of whole rows (one slice each) and
// more than 2 blocks per SM therefore reserves just over a third of the SM's
// shared memory per block (unused), which holds it at 2 resident blocks per
// SM: 5 -> 2 blocks per SM took the 65536-token pack from 1326 to 1302 us and
// the two-hop pack from 555 to 548 us (3 and 4 blocks per SM fell in between,
// 1 block was slower on the first); on the 8192-token training workload the
// same hold gives 78.6 -> 75.7 us.  A decode-sized launch (rows split into
// column slices) keeps every warp for latency: the hold cost it 22.8 -> 24.2 us.
constexpr int kU = 2;
constexpr int kResidentBlocks = 2;

template <int KM, int NL, int U>
__global__ void __launch_bounds__(256) fanout_kernel(FanoutArgs a, DeviceCtx ctx) {
  wait_prior_grids();
  constexpr int W = NL * KM;
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int nvec = (int)(a.rb / 16);
  const int n_work = a.n_items * a.slices;  // < 2^31: slices > 1 only for few rows
  bool bounds = false;
  for (unsigned wk = blockIdx.x * wpb + (threadIdx.x >> 5); wk < (unsigned)n_work; wk += gridDim.x * wpb) {
    const int item = (int)(wk / (unsigned)a.slices);
    const int vbeg = (int)(wk % (unsigned)a.slices) * a.svec;
    const int vend = min(nvec, vbeg + a.svec);
    int my = -1;
    if (lane < W) {
      const int l = lane / KM, j = lane % KM;
      if (j < a.k) {
        my = __ldcs(a.lists[l] + (size_t)item * a.k + j);
        if (my >= a.dst_cap[l] || my < -1) {
          bounds = true;
          my = -1;
        }
      }
    }
    const unsigned dmask = __ballot_sync(kFull, my >= 0);
    uint8_t *dst[W];
#pragma unroll
    for (int j = 0; j < W; ++j) {
      const int r = __shfl_sync(kFull, my, j);
      dst[j] = a.dst[j / KM] + (size_t)(r < 0 ? 0 : r) * a.rb;
    }
    const uint8_t *srow = a.src + (size_t)item * a.rb;
    for (int v0 = vbeg + lane; v0 < vend; v0 += 32 * U) {
      uint4 x[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (v0 + 32 * u < vend) x[u] = ld_stream_v4(srow + (size_t)(v0 + 32 * u) * 16);
#pragma unroll
      for (int j = 0; j < W; ++j)
        if (dmask >> j & 1u)
#pragma unroll
          for (int u = 0; u < U; ++u)
            if (v0 + 32 * u < vend) st_v4(dst[j] + (size_t)(v0 + 32 * u) * 16, x[u]);
    }
  }
  if (bounds) set_status(ctx.status, MOE_ERR_BOUNDS);
}

template <int KM, int NL>
cudaError_t launch_kn(const FanoutArgs &a, const DeviceCtx &ctx, cudaStream_t s) {
  const int wpb = 8;
  const long blocks = ((long)a.n_items * a.slices + wpb - 1) / wpb;
  int smem = 0;
  if ((a.slices == 1 || a.hold) && blocks > 2L * ctx.num_sms && ctx.smem_per_sm > 0) {  // decode keeps all warps
    smem = ctx.smem_per_sm / (kResidentBlocks + 1) + 1024;  // room for 2 blocks, not for 3
    static std::atomic<unsigned long long> smem_set{0};
    cudaError_t err = set_smem_limit_once(fanout_kernel<KM, NL, kU>, 160 * 1024, smem_set);
    if (err != cudaSuccess) return err;
  }
  cudaError_t err = launch_after_prior(fanout_kernel<KM, NL, kU>, dim3((unsigned)blocks), dim3(wpb * 32),
                                       (size_t)smem, s, a, ctx);
  if (err != cudaSuccess) return err;
  return count_launch(cudaGetLastError());
}

template <int NL>
cudaError_t launch_nl(const FanoutArgs &a, const DeviceCtx &ctx, cudaStream_t s) {
  if (a.k <= 2) return launch_kn<2, NL>(a, ctx, s);
  if (a.k <= 4) return launch_kn<4, NL>(a, ctx, s);
  if (a.k <= 8) return launch_kn<8, NL>(a, ctx, s);
  return launch_kn<16, NL>(a, ctx, s);
}

cudaError_t launch_fanout(FanoutArgs a, const DeviceCtx &ctx, cudaStream_t s) {
  if (a.n_items <= 0) return cudaSuccess;
  row_slices(a.n_items, (int)(a.rb / 16), ctx.num_sms, a.slices, a.svec);
  // One to four rows per resident warp (two blocks per SM under the hold):
  // half rows even out the last, part-empty turn (75.7 -> 74.1 us on the
  // 8192-token training workload), and keep the hold.
  const long warps = (long)kResidentBlocks * 8 * ctx.num_sms;
  if (a.slices == 1 && a.n_items > warps && a.n_items <= 4 * warps) {
    const int nvec = (int)(a.rb / 16);
    a.svec = ((nvec + 1) / 2 + 31) / 32 * 32;
    a.slices = (nvec + a.svec - 1) / a.svec;
    a.hold = 1;
  }
  return a.lists[1] ? launch_nl<2>(a, ctx, s) : launch_nl<1>(a, ctx, s);
}

}  // namespace

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
