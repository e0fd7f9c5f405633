// METRO greedy replica assignment by one block (shared by the assignment
// kernel and the fused single-launch front end).
//
// "METRO AllGather vs AllToAll for MoE decode" (fanout.sh), sections "changes
// the routing information" and "Add the expert-weight traffic term": each
// active expert goes to one of its replicas on the GPU with the fewest
// already-activated experts (a greedy, not the optimal min-max assignment).
// Experts are visited in ascending id; ties go to the lower rank, then to the
// lower slot id.
//
// The greedy is serial only through the experts that have a choice.  An
// expert with one valid replica ("forced") adds one activated expert to a
// fixed rank whatever happened before it, so the count a choice expert m sees
// on rank r splits into
//   forced(m, r) = forced active experts below m on r, and
//   chosen(r)    = choice experts before m that went to r.
// forced(m, r) needs no walk: the experts are cut into 32-expert chunks, a
// bitmask per (chunk, rank) marks the chunk's forced active experts on that
// rank, and forced(m, r) = (sum of the mask populations of the earlier chunks)
// + popc(mask[chunk(m)][r] & lanes below m) -- built by the whole block in
// parallel.  The block then rewrites each replica entry of a choice expert as
//   forced(m, r) << 21 | r << 15 | slot
// so that the walk over the choice experts, in ascending id, adds
// chosen(r) << 21 and takes the minimum: the tie rules are the key's bit
// order.  Counts stay below 2^11 (E <= 1024), so the sum never carries into
// the rank bits.  When no choice expert has more than kScalarReps replicas
// and there are at most 255 choice experts (the usual redundant-replica
// maps), one thread walks with chosen() packed 8 bits a rank in 64-bit
// registers and the next expert's keys loaded ahead: a step is a few register
// operations, with no shared-memory round trip and no warp-collective
// operation on the chain.  Otherwise warp 0 walks: lane i takes replica i,
// chosen() sits in lane registers (lane r holds ranks r and r + 32, read with
// two shuffles) and one redux.sync.min picks the winner.
#pragma once

#include "moe_internal.cuh"

namespace moe {

// Shared memory of metro_stage / metro_solve, as offsets in ints from a
// 16-byte aligned base.
struct MetroPlan {
  int off;    // [E + 1] replica offsets
  int key;    // [n_entries] rank << 15 | slot of each replica entry, -1 if invalid;
              // for an active choice expert, forced(m, r) << 21 added (0xffffffff if invalid)
  int fk;     // [E] forced key (>= 0), kChoice (2+ valid replicas), kNone (none valid), kBadOff
  int cnt;    // [E] the demand counts, when metro_stage was given them
  int list;   // [E] active choice experts, ascending
  int rec;    // [E] per list entry: its expert's first replica entry
  int cmask;  // [C] per chunk: active choice experts (bit = expert - 32 * chunk)
  int mask;   // [C][R] per chunk and rank: forced active experts
  int pre;    // [C + 1][R] forced active experts of all earlier chunks
  int chosen; // [R] choice experts assigned to each rank (after the walk)
  int kw;     // [256][kScalarReps] the first replica keys of the first 256 list entries
  int cw;     // [16] the one-thread walk's packed counts (8 x 64-bit)
  int nlist;  // [1] length of list
  int maxrep; // [1] most replica entries of a choice expert
  int total;
};

constexpr int kChoice = -2;
constexpr int kNone = -1;
constexpr int kBadOff = -3;
constexpr int kScalarReps = 4;  // replicas per choice expert the one-thread walk handles (the
                                // walk loads them as one 16-byte vector)

__host__ __device__ inline MetroPlan metro_plan(int E, int n_entries, int R) {
  const int C = (E + 31) / 32;
  MetroPlan p;
  int o = 0;
  p.off = o;    o += E + 1;
  p.key = o;    o += n_entries;
  p.fk = o;     o += E;
  p.cnt = o;    o += E;
  p.list = o;   o += E;
  p.rec = o;    o += E;
  p.cmask = o;  o += C;
  p.mask = o;   o += C * R;
  p.pre = o;    o += (C + 1) * R;
  p.chosen = o; o += R;
  o = (o + 3) & ~3;  // 16-byte aligned (the plan starts 16-byte aligned)
  p.kw = o;     o += 256 * 4;
  p.cw = o;     o += 16;
  p.nlist = o;  o += 1;
  p.maxrep = o; o += 1;
  p.total = o;
  return p;
}

// Shared memory the assignment needs, in ints.
__host__ __device__ inline int assign_smem_ints(int E, int n_entries, int R) {
  return metro_plan(E, n_entries, R).total;
}

// Stages the replica map and classifies every expert by its valid replicas;
// stages the demand counts too when `counts` is given (the fused front end
// runs this before its first grid barrier, when the counts are not complete,
// and passes null).  Every thread of the block calls it (at least 8 warps);
// ends with __syncthreads.
__device__ __forceinline__ void metro_stage(int E, const int *__restrict__ off,
                                            const int *__restrict__ slots, int n_entries,
                                            const int *__restrict__ slot_rank, int S, int R,
                                            const int *__restrict__ counts, int *sm,
                                            const MetroPlan &P) {
  int *s_off = sm + P.off, *s_key = sm + P.key, *s_fk = sm + P.fk;
  const int C = (E + 31) / 32;
  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_off[i] = off[i];
  if (counts)
    for (int i = threadIdx.x; i < E; i += blockDim.x) sm[P.cnt + i] = counts[i];
  for (int i = threadIdx.x; i < n_entries; i += blockDim.x) {
    const int sl = slots[i];
    int key = -1;
    if ((unsigned)sl < (unsigned)S) {
      const int r = slot_rank[sl];
      if ((unsigned)r < (unsigned)R) key = (r << 15) | sl;
    }
    s_key[i] = key;
  }
  for (int i = threadIdx.x; i < C * R; i += blockDim.x) sm[P.mask + i] = 0;
  for (int i = threadIdx.x; i < R; i += blockDim.x) sm[P.chosen + i] = 0;
  if (threadIdx.x == 0) sm[P.maxrep] = 0;
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int lo = s_off[e], hi = s_off[e + 1];
    int fk = kNone;
    if (lo < 0 || hi > n_entries || lo > hi) {
      fk = kBadOff;
    } else {
      int nvalid = 0;
      for (int i = lo; i < hi && nvalid < 2; ++i)
        if (s_key[i] >= 0) {
          ++nvalid;
          fk = s_key[i];
        }
      if (nvalid >= 2) fk = kChoice;
    }
    s_fk[e] = fk;
  }
  __syncthreads();
}

// The replica map loaded into registers before the caller's other work
// (the fused front end issues these loads before it routes, so their latency
// hides behind the routing): thread i holds entries i and i + 256 of the
// offsets, the slot list and the slot -> rank table.  `ok` says the map is
// small enough (E + 1, entries and slots each <= 512) -- otherwise
// metro_stage loads it itself.
struct MetroPrefetch {
  static constexpr int kPer = 2;
  bool ok;
  int off[kPer], slot[kPer], srank[kPer];
  __device__ __forceinline__ void load(int E, const int *__restrict__ off_g, const int *__restrict__ slots_g,
                                       int n_entries, const int *__restrict__ slot_rank_g, int S) {
    ok = E + 1 <= kPer * 256 && n_entries <= kPer * 256 && S <= kPer * 256 && blockDim.x == 256;
    if (!ok) return;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int i = (int)threadIdx.x + q * 256;
      off[q] = i <= E ? off_g[i] : 0;
      slot[q] = i < n_entries ? slots_g[i] : 0;
      srank[q] = i < S ? slot_rank_g[i] : 0;
    }
  }
};

// metro_stage from a prefetched map (no global loads): the slot -> rank
// table goes through the P.kw area (free until the solve).
__device__ __forceinline__ void metro_stage_prefetched(int E, int n_entries, int S, int R,
                                                       const MetroPrefetch &pf, int *sm,
                                                       const MetroPlan &P) {
  int *s_off = sm + P.off, *s_key = sm + P.key, *s_fk = sm + P.fk, *s_srank = sm + P.kw;
  const int C = (E + 31) / 32;
#pragma unroll
  for (int q = 0; q < MetroPrefetch::kPer; ++q) {
    const int i = (int)threadIdx.x + q * 256;
    if (i <= E) s_off[i] = pf.off[q];
    if (i < S) s_srank[i] = pf.srank[q];
  }
  for (int i = threadIdx.x; i < C * R; i += blockDim.x) sm[P.mask + i] = 0;
  for (int i = threadIdx.x; i < R; i += blockDim.x) sm[P.chosen + i] = 0;
  if (threadIdx.x == 0) sm[P.maxrep] = 0;
  __syncthreads();
#pragma unroll
  for (int q = 0; q < MetroPrefetch::kPer; ++q) {
    const int i = (int)threadIdx.x + q * 256;
    if (i < n_entries) {
      const int sl = pf.slot[q];
      int key = -1;
      if ((unsigned)sl < (unsigned)S) {
        const int r = s_srank[sl];
        if ((unsigned)r < (unsigned)R) key = (r << 15) | sl;
      }
      s_key[i] = key;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int lo = s_off[e], hi = s_off[e + 1];
    int fk = kNone;
    if (lo < 0 || hi > n_entries || lo > hi) {
      fk = kBadOff;
    } else {
      int nvalid = 0;
      for (int i = lo; i < hi && nvalid < 2; ++i)
        if (s_key[i] >= 0) {
          ++nvalid;
          fk = s_key[i];
        }
      if (nvalid >= 2) fk = kChoice;
    }
    s_fk[e] = fk;
  }
  __syncthreads();
}

// The walk by one thread: chosen(r) is byte r % 8 of c[r / 8] (counts stay
// below 256: at most 255 choice experts), selected and bumped with register
// operations only; each expert's keys are one 16-byte shared load, issued an
// expert ahead.  Leaves the packed counts in shared memory (P.cw).
template <int NW>
__device__ __forceinline__ void scalar_walk(int n, int *sm, const MetroPlan &P, int *s_rank,
                                            bool write_out, int *expert_slot, int *expert_rank) {
  static_assert(kScalarReps == 4, "one uint4 per expert");
  const int *s_list = sm + P.list;
  const uint4 *s_kw = reinterpret_cast<const uint4 *>(sm + P.kw);
  unsigned long long c[NW];
#pragma unroll
  for (int q = 0; q < NW; ++q) c[q] = 0ull;
  auto count_of = [&](unsigned r) -> unsigned {
    unsigned long long word = c[0];
#pragma unroll
    for (int q = 1; q < NW; ++q) word = ((r >> 3) == (unsigned)q) ? c[q] : word;
    return (unsigned)(word >> ((r & 7u) * 8u)) & 0xffu;
  };
  auto eval = [&](unsigned kb, unsigned &best) {
    if (kb != 0xffffffffu) best = min(best, kb + (count_of((kb >> 15) & 63u) << 21));
  };
  uint4 nk = make_uint4(0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu);
  int nm = 0;
  if (n > 0) {
    nk = s_kw[0];
    nm = s_list[0];
  }
  for (int j = 0; j < n; ++j) {
    const uint4 kb = nk;
    const int m = nm;
    if (j + 1 < n) {  // independent of the walk: loaded ahead
      nk = s_kw[j + 1];
      nm = s_list[j + 1];
    }
    unsigned best = 0xffffffffu;
    eval(kb.x, best);
    eval(kb.y, best);
    eval(kb.z, best);
    eval(kb.w, best);
    const unsigned w = (best >> 15) & 63u;  // a choice expert has 2+ valid replicas
    const unsigned long long inc = 1ull << ((w & 7u) * 8u);
#pragma unroll
    for (int q = 0; q < NW; ++q) c[q] += ((w >> 3) == (unsigned)q) ? inc : 0ull;
    s_rank[m] = (int)w;
    if (write_out) {
      expert_slot[m] = best & 0x7fff;
      expert_rank[m] = (int)w;
    }
  }
  unsigned long long *cw = reinterpret_cast<unsigned long long *>(sm + P.cw);
#pragma unroll
  for (int q = 0; q < 8; ++q) cw[q] = q < NW ? c[q] : 0ull;
}

// The greedy over the demand vector, after metro_stage (once: it rewrites the
// staged keys).  `counts` is read through L2 (other blocks of the same launch
// may have written it); null means the counts metro_stage staged.  Every
// thread of the block calls it.  Writes the expert -> rank map to `s_rank`
// (shared, E ints; -1 for inactive experts) and, when `write_out`, the global
// outputs expert_slot, expert_rank and rank_active.  Returns after a
// __syncthreads.
__device__ __forceinline__ void metro_solve(const int *counts, int E, int R, int *sm,
                                            const MetroPlan &P, int *s_rank, bool write_out,
                                            int *expert_slot, int *expert_rank, int *rank_active,
                                            const DeviceCtx &ctx) {
  constexpr unsigned kFull = 0xffffffffu;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int C = (E + 31) / 32;
  const int *s_off = sm + P.off, *s_fk = sm + P.fk;
  unsigned *s_key = reinterpret_cast<unsigned *>(sm + P.key);
  int *s_list = sm + P.list, *s_rec = sm + P.rec, *s_cmask = sm + P.cmask;
  unsigned *s_mask = reinterpret_cast<unsigned *>(sm + P.mask);
  int *s_pre = sm + P.pre, *s_chosen = sm + P.chosen;

  // 1: classify with the demand, one warp per 32-expert chunk: forced
  // experts go straight to their rank and into the chunk's rank masks
  bool bad = false;
  for (int c = warp; c < C; c += nwarps) {
    const int e = c * 32 + lane;
    bool choice = false;
    int r = -1;
    if (e < E) {
      const int cnt = counts ? __ldcg(counts + e) : sm[P.cnt + e];
      const int fk = s_fk[e];
      if (cnt < 0 || fk == kBadOff) bad = true;
      int slot = -1;
      if (cnt > 0) {
        if (fk >= 0) {
          slot = fk & 0x7fff;
          r = fk >> 15;
        } else if (fk == kChoice) {
          choice = true;
        } else {
          bad = true;  // active expert without a valid replica
        }
      }
      if (!choice) {
        s_rank[e] = r;
        if (write_out) {
          expert_slot[e] = slot;
          expert_rank[e] = r;
        }
      }
    }
    // lanes of forced experts on the same rank: the lowest one writes the mask
    const unsigned peers = __match_any_sync(kFull, r >= 0 ? r : 64 + lane);
    if (r >= 0 && lane == __ffs(peers) - 1) s_mask[c * R + r] = peers;
    const unsigned cm = __ballot_sync(kFull, choice);
    if (lane == 0) s_cmask[c] = (int)cm;
  }
  if (bad) set_status(ctx.status, MOE_ERR_BAD_INPUT);
  __syncthreads();

  // 2: forced experts of earlier chunks per (chunk, rank), row C = all
  // chunks, and the ascending list of active choice experts, each chunk's
  // experts after those of the earlier chunks: exclusive warp scans over the
  // chunks (lane c holds chunk c; C <= 32), one per rank and one for the list.
  auto warp_scan = [&](int v) {  // inclusive prefix sum over the lanes
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int t = __shfl_up_sync(kFull, v, d);
      if (lane >= d) v += t;
    }
    return v;
  };
  for (int r = warp; r < R; r += nwarps) {
    const int v = lane < C ? __popc(s_mask[lane * R + r]) : 0;
    const int incl = warp_scan(v);
    if (lane < C) s_pre[lane * R + r] = incl - v;
    if (lane == C - 1) s_pre[C * R + r] = incl;
  }
  if (warp == nwarps - 1) {
    const unsigned cm = lane < C ? (unsigned)s_cmask[lane] : 0u;
    const int v = __popc(cm);
    const int incl = warp_scan(v);
    int base = incl - v;
    for (unsigned m = cm; m; m &= m - 1) s_list[base++] = lane * 32 + __ffs(m) - 1;
    if (lane == 31) sm[P.nlist] = incl;
  }
  __syncthreads();

  // 3: every replica entry of a choice expert m gets forced(m, r) << 21
  const int n = sm[P.nlist];
  for (int j = tid; j < n; j += blockDim.x) {
    const int m = s_list[j], c = m >> 5;
    const unsigned below = (1u << (m & 31)) - 1u;
    const int lo = s_off[m], hi = s_off[m + 1];
    s_rec[j] = lo;
    atomicMax(&sm[P.maxrep], hi - lo);
    for (int i = lo; i < hi; ++i) {
      const unsigned kb = s_key[i];
      unsigned key = 0xffffffffu;
      if ((int)kb >= 0) {
        const int r = kb >> 15;
        const unsigned f = (unsigned)(s_pre[c * R + r] + __popc(s_mask[c * R + r] & below));
        key = (f << 21) | kb;
      }
      s_key[i] = key;
      if (j < 256 && i - lo < kScalarReps) sm[P.kw + j * kScalarReps + (i - lo)] = (int)key;
    }
    if (j < 256)
      for (int q = hi - lo; q < kScalarReps; ++q) sm[P.kw + j * kScalarReps + q] = -1;
  }
  __syncthreads();

  // 4: the walk over the choice experts
  if (sm[P.maxrep] <= kScalarReps && n <= 255) {
    if (tid == 0) {
      if (R <= 8)
        scalar_walk<1>(n, sm, P, s_rank, write_out, expert_slot, expert_rank);
      else if (R <= 16)
        scalar_walk<2>(n, sm, P, s_rank, write_out, expert_slot, expert_rank);
      else if (R <= 32)
        scalar_walk<4>(n, sm, P, s_rank, write_out, expert_slot, expert_rank);
      else
        scalar_walk<8>(n, sm, P, s_rank, write_out, expert_slot, expert_rank);
    }
    __syncthreads();
    const unsigned char *cb = reinterpret_cast<const unsigned char *>(sm + P.cw);
    for (int r = tid; r < R; r += blockDim.x) s_chosen[r] = cb[r];  // little-endian bytes
  } else if (warp == 0) {  // warp 0, chosen() in lane registers
    int ch0 = 0, ch1 = 0;  // choice experts so far on ranks lane and lane + 32
    for (int j = 0; j < n; ++j) {
      const int m = s_list[j], lo = s_rec[j], hi = s_off[m + 1];
      unsigned best = 0xffffffffu;
      for (int base = lo; base < hi; base += 32) {
        const unsigned k2 = base + lane < hi ? s_key[base + lane] : 0xffffffffu;
        const int r2 = (k2 >> 15) & 63;
        const int b0 = __shfl_sync(kFull, ch0, r2 & 31), b1 = __shfl_sync(kFull, ch1, r2 & 31);
        if (k2 != 0xffffffffu) best = min(best, k2 + ((unsigned)(r2 < 32 ? b0 : b1) << 21));
      }
      best = __reduce_min_sync(kFull, best);
      const int w = (best >> 15) & 63;  // a choice expert has 2+ valid replicas
      ch0 += (lane == (w & 31) && w < 32) ? 1 : 0;
      ch1 += (lane == (w & 31) && w >= 32) ? 1 : 0;
      if (lane == 0) {
        s_rank[m] = w;
        if (write_out) {
          expert_slot[m] = best & 0x7fff;
          expert_rank[m] = w;
        }
      }
    }
    if (lane < R) s_chosen[lane] = ch0;
    if (lane + 32 < R) s_chosen[lane + 32] = ch1;
  }
  __syncthreads();
  if (write_out)
    for (int r = tid; r < R; r += blockDim.x) rank_active[r] = s_pre[C * R + r] + s_chosen[r];
  __syncthreads();
}

}  // namespace moe
