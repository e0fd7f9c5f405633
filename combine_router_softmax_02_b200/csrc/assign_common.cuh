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
// so that warp 0 can walk the choice experts, in ascending id, with one
// shared load per replica: lane i takes replica i, adds chosen(r) << 21 (kept
// in lane registers: lane r holds ranks r and r + 32, read with two shuffles),
// one redux.sync.min picks the winner -- the tie rules are the key's bit
// order -- and the winner's lane increments its count.  Counts stay below
// 2^11 (E <= 1024), so the sum never carries into the rank bits.  The loads
// of the next expert do not depend on the walk and are issued one expert
// ahead.
#pragma once

#include "moe_internal.cuh"

namespace moe {

// Shared memory of metro_stage / metro_solve, as offsets in ints.
struct MetroPlan {
  int off;    // [E + 1] replica offsets
  int key;    // [n_entries] rank << 15 | slot of each replica entry, -1 if invalid;
              // for an active choice expert, forced(m, r) << 21 added (0xffffffff if invalid)
  int fk;     // [E] forced key (>= 0), kChoice (2+ valid replicas), kNone (none valid), kBadOff
  int list;   // [E] active choice experts, ascending
  int rec;    // [E] per list entry: its expert's first replica entry
  int cmask;  // [C] per chunk: active choice experts (bit = expert - 32 * chunk)
  int mask;   // [C][R] per chunk and rank: forced active experts
  int pre;    // [C + 1][R] forced active experts of all earlier chunks
  int nlist;  // [1] length of list
  int total;
};

constexpr int kChoice = -2;
constexpr int kNone = -1;
constexpr int kBadOff = -3;

__host__ __device__ inline MetroPlan metro_plan(int E, int n_entries, int R) {
  const int C = (E + 31) / 32;
  MetroPlan p;
  int o = 0;
  p.off = o;   o += E + 1;
  p.key = o;   o += n_entries;
  p.fk = o;    o += E;
  p.list = o;  o += E;
  p.rec = o;   o += E;
  p.cmask = o; o += C;
  p.mask = o;  o += C * R;
  p.pre = o;   o += (C + 1) * R;
  p.nlist = o; o += 1;
  p.total = o;
  return p;
}

// Shared memory the assignment needs, in ints.
__host__ __device__ inline int assign_smem_ints(int E, int n_entries, int R) {
  return metro_plan(E, n_entries, R).total;
}

// Stages the replica map and classifies every expert by its valid replicas.
// Needs no demand counts, so the fused front end runs it before its first
// grid barrier.  Every thread of the block calls it (at least 64 + R
// threads); ends with __syncthreads.
__device__ __forceinline__ void metro_stage(int E, const int *__restrict__ off,
                                            const int *__restrict__ slots, int n_entries,
                                            const int *__restrict__ slot_rank, int S, int R,
                                            int *sm, const MetroPlan &P) {
  int *s_off = sm + P.off, *s_key = sm + P.key, *s_fk = sm + P.fk;
  const int C = (E + 31) / 32;
  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_off[i] = off[i];
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

// The greedy over the demand vector `counts` (read through L2: other blocks
// of the same launch may have written it), after metro_stage (once: it
// rewrites the staged keys).  Every thread of the block calls it.  Writes the
// expert -> rank map to `s_rank` (shared, E ints; -1 for inactive experts)
// and, when `write_out`, the global outputs expert_slot, expert_rank and
// rank_active.  Returns after a __syncthreads.
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
  int *s_pre = sm + P.pre;

  // 1: classify with the demand, one warp per 32-expert chunk: forced
  // experts go straight to their rank and into the chunk's rank masks
  bool bad = false;
  for (int c = warp; c < C; c += nwarps) {
    const int e = c * 32 + lane;
    bool choice = false;
    int r = -1;
    if (e < E) {
      const int cnt = __ldcg(counts + e);
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

  // 2: forced experts of earlier chunks per rank (threads 64 .. 64 + R - 1),
  // and the ascending list of active choice experts (warp 0)
  if (tid >= 64 && tid < 64 + R) {
    const int r = tid - 64;
    int run = 0;
    for (int c = 0; c < C; ++c) {
      s_pre[c * R + r] = run;
      run += __popc(s_mask[c * R + r]);
    }
    s_pre[C * R + r] = run;
  }
  if (warp == 0) {
    int base = 0;
    for (int c = 0; c < C; ++c) {
      const unsigned cm = (unsigned)s_cmask[c];
      if (cm >> lane & 1u) s_list[base + __popc(cm & lanemask_lt())] = c * 32 + lane;
      base += __popc(cm);
    }
    if (lane == 0) sm[P.nlist] = base;
  }
  __syncthreads();

  // 3: every replica entry of a choice expert m gets forced(m, r) << 21
  const int n = sm[P.nlist];
  for (int j = tid; j < n; j += blockDim.x) {
    const int m = s_list[j], c = m >> 5;
    const unsigned below = (1u << (m & 31)) - 1u;
    const int lo = s_off[m], hi = s_off[m + 1];
    s_rec[j] = lo;
    for (int i = lo; i < hi; ++i) {
      const unsigned kb = s_key[i];
      if ((int)kb < 0) {
        s_key[i] = 0xffffffffu;
      } else {
        const int r = kb >> 15;
        const unsigned f = (unsigned)(s_pre[c * R + r] + __popc(s_mask[c * R + r] & below));
        s_key[i] = (f << 21) | kb;
      }
    }
  }
  __syncthreads();

  // 4: the walk over the choice experts (warp 0)
  if (warp == 0) {
    int ch0 = 0, ch1 = 0;  // choice experts so far on ranks lane and lane + 32
    int m = 0, lo = 0, hi = 0;
    unsigned kb = 0xffffffffu;
    if (n > 0) {
      m = s_list[0];
      lo = s_rec[0];
      hi = s_off[m + 1];
      kb = lo + lane < hi ? s_key[lo + lane] : 0xffffffffu;
    }
    for (int j = 0; j < n; ++j) {
      int m2 = 0, lo2 = 0, hi2 = 0;
      unsigned kb2 = 0xffffffffu;
      if (j + 1 < n) {  // the next expert's loads, ahead of this one's walk
        m2 = s_list[j + 1];
        lo2 = s_rec[j + 1];
        hi2 = s_off[m2 + 1];
        kb2 = lo2 + lane < hi2 ? s_key[lo2 + lane] : 0xffffffffu;
      }
      const int rr = (kb >> 15) & 63;
      const int a0 = __shfl_sync(kFull, ch0, rr & 31), a1 = __shfl_sync(kFull, ch1, rr & 31);
      unsigned best = kb != 0xffffffffu ? kb + ((unsigned)(rr < 32 ? a0 : a1) << 21) : 0xffffffffu;
      for (int base = lo + 32; base < hi; base += 32) {  // more than 32 replicas
        const unsigned k2 = base + lane < hi ? s_key[base + lane] : 0xffffffffu;
        const int r2 = (k2 >> 15) & 63;
        const int b0 = __shfl_sync(kFull, ch0, r2 & 31), b1 = __shfl_sync(kFull, ch1, r2 & 31);
        if (k2 != 0xffffffffu) best = min(best, k2 + ((unsigned)(r2 < 32 ? b0 : b1) << 21));
      }
      best = __reduce_min_sync(kFull, best);
      const int w = (best >> 15) & 63;  // a choice expert has 2+ valid replicas
      if (lane == (w & 31)) {
        if (w < 32)
          ++ch0;
        else
          ++ch1;
      }
      if (lane == 0) {
        s_rank[m] = w;
        if (write_out) {
          expert_slot[m] = best & 0x7fff;
          expert_rank[m] = w;
        }
      }
      m = m2;
      lo = lo2;
      hi = hi2;
      kb = kb2;
    }
    if (write_out) {
      if (lane < R) rank_active[lane] = s_pre[C * R + lane] + ch0;
      if (lane + 32 < R) rank_active[lane + 32] = s_pre[C * R + lane + 32] + ch1;
    }
  }
  __syncthreads();
}

}  // namespace moe
