// Union step: batch-union of the experts a batch selected (Colibri README,
// "Mai aspettare il disco due volte": positions of a batch read each unique
// expert once; getting-started guide, "2. Union": duplicates removed when
// several tokens of a batch pick the same expert), plus the FFN tile plan.
#pragma once
#include "common.cuh"
#include "k_router.cuh"

namespace coli {

constexpr int kUnionThreads = 1024;
constexpr int kUnionWarps = kUnionThreads / 32;
constexpr int kFusedRouteMaxT = 128;      // route + union + plan in one CTA up to this batch

// Stable counting sort of the pairs p = t*k + j by expert id, in one CTA and
// without atomics.  Warp w owns the contiguous pair range [w*C, (w+1)*C).
//  1. Each warp builds its private histogram hist[w][e]: lanes holding the
//     same id are grouped with __match_any_sync and the group's lowest lane
//     adds the group size (one writer per bin per step).
//  2. Thread e turns column e into per-warp running offsets; a block scan
//     over the per-expert totals gives each expert's segment start; experts
//     with a non-zero count are compacted into unique_ids / seg_off (and their
//     counts into seg_cnt, in shared memory, for the plan).
//  3. Each warp walks its range again in the same order and writes
//     perm[pos] = p, pair_pos[p] = pos with pos = its (expert, warp) base +
//     rank among earlier equal ids, so equal ids keep pair order.
// `ids` may point to global or shared memory.  Returns U (valid in every
// thread).  hist: kUnionWarps * E ints of shared memory.
__device__ __forceinline__ int block_union(const int32_t* ids, int P, int E, int* hist, int* scratch,
                                           int* seg_cnt, int32_t* __restrict__ unique_ids,
                                           int32_t* __restrict__ n_unique, int32_t* __restrict__ seg_off,
                                           int32_t* __restrict__ perm, int32_t* __restrict__ pair_pos,
                                           uint32_t* __restrict__ status) {
  __shared__ int carry_pairs, carry_u;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kUnionWarps * E; i += blockDim.x) hist[i] = 0;
  if (threadIdx.x == 0) {
    carry_pairs = 0;
    carry_u = 0;
  }
  __syncthreads();

  const int chunk = ((P + kUnionWarps - 1) / kUnionWarps + 31) & ~31;
  const int p_begin = min(P, warp * chunk), p_end = min(P, p_begin + chunk);
  int* myhist = hist + warp * E;
  bool bad = false;
  for (int base = p_begin; base < p_end; base += 32) {
    const int p = base + lane;
    int e = -1;
    if (p < p_end) {
      e = ids[p];
      if (e < 0 || e >= E) {
        bad = true;
        e = -1;
      }
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) myhist[e] += __popc(peers);
    __syncwarp();
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0 && status) atomicOr(status, COLI_FLAG_BAD_ID);
  __syncthreads();

  // per-expert totals and per-(warp, expert) offsets within the expert
  for (int e0 = 0; e0 < E; e0 += blockDim.x) {
    const int e = e0 + threadIdx.x;
    int cnt = 0;
    if (e < E) {
      for (int w = 0; w < kUnionWarps; ++w) {
        const int c = hist[w * E + e];
        hist[w * E + e] = cnt;
        cnt += c;
      }
    }
    int tot_pairs = 0, tot_u = 0;
    const int off = block_exclusive_scan(cnt, scratch, &tot_pairs);
    const int uidx = block_exclusive_scan(cnt > 0 ? 1 : 0, scratch, &tot_u);
    const int cp = carry_pairs, cu = carry_u;
    if (e < E) {
      for (int w = 0; w < kUnionWarps; ++w) hist[w * E + e] += cp + off;
      if (cnt > 0) {
        unique_ids[cu + uidx] = e;
        seg_off[cu + uidx] = cp + off;
        seg_cnt[cu + uidx] = cnt;
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      carry_pairs = cp + tot_pairs;
      carry_u = cu + tot_u;
    }
    __syncthreads();
  }
  const int U = carry_u;
  if (threadIdx.x == 0) {
    *n_unique = U;
    seg_off[U] = carry_pairs;
  }

  for (int base = p_begin; base < p_end; base += 32) {
    const int p = base + lane;
    int e = -1;
    if (p < p_end) {
      e = ids[p];
      if (e < 0 || e >= E) e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const unsigned lower = peers & ((1u << lane) - 1u);
    if (e >= 0) {
      const int pos = myhist[e] + __popc(lower);
      perm[pos] = p;
      pair_pos[p] = pos;
    } else if (p < p_end) {
      pair_pos[p] = -1;
    }
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) myhist[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  return U;
}

// FFN tile plan.  Segments are the S shared experts (every token, weight 1)
// followed by the U unique routed experts.  Segment u is cut into token
// blocks of `tokb` tokens; plan = [n_seg, total_blocks, tile_off[0..n_seg]]
// with tile_off the exclusive prefix of the blocks per segment.  Shared
// segments come first so their tiles do not depend on the routing.
// Also zeroes the FFN's completion counters (tb_done per token block,
// rb_done per output row block) for this call.
__device__ __forceinline__ void block_plan(int U, const int* seg_cnt, int T, int S, int tokb, int* scratch,
                                           int32_t* __restrict__ plan, int32_t* __restrict__ tb_done,
                                           int32_t* __restrict__ rb_done, int n_rb, const int32_t* unique_ids = nullptr, int eb = 0, int ee = 0x7fffffff) {
  __shared__ int carry;
  const int n_seg = U + S;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int u0 = 0; u0 < n_seg; u0 += blockDim.x) {
    const int u = u0 + threadIdx.x;
    int nb = 0;
    if (u < S) nb = (T + tokb - 1) / tokb;
    else if (u < n_seg) {
      // routed segments of experts outside [eb, ee) get no blocks (expert-parallel rank)
      const int eid = unique_ids ? unique_ids[u - S] : eb;
      nb = (eid >= eb && eid < ee) ? (seg_cnt[u - S] + tokb - 1) / tokb : 0;
    }
    int tot = 0;
    const int ex = block_exclusive_scan(nb, scratch, &tot);
    const int c = carry;
    if (u < n_seg) plan[2 + u] = c + ex;
    __syncthreads();
    if (threadIdx.x == 0) carry = c + tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    plan[0] = n_seg;
    plan[1] = carry;
    plan[2 + n_seg] = carry;
  }
  if (tb_done)
    for (int i = threadIdx.x; i < carry; i += blockDim.x) tb_done[i] = 0;
  if (rb_done)
    for (int i = threadIdx.x; i < n_rb; i += blockDim.x) rb_done[i] = 0;
}

// Union of a routed batch (any size) and, if `plan` is given, the FFN tile plan.
// Dynamic shared memory: kUnionWarps * E ints.
__global__ void __launch_bounds__(kUnionThreads, 1)
    union_kernel(const int32_t* __restrict__ ids, int P, int E, int32_t* __restrict__ unique_ids,
                 int32_t* __restrict__ n_unique, int32_t* __restrict__ seg_off, int32_t* __restrict__ perm,
                 int32_t* __restrict__ pair_pos, uint32_t* __restrict__ status, int T, int S, int tokb,
                 int32_t* __restrict__ plan, int32_t* __restrict__ tb_done, int32_t* __restrict__ rb_done,
                 int n_rb) {
  extern __shared__ int hist[];
  __shared__ int scratch[33];
  __shared__ int seg_cnt[1024];
  pdl_wait();
  pdl_trigger();
  const int U = block_union(ids, P, E, hist, scratch, seg_cnt, unique_ids, n_unique, seg_off, perm, pair_pos, status);
  if (plan) block_plan(U, seg_cnt, T, S, tokb, scratch, plan, tb_done, rb_done, n_rb);
}

// ---------------------------------------------------------------------------
// Union of a large batch over many CTAs (the prefill form's batches): the same
// stable counting sort, split in three launches.
//   1. union_count_kernel: CTA b counts the ids of its chunk of pairs per
//      expert (shared-memory atomics: counts do not depend on order) into
//      cnt[b][e];
//   2. union_scan_kernel (one CTA): per expert, an exclusive scan over the
//      chunks; over experts, the segment starts; cnt[b][e] becomes the first
//      position of chunk b's pairs of expert e; unique ids and segments;
//   3. union_scatter_kernel: CTA b ranks its pairs inside each expert with
//      per-warp histograms over contiguous pair ranges (as block_union does)
//      and writes perm / pair_pos, so equal ids keep pair order.
// cnt: ceil(P / chunk) * E ints of workspace; chunk a multiple of 1024.
inline int union_chunk(int P) {
  const int c = (P + 511) / 512;
  return c <= 1024 ? 1024 : (c + 1023) / 1024 * 1024;
}

__global__ void __launch_bounds__(1024) union_count_kernel(const int32_t* __restrict__ ids, int P, int E, int chunk,
                                                           int32_t* __restrict__ cnt, uint32_t* __restrict__ status) {
  extern __shared__ int hist[];
  pdl_wait();
  pdl_trigger();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int p0 = blockIdx.x * chunk, p1 = min(P, p0 + chunk);
  bool bad = false;
  for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
    const int e = ids[p];
    if (e < 0 || e >= E) bad = true;
    else atomicAdd(&hist[e], 1);
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, COLI_FLAG_BAD_ID);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[static_cast<size_t>(blockIdx.x) * E + e] = hist[e];
}

__global__ void __launch_bounds__(1024) union_scan_kernel(int32_t* __restrict__ cnt, int NB, int E,
                                                          int32_t* __restrict__ unique_ids,
                                                          int32_t* __restrict__ n_unique,
                                                          int32_t* __restrict__ seg_off) {
  __shared__ int scratch[33];
  __shared__ int carry_pairs, carry_u;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) {
    carry_pairs = 0;
    carry_u = 0;
  }
  __syncthreads();
  for (int e0 = 0; e0 < E; e0 += blockDim.x) {
    const int e = e0 + threadIdx.x;
    int tot = 0;
    if (e < E)
      for (int b = 0; b < NB; ++b) {
        int32_t* c = cnt + static_cast<size_t>(b) * E + e;
        const int v = *c;
        *c = tot;
        tot += v;
      }
    int tot_pairs = 0, tot_u = 0;
    const int off = block_exclusive_scan(tot, scratch, &tot_pairs);
    const int uidx = block_exclusive_scan(tot > 0 ? 1 : 0, scratch, &tot_u);
    const int cp = carry_pairs, cu = carry_u;
    if (e < E) {
      for (int b = 0; b < NB; ++b) cnt[static_cast<size_t>(b) * E + e] += cp + off;
      if (tot > 0) {
        unique_ids[cu + uidx] = e;
        seg_off[cu + uidx] = cp + off;
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      carry_pairs = cp + tot_pairs;
      carry_u = cu + tot_u;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    *n_unique = carry_u;
    seg_off[carry_u] = carry_pairs;
  }
}

// Dynamic shared memory: kUnionWarps * E ints.
__global__ void __launch_bounds__(kUnionThreads) union_scatter_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                                      int chunk, const int32_t* __restrict__ base,
                                                                      int32_t* __restrict__ perm,
                                                                      int32_t* __restrict__ pair_pos) {
  extern __shared__ int hist[];
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kUnionWarps * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int c0 = blockIdx.x * chunk, c1 = min(P, c0 + chunk);
  const int per_warp = chunk / kUnionWarps;                   // a multiple of 32
  const int p_begin = min(c1, c0 + warp * per_warp), p_end = min(c1, p_begin + per_warp);
  int* myhist = hist + warp * E;
  for (int b0 = p_begin; b0 < p_end; b0 += 32) {
    const int p = b0 + lane;
    int e = -1;
    if (p < p_end) {
      e = ids[p];
      if (e < 0 || e >= E) e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) myhist[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // per (warp, expert) first position: the chunk's base for the expert plus
  // the counts of the lower warps
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int off = base[static_cast<size_t>(blockIdx.x) * E + e];
    for (int w = 0; w < kUnionWarps; ++w) {
      const int c = hist[w * E + e];
      hist[w * E + e] = off;
      off += c;
    }
  }
  __syncthreads();
  for (int b0 = p_begin; b0 < p_end; b0 += 32) {
    const int p = b0 + lane;
    int e = -1;
    if (p < p_end) {
      e = ids[p];
      if (e < 0 || e >= E) e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const unsigned lower = peers & ((1u << lane) - 1u);
    if (e >= 0) {
      const int pos = myhist[e] + __popc(lower);
      perm[pos] = p;
      pair_pos[p] = pos;
    } else if (p < p_end) {
      pair_pos[p] = -1;
    }
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) myhist[e] += __popc(peers);
    __syncwarp();
  }
}

// Plan from an existing union (coli_moe_expert_ffn), one CTA.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ n_unique,
                                                    const int32_t* __restrict__ seg_off, int T, int S, int tokb,
                                                    int32_t* __restrict__ plan, int32_t* __restrict__ tb_done,
                                                    int32_t* __restrict__ rb_done, int n_rb) {
  __shared__ int scratch[33];
  __shared__ int seg_cnt[1024];
  pdl_wait();
  pdl_trigger();
  const int U = *n_unique;
  for (int u = threadIdx.x; u < U; u += blockDim.x) seg_cnt[u] = seg_off[u + 1] - seg_off[u];
  __syncthreads();
  block_plan(U, seg_cnt, T, S, tokb, scratch, plan, tb_done, rb_done, n_rb);
}

// Small batches (T <= kFusedRouteMaxT): Route, Union and the tile plan in one
// CTA.  Warp w routes tokens w, w + 32, ...; the selected ids go to shared
// memory and to `ids_out`; then the union and the plan as above.
// Dynamic shared memory: kUnionWarps * E ints + T * k ints.
template <int NV>
__global__ void __launch_bounds__(kUnionThreads, 1)
    route_union_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int T, int E, int k,
                       int32_t* __restrict__ ids_out, float* __restrict__ w_out, int32_t* __restrict__ unique_ids,
                       int32_t* __restrict__ n_unique, int32_t* __restrict__ seg_off, int32_t* __restrict__ perm,
                       int32_t* __restrict__ pair_pos, uint32_t* __restrict__ status, int S, int tokb,
                       int32_t* __restrict__ plan, int32_t* __restrict__ tb_done, int32_t* __restrict__ rb_done,
                       int n_rb, int eb, int ee) {
  extern __shared__ int smem_i[];
  int* hist = smem_i;
  int* ids_s = smem_i + kUnionWarps * E;
  __shared__ int scratch[33];
  __shared__ int seg_cnt[1024];
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int t = warp; t < T; t += kUnionWarps) {
    int id;
    float w;
    const bool bad = route_token<NV>(logits + static_cast<size_t>(t) * E, bias, E, k, lane, &id, &w);
    if (lane < k) {
      ids_s[t * k + lane] = id;
      ids_out[static_cast<size_t>(t) * k + lane] = id;
      w_out[static_cast<size_t>(t) * k + lane] = w;
    }
    if (bad && lane == 0) atomicOr(status, COLI_FLAG_NONFINITE);
  }
  __syncthreads();
  const int U = block_union(ids_s, T * k, E, hist, scratch, seg_cnt, unique_ids, n_unique, seg_off, perm, pair_pos,
                            status);
  block_plan(U, seg_cnt, T, S, tokb, scratch, plan, tb_done, rb_done, n_rb, unique_ids, eb, ee);
}

// ---------------------------------------------------------------------------
// Small batches (T*k <= 128): the union in ONE warp, without block barriers.
// The 128 keys (expert << 8 | pair) live four per lane (key i in lane i/4,
// slot i%4; unused keys are INT_MAX) and are put in order by a bitonic
// network: partners within a lane swap in registers, partners in other lanes
// are exchanged with __shfl_xor_sync.  Sorting by (expert, pair) is exactly
// the stable grouping of pairs by expert.
constexpr int kWarpUnionMaxP = 128;

// The stage loops are kept rolled (only the four in-lane slots are unrolled):
// this kernel runs once per layer right after the expert FFN has streamed the
// weights through L2, so its code is fetched cold every time and a small code
// footprint matters more than loop overhead.
__device__ __forceinline__ void warp_bitonic_sort128(int (&key)[4], int lane) {
#pragma unroll 1
  for (int k = 2; k <= 128; k <<= 1) {
#pragma unroll 1
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j >= 4) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int i = lane * 4 + r;
          const int other = __shfl_xor_sync(0xffffffffu, key[r], j >> 2);
          const bool up = (i & k) == 0, lower = (i & j) == 0;
          const int lo = min(key[r], other), hi = max(key[r], other);
          key[r] = (lower == up) ? lo : hi;
        }
      } else {
        // in-lane pairs (r, r ^ j), each updated once from its lower slot
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int i = lane * 4 + r;
          const bool up = (i & k) == 0, lower = (i & j) == 0;
          if (lower) {
            const int rr = r ^ j;
            int a = key[r], b = j == 1 ? key[r ^ 1] : key[r ^ 2];
            const int lo = min(a, b), hi = max(a, b);
            a = up ? lo : hi;
            b = up ? hi : lo;
            key[r] = a;
            if (rr == (r ^ 1) && j == 1) key[r ^ 1] = b;
            else key[r ^ 2] = b;
          }
        }
      }
    }
  }
}

// ids: T*k routed experts (shared memory); writes the union outputs, the plan
// and zeroes the FFN counters (when tb_done / rb_done are not NULL), like
// block_union + block_plan.  Called by one warp; the outputs may be in global
// or shared memory.
__device__ __forceinline__ void warp_union_plan(const int* ids, int P, int E, int T, int S, int tokb,
                                                int32_t* __restrict__ unique_ids, int32_t* __restrict__ n_unique,
                                                int32_t* __restrict__ seg_off, int32_t* __restrict__ perm,
                                                int32_t* __restrict__ pair_pos, uint32_t* __restrict__ status,
                                                int32_t* __restrict__ plan, int32_t* __restrict__ tb_done,
                                                int32_t* __restrict__ rb_done, int n_rb, int lane, int eb, int ee) {
  int key[4];
  bool bad = false;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int p = lane * 4 + r;
    key[r] = 0x7fffffff;
    if (p < P) {
      const int e = ids[p];
      if (e < 0 || e >= E) bad = true;
      else key[r] = (e << 8) | p;
      pair_pos[p] = -1;
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0 && status) atomicOr(status, COLI_FLAG_BAD_ID);
  warp_bitonic_sort128(key, lane);
  // segment starts: a valid key whose expert differs from the previous key's
  const int prev_last = __shfl_up_sync(0xffffffffu, key[3], 1);
  int flags = 0, nvalid = 0;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const bool valid = key[r] != 0x7fffffff;
    const int prev = (r == 0) ? (lane == 0 ? -1 : prev_last) : key[r - 1];
    const bool start = valid && (prev == -1 || (prev >> 8) != (key[r] >> 8));
    flags |= (start ? 1 : 0) << r;
    nvalid += valid ? 1 : 0;
  }
  int cnt = __popc(flags), incl = cnt, vincl = nvalid;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, incl, o), b = __shfl_up_sync(0xffffffffu, vincl, o);
    if (lane >= o) {
      incl += a;
      vincl += b;
    }
  }
  const int U = __shfl_sync(0xffffffffu, incl, 31);
  const int Pv = __shfl_sync(0xffffffffu, vincl, 31);
  int u = incl - cnt;
  __syncwarp();
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = lane * 4 + r;
    if (key[r] != 0x7fffffff) {
      const int p = key[r] & 0xff;
      perm[i] = p;
      pair_pos[p] = i;
      if (flags & (1 << r)) {
        unique_ids[u] = key[r] >> 8;
        seg_off[u] = i;
        ++u;
      }
    }
  }
  if (lane == 0) {
    *n_unique = U;
    seg_off[U] = Pv;
  }
  __syncwarp();
  // plan over S shared segments then U routed ones (U <= 128, S <= 4)
  int nb[5], lsum = 0;
#pragma unroll
  for (int q = 0; q < 5; ++q) {
    const int sidx = lane * 5 + q;
    int v = 0;
    if (sidx < S) {
      v = (T + tokb - 1) / tokb;
    } else if (sidx < S + U) {
      // routed segments of experts outside [eb, ee) get no blocks (an expert-parallel
      // rank computes its own experts only)
      const int uu = sidx - S;
      const int c = ((uu + 1 < U) ? seg_off[uu + 1] : Pv) - seg_off[uu];
      const int eid = unique_ids[uu];
      v = (eid >= eb && eid < ee) ? (c + tokb - 1) / tokb : 0;
    }
    nb[q] = v;
    lsum += v;
  }
  int lincl = lsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, lincl, o);
    if (lane >= o) lincl += a;
  }
  const int total = __shfl_sync(0xffffffffu, lincl, 31);
  int run = lincl - lsum;
  const int n_seg = U + S;
#pragma unroll
  for (int q = 0; q < 5; ++q) {
    const int sidx = lane * 5 + q;
    if (sidx < n_seg) plan[2 + sidx] = run;
    run += nb[q];
  }
  if (lane == 0) {
    plan[0] = n_seg;
    plan[1] = total;
    plan[2 + n_seg] = total;
  }
  if (tb_done)
    for (int i = lane; i < total; i += 32) tb_done[i] = 0;
  if (rb_done)
    for (int i = lane; i < n_rb; i += 32) rb_done[i] = 0;
}

// The same for T*k <= 32, one key per lane: a 32-wide bitonic sort (15
// shuffle stages), segment starts by ballot, and the plan's per-segment block
// counts from the distance to the next segment start -- no global reads back.
__device__ __forceinline__ void warp_union_plan32(const int* ids, int P, int E, int T, int S, int tokb,
                                                  int32_t* __restrict__ unique_ids, int32_t* __restrict__ n_unique,
                                                  int32_t* __restrict__ seg_off, int32_t* __restrict__ perm,
                                                  int32_t* __restrict__ pair_pos, uint32_t* __restrict__ status,
                                                  int32_t* __restrict__ plan, int32_t* __restrict__ tb_done,
                                                  int32_t* __restrict__ rb_done, int n_rb, int lane, int eb, int ee) {
  int key = 0x7fffffff;
  bool bad = false;
  if (lane < P) {
    const int e = ids[lane];
    if (e < 0 || e >= E) bad = true;
    else key = (e << 8) | lane;
    pair_pos[lane] = -1;
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0 && status) atomicOr(status, COLI_FLAG_BAD_ID);
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const int other = __shfl_xor_sync(0xffffffffu, key, j);
      const bool up = (lane & k) == 0, lower = (lane & j) == 0;
      key = (lower == up) ? min(key, other) : max(key, other);
    }
  }
  const bool valid = key != 0x7fffffff;
  const int prev = __shfl_up_sync(0xffffffffu, key, 1);
  const bool start = valid && (lane == 0 || (prev >> 8) != (key >> 8));
  const uint32_t smask = __ballot_sync(0xffffffffu, start);
  const int Pv = __popc(__ballot_sync(0xffffffffu, valid));
  const int U = __popc(smask);
  const int u = __popc(smask & ((1u << lane) - 1u));
  // pairs of the segment starting here: up to the next start (or the end)
  const uint32_t later = lane == 31 ? 0u : (smask & ~((2u << lane) - 1u));
  const int cnt = start ? (later ? __ffs(later) - 1 : Pv) - lane : 0;
  __syncwarp();   // the -1 stores above come before the pair_pos stores below
  if (valid) {
    const int p = key & 0xff;
    perm[lane] = p;
    pair_pos[p] = lane;
    if (start) {
      unique_ids[u] = key >> 8;
      seg_off[u] = lane;
    }
  }
  // plan: S shared segments of T tokens, then the U routed ones in order
  const int nb_shared = (T + tokb - 1) / tokb;
  // (routed segments of experts outside [eb, ee) get no blocks)
  int nb = (start && (key >> 8) >= eb && (key >> 8) < ee) ? (cnt + tokb - 1) / tokb : 0;
  int incl = nb;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += a;
  }
  const int routed_total = __shfl_sync(0xffffffffu, incl, 31);
  const int total = S * nb_shared + routed_total;
  const int n_seg = U + S;
  if (start) plan[2 + S + u] = S * nb_shared + incl - nb;
  if (lane < S) plan[2 + lane] = lane * nb_shared;
  if (lane == 0) {
    *n_unique = U;
    seg_off[U] = Pv;
    plan[0] = n_seg;
    plan[1] = total;
    plan[2 + n_seg] = total;
  }
  if (tb_done)
    for (int i = lane; i < total; i += 32) tb_done[i] = 0;
  if (rb_done)
    for (int i = lane; i < n_rb; i += 32) rb_done[i] = 0;
}

// Route + union + plan for T*k <= 128: warp w routes tokens w, w + nwarps, ...;
// then warp 0 alone builds the union and the plan.  The union covers every
// selected expert; the plan gives blocks to the S shared segments and to the
// routed experts in [eb, ee) only (the whole range [0, E) except on an
// expert-parallel rank).
template <int NV>
__global__ void __launch_bounds__(256) route_union_small_kernel(
    const float* __restrict__ logits, const float* __restrict__ bias, int T, int E, int k,
    int32_t* __restrict__ ids_out, float* __restrict__ w_out, int32_t* __restrict__ unique_ids,
    int32_t* __restrict__ n_unique, int32_t* __restrict__ seg_off, int32_t* __restrict__ perm,
    int32_t* __restrict__ pair_pos, uint32_t* __restrict__ status, int S, int tokb, int32_t* __restrict__ plan,
    int32_t* __restrict__ tb_done, int32_t* __restrict__ rb_done, int n_rb, int eb, int ee) {
  __shared__ int ids_s[kWarpUnionMaxP];
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int t = warp; t < T; t += nwarps) {
    int id;
    float w;
    const bool bad = route_token<NV>(logits + static_cast<size_t>(t) * E, bias, E, k, lane, &id, &w);
    if (lane < k) {
      ids_s[t * k + lane] = id;
      ids_out[static_cast<size_t>(t) * k + lane] = id;
      w_out[static_cast<size_t>(t) * k + lane] = w;
    }
    if (bad && lane == 0) atomicOr(status, COLI_FLAG_NONFINITE);
  }
  if (nwarps > 1) __syncthreads();
  else __syncwarp();
  if (warp == 0) {
    if (T * k <= 32)
      warp_union_plan32(ids_s, T * k, E, T, S, tokb, unique_ids, n_unique, seg_off, perm, pair_pos, status, plan,
                        tb_done, rb_done, n_rb, lane, eb, ee);
    else
      warp_union_plan(ids_s, T * k, E, T, S, tokb, unique_ids, n_unique, seg_off, perm, pair_pos, status, plan,
                      tb_done, rb_done, n_rb, lane, eb, ee);
  }
}

}  // namespace coli
