// Union step: batch-union of the experts a batch selected (Colibri README,
// "Mai aspettare il disco due volte": positions of a batch read each unique
// expert once; getting-started guide, "2. Union": duplicates removed when
// several tokens of a batch pick the same expert), plus the FFN tile plan.
#pragma once
#include "common.cuh"

namespace coli {

constexpr int kUnionThreads = 1024;
constexpr int kUnionWarps = kUnionThreads / 32;

// Stable counting sort of the pairs p = t*k + j by expert id, in one CTA and
// without atomics.  Warp w owns the contiguous pair range [w*C, (w+1)*C).
//  1. Each warp builds its private histogram hist[w][e]: lanes holding the
//     same id are grouped with __match_any_sync and the group's lowest lane
//     adds the group size (one writer per bin per step).
//  2. Thread e turns column e into per-warp running offsets; a block scan
//     over the per-expert totals gives each expert's segment start; experts
//     with a non-zero count are compacted into unique_ids / seg_off.
//  3. Each warp walks its range again in the same order and writes
//     perm[pos] = p, pair_pos[p] = pos with pos = its (expert, warp) base +
//     rank among earlier equal ids, so equal ids keep pair order.
// Dynamic shared memory: kUnionWarps * E ints.
__global__ void __launch_bounds__(kUnionThreads, 1)
    union_kernel(const int32_t* __restrict__ ids, int P, int E, int32_t* __restrict__ unique_ids,
                 int32_t* __restrict__ n_unique, int32_t* __restrict__ seg_off, int32_t* __restrict__ perm,
                 int32_t* __restrict__ pair_pos, uint32_t* __restrict__ status) {
  extern __shared__ int hist[];  // [kUnionWarps][E]
  __shared__ int scratch[33];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kUnionWarps * E; i += blockDim.x) hist[i] = 0;
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
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, COLI_FLAG_BAD_ID);
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
    // carry from earlier chunks of experts
    __shared__ int carry_pairs, carry_u;
    if (e0 == 0 && threadIdx.x == 0) {
      carry_pairs = 0;
      carry_u = 0;
    }
    __syncthreads();
    const int cp = carry_pairs, cu = carry_u;
    if (e < E) {
      for (int w = 0; w < kUnionWarps; ++w) hist[w * E + e] += cp + off;
      if (cnt > 0) {
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
    if (e0 + (int)blockDim.x >= E && threadIdx.x == 0) {
      *n_unique = carry_u;
      seg_off[carry_u] = carry_pairs;
    }
  }
  __syncthreads();

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
}

// FFN tile plan, one CTA.  Segments are the U unique routed experts followed
// by the S shared experts (every token, weight 1).  Segment u is cut into
// token blocks of kTokBlock; plan = [n_seg, total_blocks, tile_off[0..n_seg]]
// with tile_off the exclusive prefix of the blocks per segment.
constexpr int kTokBlock = 64;

__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ n_unique,
                                                    const int32_t* __restrict__ seg_off, int T, int S,
                                                    int32_t* __restrict__ plan) {
  __shared__ int scratch[33];
  __shared__ int carry;
  const int U = *n_unique;
  const int n_seg = U + S;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int u0 = 0; u0 < n_seg; u0 += blockDim.x) {
    const int u = u0 + threadIdx.x;
    int nb = 0;
    if (u < U) {
      nb = (seg_off[u + 1] - seg_off[u] + kTokBlock - 1) / kTokBlock;
    } else if (u < n_seg) {
      nb = (T + kTokBlock - 1) / kTokBlock;
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
}

}  // namespace coli
