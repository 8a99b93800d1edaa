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
                                           int32_t* __restrict__ rb_done, int n_rb) {
  __shared__ int carry;
  const int n_seg = U + S;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int u0 = 0; u0 < n_seg; u0 += blockDim.x) {
    const int u = u0 + threadIdx.x;
    int nb = 0;
    if (u < S) nb = (T + tokb - 1) / tokb;
    else if (u < n_seg) nb = (seg_cnt[u - S] + tokb - 1) / tokb;
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
                       int n_rb) {
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
  block_plan(U, seg_cnt, T, S, tokb, scratch, plan, tb_done, rb_done, n_rb);
}

}  // namespace coli
