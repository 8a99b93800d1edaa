// Host-RAM expert tier: placement of a batch's experts in device slots, the
// usage counts that steer it, and the copies of the misses from host memory.
//
// Colibri README, "Una gerarchia di memoria, non un requisito di memoria" and
// "Mai aspettare il disco due volte"; getting-started guide, the per-token path,
// steps 3-5 (Place, Overlap, Learn): where an expert is read from changes the
// speed only, never the routing or the weights' precision; misses are loaded
// while resident experts compute; the engine records which experts the
// workload routes to and keeps the hottest resident.
#pragma once
#include "common.cuh"

namespace coli {

// The tier's device state (int32 words), in this order: slot_of[E], owner[C],
// usage[E], last[C], counters[4] (calls, hits, misses, fills), n_fill,
// fill_e[C], fill_s[C].
struct TierState {
  int32_t* slot_of;
  int32_t* owner;
  uint32_t* usage;
  uint32_t* last;
  uint32_t* ctr;
  int32_t* n_fill;
  int32_t* fill_e;
  int32_t* fill_s;
};

__host__ __device__ inline size_t tier_state_words(int E, int C) {
  return static_cast<size_t>(E) * 2 + static_cast<size_t>(C) * 4 + 5;
}

__host__ __device__ inline TierState tier_state(void* base, int E, int C) {
  int32_t* p = static_cast<int32_t*>(base);
  TierState t;
  t.slot_of = p;
  t.owner = p + E;
  t.usage = reinterpret_cast<uint32_t*>(p + E + C);
  t.last = reinterpret_cast<uint32_t*>(p + 2 * E + C);
  t.ctr = reinterpret_cast<uint32_t*>(p + 2 * E + 2 * C);
  t.n_fill = p + 2 * E + 2 * C + 4;
  t.fill_e = p + 2 * E + 2 * C + 5;
  t.fill_s = p + 2 * E + 3 * C + 5;
  return t;
}

__global__ void __launch_bounds__(256) tier_reset_kernel(void* state, int E, int C) {
  const TierState t = tier_state(state, E, C);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < E; i += gridDim.x * blockDim.x) {
    t.slot_of[i] = -1;
    t.usage[i] = 0;
  }
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < C; i += gridDim.x * blockDim.x) {
    t.owner[i] = -1;
    t.last[i] = 0;
  }
  if (blockIdx.x == 0 && threadIdx.x < 5) t.ctr[threadIdx.x] = 0;   // counters and n_fill
}

// Eviction order of slot c (smaller goes first): empty slots, then the slot
// whose expert was routed least often, then the least recently used; ties to
// the lower slot index (the caller compares indices).
__device__ __forceinline__ uint64_t tier_key(const TierState& t, int c) {
  const int e = t.owner[c];
  if (e < 0) return 0ull;
  const uint32_t u = t.usage[e];
  return (1ull << 63) | (static_cast<uint64_t>(u > 0x7fffffffu ? 0x7fffffffu : u) << 32) | t.last[c];
}

// Place experts ids[0..n) in one block of 256 threads.  A layer call passes
// seg_off (and n_ptr: n is the union's size on the device): the ids are a
// union, each distinct, and seg_off gives each one's routed pairs, added to
// usage after placement; slot_ids[u] receives the slot of ids[u].  A prefetch
// passes neither: ids may repeat and nothing is counted.  Ids outside [0, E)
// set COLI_FLAG_BAD_ID and are skipped.  Each call's slots are stamped with the
// call count so that no slot is evicted by the call that uses it; the caller
// guarantees at most C distinct ids (an id left without a slot would also set
// COLI_FLAG_BAD_ID and map to slot 0, so that no access goes astray).
__global__ void __launch_bounds__(256) tier_place_kernel(const int32_t* __restrict__ ids, int n,
                                                         const int32_t* __restrict__ n_ptr,
                                                         const int32_t* __restrict__ seg_off, int E, int C,
                                                         void* state, int32_t* __restrict__ slot_ids,
                                                         uint32_t* __restrict__ status) {
  pdl_wait();
  pdl_trigger();
  const TierState t = tier_state(state, E, C);
  __shared__ uint32_t s_clock;
  __shared__ uint64_t s_key[8];
  __shared__ int s_idx[8];
  __shared__ int s_misses;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (n_ptr) n = *n_ptr;
  if (tid == 0) {
    s_clock = ++t.ctr[0];
    s_misses = 0;
  }
  __syncthreads();
  const uint32_t clock = s_clock;
  // hits first: stamp their slots so that no miss of this call evicts them
  for (int u = tid; u < n; u += blockDim.x) {
    const int e = ids[u];
    if (e < 0 || e >= E) {
      atomicOr(status, COLI_FLAG_BAD_ID);
      if (slot_ids) slot_ids[u] = 0;   // a valid slot: the output is wrong (flagged), no access goes astray
      continue;
    }
    const int s = t.slot_of[e];
    if (s >= 0) t.last[s] = clock;
  }
  __syncthreads();
  // misses in list order, each into the first slot of the eviction order
  for (int u = 0; u < n; ++u) {
    const int e = ids[u];
    if (e < 0 || e >= E || t.slot_of[e] >= 0) continue;   // uniform: every thread reads the same words
    uint64_t bk = ~0ull;
    int bc = 0x7fffffff;
    for (int c = tid; c < C; c += blockDim.x) {
      if (t.last[c] == clock && t.owner[c] >= 0) continue;   // used by this call
      const uint64_t k = tier_key(t, c);
      if (k < bk || (k == bk && c < bc)) {
        bk = k;
        bc = c;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint64_t ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oc = __shfl_xor_sync(0xffffffffu, bc, o);
      if (ok < bk || (ok == bk && oc < bc)) {
        bk = ok;
        bc = oc;
      }
    }
    if (lane == 0) {
      s_key[warp] = bk;
      s_idx[warp] = bc;
    }
    __syncthreads();
    if (tid == 0) {
      for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w)
        if (s_key[w] < bk || (s_key[w] == bk && s_idx[w] < bc)) {
          bk = s_key[w];
          bc = s_idx[w];
        }
      if (bc < C) {
        const int old = t.owner[bc];
        if (old >= 0) t.slot_of[old] = -1;
        t.owner[bc] = e;
        t.slot_of[e] = bc;
        t.last[bc] = clock;
        t.fill_e[s_misses] = e;
        t.fill_s[s_misses] = bc;
        ++s_misses;
      }
    }
    __syncthreads();
  }
  if (tid == 0) {
    *t.n_fill = s_misses;
    t.ctr[3] += s_misses;
    if (seg_off) {
      t.ctr[1] += n - s_misses;
      t.ctr[2] += s_misses;
    }
  }
  if (seg_off) {
    for (int u = tid; u < n; u += blockDim.x) {
      const int e = ids[u];
      if (e < 0 || e >= E) continue;
      t.usage[e] += static_cast<uint32_t>(seg_off[u + 1] - seg_off[u]);
      const int sl = t.slot_of[e];
      if (sl < 0) atomicOr(status, COLI_FLAG_BAD_ID);
      if (slot_ids) slot_ids[u] = sl >= 0 ? sl : 0;
    }
  }
}

// The host-memory sources and device slots of one expert matrix kind.
struct TierCopy {
  const uint4* src[6];   // host: gate q, up q, down q, gate s, up s, down s (expert-major)
  uint4* dst[6];         // device slots, same layouts
  long per[6];           // 16-byte chunks per expert
};

// Copies the experts placed by tier_place_kernel (fill list in the state)
// from page-locked host memory into their slots: every CTA strides over all
// chunks of all listed experts, loads before stores.
__global__ void __launch_bounds__(256) tier_fill_kernel(const __grid_constant__ TierCopy cp, void* state, int E,
                                                        int C) {
  pdl_wait();
  pdl_trigger();
  const TierState t = tier_state(state, E, C);
  const int nf = *t.n_fill;
  const long stride = static_cast<long>(gridDim.x) * blockDim.x;
  for (int f = 0; f < nf; ++f) {
    const long e = t.fill_e[f], s = t.fill_s[f];
#pragma unroll 1
    for (int m = 0; m < 6; ++m) {
      const long per = cp.per[m];
      const uint4* src = cp.src[m] + e * per;
      uint4* dst = cp.dst[m] + s * per;
      long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x;
      for (; i + 3 * stride < per; i += 4 * stride) {
        const uint4 v0 = src[i], v1 = src[i + stride], v2 = src[i + 2 * stride], v3 = src[i + 3 * stride];
        dst[i] = v0;
        dst[i + stride] = v1;
        dst[i + 2 * stride] = v2;
        dst[i + 3 * stride] = v3;
      }
      for (; i < per; i += stride) dst[i] = src[i];
    }
  }
}

}  // namespace coli
