// Device helpers shared by the kernels of libcolimoe: shared-memory barriers,
// bulk/tensor copies, bounded waits and the device status word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "coli_moe.h"

namespace coli {

// Every wait on a barrier gives up after this long (ns of %globaltimer), sets
// COLI_FLAG_TIMEOUT and lets the kernel return instead of hanging the GPU.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed.  Returns false
// (and leaves the barrier alone) if `abort_flag` was raised by another warp or
// if the wait ran past limit_ns (kWaitLimitNs unless a test passes a shorter
// limit), in which case it raises `abort_flag` and sets COLI_FLAG_TIMEOUT in
// the status word.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit_ns) {
        atomicOr(status, COLI_FLAG_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// 2-D tiled TMA load (no multicast) into this CTA's shared memory, completing
// `bytes` on `bar`.  x is the innermost coordinate (in elements of the map).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t x,
                                            int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y)
      : "memory");
}

// L2 cache policies (createpolicy): data read once and not shared with other
// CTAs goes in with evict_first, so that it does not push out what the kernel
// reads again later; data written now and read back at the end of the kernel
// goes in with evict_last.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// tma_load_2d with an L2 cache policy.
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t x,
                                                 int32_t y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

// One fp32 store to global memory (L2) with an L2 cache policy.
__device__ __forceinline__ void st_f32_hint(float* p, float v, uint64_t policy) {
  asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(policy) : "memory");
}

// Contiguous bulk copy global -> shared (both 16-byte aligned, bytes % 16 == 0).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Programmatic dependent launch: wait until the preceding kernel in the stream
// has completed and its memory is visible (a no-op when there is none), and
// let the next kernel's CTAs start their prologue.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint16_t lds16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.b16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ float half_bits_to_float(uint16_t b) { return __half2float(__ushort_as_half(b)); }

// fp16 bits of a bf16 value: exact unless |v| < 2^-17 (rounded to fp16's
// subnormal grid) or |v| >= 65536 (infinity; `range` is set).
__device__ __forceinline__ uint16_t bf16_to_f16_bits(uint16_t b, bool& range) {
  const float f = bf16_bits_to_float(b);
  range |= fabsf(f) >= 65536.0f && fabsf(f) != INFINITY;
  return __half_as_ushort(__float2half_rn(f));
}

// The same for eight values in place.
__device__ __forceinline__ void to_f16_8(uint16_t (&e)[8], bool& range) {
#pragma unroll
  for (int q = 0; q < 8; ++q) e[q] = bf16_to_f16_bits(e[q], range);
}

// Position of natural element i (within a row) in the fragment-ordered copy of
// an activation row: every block of 8 elements is stored as
// x0 x4 x1 x5 x2 x6 x3 x7, so that one 16-byte load gives the bf16 pairs
// (x0,x4) (x1,x5) (x2,x6) (x3,x7) that match the nibble pairs a 32-bit code
// word yields under the 0x000F000F mask at shifts 0, 4, 8 and 12.
__device__ __forceinline__ int frag_pos(int i) {
  const int p = i & 7;
  return (i & ~7) | (p < 4 ? 2 * p : 2 * (p - 4) + 1);
}

// ---------------------------------------------------------------------------
// Integer activation planes of the decode form for batches of up to 8 tokens.
//
// The expert input of one token (and each 128-row slice of h of one pair) is
// put on a fixed-point grid of its own: v -> q = rint(v * 2^e), with e the
// power of two that brings the largest |v| into [2^13, 2^14).  Every value
// whose magnitude is at least 2^-6 of that largest one lands on the grid
// exactly (a bf16 value has 8 significant bits); the smaller ones are rounded
// to the nearest grid point, the grid step being at most max|v| * 2^-13.
// |q| < 2^14 is then written as
// two signed bytes, q = 256 * hi + lo with lo in [-128, 127] and hi in
// [-64, 64]: the "low" and "high" planes, the B operands of an integer MMA
// (mma.sync m16n8k32, u8/s8 x s8 -> s32) against the int4 (or int8) codes.
//
// Record of one 32-wide K group of one token: 72 bytes,
//   [0, 32)   low plane, [32, 64) high plane: lane c (0..3) of an MMA quad
//             owns elements 8c .. 8c+7 of the group, stored as the 4 even
//             ones then the 4 odd ones (the order in which an int4 code word
//             of 8 nibbles splits into its low and high nibbles);
//   [64, 72)  two int32: the MMA accumulator's start value for the low and
//             the high column, kPlaneMagic - 8 * (sum of the low plane) and
//             -8 * (sum of the high plane).  The -8 * sum terms cancel the +8
//             that turns a two's-complement int4 code into an unsigned byte;
//             kPlaneMagic (1.5 * 2^23 as an fp32 bit pattern) makes the
//             combined integer 256 * d_hi + d_lo readable as the float
//             1.5 * 2^23 + value, exactly, for |value| < 2^22.
// A token's records for all K follow each other: H / 32 records.
constexpr int kPlaneRec = 72;
constexpr int kPlaneMagic = 0x4B400000;
constexpr float kPlaneMagicF = 12582912.0f;

// floor(log2 m) for a finite m > 0 (subnormals included).
__device__ __forceinline__ int ilog2f(float m) {
  int e2;
  frexpf(m, &e2);
  return e2 - 1;
}

// The grid exponent for a largest magnitude m (0 when m == 0): max|v| * 2^e
// lies in [2^13, 2^14).
__device__ __forceinline__ int plane_exponent(float m) { return m > 0.f ? 13 - ilog2f(m) : 0; }

// 2^k for |k| <= 126.
__device__ __forceinline__ float pow2i(int k) { return __int_as_float((k + 127) << 23); }

// 2^e as two factors (each exact for |e| <= 252).
__device__ __forceinline__ void pow2_split(int e, float& f1, float& f2) {
  const int a = e / 2;
  f1 = pow2i(a);
  f2 = pow2i(e - a);
}

// Eight values v[0..7] (elements 8c .. 8c+7 of a group) on the grid 2^-e
// (factors f1 * f2 = 2^e): the lane's 8 bytes of each plane and its partial
// plane sums.
__device__ __forceinline__ void planes8(const float (&v)[8], float f1, float f2, uint2& lo, uint2& hi, int& slo,
                                        int& shi) {
  int l[8], h[8];
  slo = 0;
  shi = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int q = __float2int_rn((v[i] * f1) * f2);
    l[i] = ((q + 128) & 255) - 128;
    h[i] = (q - l[i]) >> 8;
    slo += l[i];
    shi += h[i];
  }
  auto pack = [](int a, int b, int c, int d) {
    return (static_cast<uint32_t>(a) & 0xffu) | ((static_cast<uint32_t>(b) & 0xffu) << 8) |
           ((static_cast<uint32_t>(c) & 0xffu) << 16) | (static_cast<uint32_t>(d) << 24);
  };
  lo = make_uint2(pack(l[0], l[2], l[4], l[6]), pack(l[1], l[3], l[5], l[7]));
  hi = make_uint2(pack(h[0], h[2], h[4], h[6]), pack(h[1], h[3], h[5], h[7]));
}

// Block-wide exclusive scan of one int per thread (blockDim.x a multiple of 32,
// <= 1024).  `scratch` holds 33 ints.  Returns the exclusive prefix; *total
// receives the sum.  Deterministic.
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int s = lane < nwarps ? scratch[lane] : 0;
    int si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += n;
    }
    if (lane < nwarps) scratch[lane] = si - s;  // exclusive prefix of warp totals
    if (lane == 31) scratch[32] = si;           // grand total
  }
  __syncthreads();
  const int res = scratch[warp] + incl - v;
  *total = scratch[32];
  __syncthreads();
  return res;
}

}  // namespace coli
