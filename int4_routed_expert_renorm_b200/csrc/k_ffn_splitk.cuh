// Split-K decode form of the int4 expert FFN, for batches of at most 8 tokens.
//
// In the two-phase decode kernel (k_ffn_decode.cuh) a down tile needs the
// whole h of its expert, i.e. the gate/up tiles of all 16 row blocks, which
// other CTAs compute: every CTA waits at the switch from gate/up to down, and
// the down projection starts its weight stream anew.  Here the unit of work
// is one gate/up tile -- (expert, token block, 128-row block rb) -- followed
// at once by the same CTA's share of the down projection that uses exactly
// those 128 h values: all H output rows over the K slice [128 rb, 128 rb +
// 128) of W_down.  A CTA never waits on another CTA before its last unit, and
// each unit is one uninterrupted weight stream (gate/up then down, 2/3 and
// 1/3 of the expert's bytes over its 16 units).
//   * gate/up: the stages and consumers of the two-phase kernel; the epilogue
//     writes h = bf16(silu(g) * u) of the tile's 128 rows into a shared-memory
//     slice buffer instead of global memory;
//   * down: stages of 512 output rows x 128 K (four 128-row tensor-map boxes
//     of 64 code bytes per row, 64B swizzle, and the rows' 8-scale boxes);
//     warp w owns stage rows [32 w, 32 w + 32) as two 16-row MMA slices and
//     all 4 groups of the slice, so no K reduction between warps is needed
//     (int8 codes: 256-row stages of two 128-byte-wide boxes, 16 rows a warp);
//     the fp32 result is a partial y per (pair, K slice, row), ypart;
//   * after its last unit every consumer warp fences its partials and checks in
//     on a CTA barrier; one thread per CTA then increments a grid counter;
//     once all CTAs have (a bounded grid-wide wait --
//     the launch is cooperative, so every CTA is resident), each CTA combines
//     a contiguous range of (token, 4 rows): y of every routed and shared
//     pair as the sum of its I/128 partials in a fixed order (four lanes each
//     add every fourth slice in turn, then their sums pairwise), then the
//     routed y's weighted in slot order, the shared y's and the residual,
//     rounded once to bf16.
// Every token's arithmetic is the same whatever else is in the batch (its own
// MMA column, fixed orders everywhere), so the form is batch-invariant.
#pragma once
#include "k_ffn_decode.cuh"

namespace coli {

constexpr int kSkMaxT = 8;                       // largest batch this form takes
constexpr int kSkDnScale = kRowBlock * 16;       // the rows' 16-byte (8-scale) boxes

// BITS 4: gate/up stages of 256 K; down stages of four 128-row boxes of 64
// code bytes per row (64B swizzle).  BITS 8: gate/up stages of 128 K (128 code
// bytes per row); down stages of two 128-row boxes of 128 bytes (128B swizzle).
template <int BITS>
struct SkDn {
  static constexpr int KCG = BITS == 4 ? 256 : 128;      // gate/up stage K
  static constexpr int BOXES = BITS == 4 ? 4 : 2;         // 128-row boxes per down stage
  static constexpr int ROWB = 128 * BITS / 8;             // code bytes per row of a 128-wide K slice
  static constexpr int CODE = kRowBlock * ROWB;           // codes of one box
  static constexpr int ROWS = BOXES * kRowBlock;          // output rows per down stage
  static constexpr int WROWS = ROWS / kFfnConsumerWarps;  // rows per consumer warp (32 or 16)
};

template <int GROUP, int BITS = 4>
struct SkCfg {
  using D = SkDn<BITS>;
  using GU = StageCfg<D::KCG, 1, 2, GROUP, BITS>;
  static constexpr int DN_USED = D::BOXES * (D::CODE + kSkDnScale);
  static constexpr int STAGE = ((GU::STAGE_USED > DN_USED ? GU::STAGE_USED : DN_USED) + 1023) / 1024 * 1024;
  static constexpr int RED_BYTES = kRowWarps * 32 * 4 * 2 * 4;   // K-half partials of both matrices
  static constexpr int META_BYTES = (3 * kMaxSeg + 4) * 4;
  static constexpr int H_BYTES = kSkMaxT * kSkHRow;
  static constexpr int NBAR = 64;
  static constexpr int FIXED = RED_BYTES + META_BYTES + H_BYTES + 1024 + NBAR * 8 + 64;
  static constexpr int NS_RAW = (227 * 1024 - FIXED) / STAGE;
  static constexpr int NS = NS_RAW > 8 ? 8 : NS_RAW;
  static constexpr size_t SMEM = static_cast<size_t>(NS) * STAGE + FIXED;
  static_assert(NS >= 3, "pipeline depth");
  static_assert(2 * NS + 2 * kRowWarps + 4 <= NBAR, "barrier slots");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(D::CODE % 1024 == 0, "swizzled boxes need 1 KiB alignment");
  static_assert(H_BYTES >= kSkMaxT * 32 * 8, "the combine's pair_pos / topk_w copies fit in the h buffer");
};

// Producer: the down stages of one unit (K slice rb of expert e, every output
// row).  Returns false on a timeout.
template <int NS, int STAGE, int GROUP, int BITS>
__device__ __forceinline__ bool produce_down_slice(const FfnArgs& a, const TileInfo& ti, const CUtensorMap* dq,
                                                   const CUtensorMap* ds, uint8_t* smem, uint64_t* full,
                                                   uint64_t* empty, int& s, uint32_t& ph, long& issued,
                                                   volatile int* abort_flag, int lane) {
  using D = SkDn<BITS>;
  const int nst = (a.H + D::ROWS - 1) / D::ROWS;
  const int sx = ((ti.rb * kRowBlock) / GROUP) & ~7;   // the slice's first scale, rounded down to its box
  const int rbase = ti.e * a.H;
  for (int st = 0; st < nst; ++st) {
    bool ok = true;
    if (lane == 0) ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, a.status);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) return false;
    if (lane == 0) {
      const int r0 = st * D::ROWS;
      const int rem = (a.H - r0) / kRowBlock;
      const int nb = rem < D::BOXES ? rem : D::BOXES;
      uint8_t* stg = smem + s * STAGE;
      mbar_arrive_expect_tx(&full[s], nb * (D::CODE + kSkDnScale));
      for (int b = 0; b < nb; ++b) {
        tma_load_2d(stg + b * D::CODE, dq, &full[s], ti.rb * D::ROWB, rbase + r0 + b * kRowBlock);
        tma_load_2d(stg + D::BOXES * D::CODE + b * kSkDnScale, ds, &full[s], sx, rbase + r0 + b * kRowBlock);
      }
    }
    __syncwarp();
    ++issued;
    if (++s == NS) {
      s = 0;
      ph ^= 1u;
    }
  }
  return true;
}

// Consumers: the down stages of one unit, B operand = the unit's h slice in
// shared memory.  Writes ypart[pair][rb][row].  Returns false on a timeout.
template <bool SINGLE, int NS, int STAGE, int GROUP, int BITS>
__device__ __forceinline__ bool consume_down_slice(const FfnArgs& a, const TileInfo& ti, const uint8_t* smem,
                                                   const uint16_t* hbuf, uint64_t* full, uint64_t* empty,
                                                   uint64_t* h_ready, uint64_t* h_free, int& s, uint32_t& ph,
                                                   uint32_t lu, volatile int* abort_flag, int warp, int lane) {
  const int g = lane >> 2, c = lane & 3;
  if (!mbar_wait(h_ready, lu & 1u, abort_flag, a.status)) return false;
  // B fragments of the slice's four 32-wide groups for token g of the block
  uint4 b[4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
    b[j] = g < ti.ntok ? *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(hbuf) + g * kSkHRow +
                                                          (j * 32 + 8 * c) * 2)
                       : make_uint4(0u, 0u, 0u, 0u);
  using D = SkDn<BITS>;
  const int soff = ((ti.rb * kRowBlock) / GROUP) & 7;   // the slice's first scale within its box
  const int nst = (a.H + D::ROWS - 1) / D::ROWS;
  for (int st = 0; st < nst; ++st) {
    if (!mbar_wait(&full[s], ph, abort_flag, a.status)) return false;
    const uint8_t* stg = smem + s * STAGE;
    const int r0 = st * D::ROWS;
    if (D::WROWS * warp < a.H - r0) {
#pragma unroll
      for (int sl = 0; sl < D::WROWS / 16; ++sl) {
        const int rl = D::WROWS * warp + 16 * sl + g;    // stage-local rows rl and rl + 8
        const int bx = rl >> 7, rr = rl & 127;
        // int4, 64B swizzle: 16-byte chunk j of box row rr sits at chunk j ^ ((rr >> 1) & 3);
        // int8, 128B swizzle: thread c's 8 bytes of group j are chunk (2j + (c >> 1)) ^ (rr & 7)
        const uint8_t* cb = stg + bx * D::CODE + rr * 64 + 4 * c;   // int4
        // int8: offset of thread c's word pair of group 0 within the (1 KiB-aligned) box
        const uint32_t cb8 = rr * 128 + (((rr & 7) ^ (c >> 1)) << 4) + 8 * (c & 1);
        const uint32_t sw = (rr >> 1) & 3;
        const uint8_t* sp = stg + D::BOXES * D::CODE + bx * kSkDnScale + rr * 16 + soff * 2;
        float s0[4], s1[4];
        if (GROUP == 32) {
          const uint2 v0 = *reinterpret_cast<const uint2*>(sp);
          const uint2 v1 = *reinterpret_cast<const uint2*>(sp + 8 * 16);
          const __half2 a0 = u32_as_half2(v0.x), a1 = u32_as_half2(v0.y);
          const __half2 c0 = u32_as_half2(v1.x), c1 = u32_as_half2(v1.y);
          s0[0] = __low2float(a0); s0[1] = __high2float(a0); s0[2] = __low2float(a1); s0[3] = __high2float(a1);
          s1[0] = __low2float(c0); s1[1] = __high2float(c0); s1[2] = __low2float(c1); s1[3] = __high2float(c1);
        } else {
          const __half2 a0 = u32_as_half2(*reinterpret_cast<const uint32_t*>(sp));
          const __half2 c0 = u32_as_half2(*reinterpret_cast<const uint32_t*>(sp + 8 * 16));
          s0[0] = s0[1] = __low2float(a0);
          s0[2] = s0[3] = __high2float(a0);
          s1[0] = s1[1] = __low2float(c0);
          s1[2] = s1[3] = __high2float(c0);
        }
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (BITS == 4) {
            const uint8_t* ca = cb + ((static_cast<uint32_t>(j) ^ sw) << 4);
            const uint32_t w0 = *reinterpret_cast<const uint32_t*>(ca);
            const uint32_t w1 = *reinterpret_cast<const uint32_t*>(ca + 8 * 64);
            uint32_t p[8];
            dq_word_pair(p, w0, w1);
            group_acc<SINGLE>(acc, p, b[j], s0[j], s1[j]);
          } else {
            const uint8_t* ca = stg + bx * D::CODE + (cb8 ^ static_cast<uint32_t>((2 * j) << 4));
            uint32_t h0[4], h1[4], l0[4], l1[4];
            dq8_row(h0, l0, *reinterpret_cast<const uint2*>(ca));
            dq8_row(h1, l1, *reinterpret_cast<const uint2*>(ca + 8 * 128));
            group_acc8<SINGLE>(acc, h0, h1, l0, l1, b[j], s0[j], s1[j]);
          }
        }
        // acc: (row rl, token 2c), (rl, 2c+1), (rl+8, 2c), (rl+8, 2c+1)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = 2 * c + (q & 1);
          if (i < ti.ntok && !(SINGLE && (q & 1))) {
            const size_t orow = static_cast<size_t>(ti.base + ti.i0 + i);
            const int r = r0 + rl + ((q & 2) ? 8 : 0);
            __stcg(a.ypart + (orow * a.I / kRowBlock + ti.rb) * a.H + r, acc[q]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (++s == NS) {
      s = 0;
      ph ^= 1u;
    }
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(h_free);
  return true;
}

// Bounded wait of one lane for a global counter to reach `target`.
__device__ __forceinline__ bool wait_counter(const int32_t* cnt, int target, volatile int* abort_flag,
                                             uint32_t* status) {
  if (ld_acquire_gpu(cnt) >= target) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (ld_acquire_gpu(cnt) >= target) return true;
    if ((it & 63u) == 0 && (*abort_flag || globaltimer() - t0 > kWaitLimitNs)) {
      if (!*abort_flag) atomicOr(status, COLI_FLAG_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

// The CTA's share of the output after every partial is in: see the file
// comment.  pos_s / w_s are shared-memory copies of pair_pos and topk_w
// (T*k each, made before the grid-wide wait); the idle stage ring holds the
// per-pair sums.  `cbar` (count: consumer warps) separates the two passes;
// returns false on a timeout.
__device__ __forceinline__ bool splitk_combine(const FfnArgs& a, const int32_t* pos_s, const float* w_s,
                                               uint8_t* ring, int ring_bytes, uint64_t* cbar, uint32_t& cph,
                                               volatile int* abort_flag, int warp, int lane) {
  const int tid = warp * 32 + lane;
  const int nthr = kFfnConsumerWarps * 32;
  const int q4 = a.H / 4;
  const long units = static_cast<long>(a.T) * q4;
  const int u0 = static_cast<int>(units * blockIdx.x / gridDim.x);
  const int u1 = static_cast<int>(units * (blockIdx.x + 1) / gridDim.x);
  const int nj = a.k + a.S;
  const int nsl = a.I / kRowBlock;
  const int ch = ring_bytes / (nj * 16);
  float4* ysum = reinterpret_cast<float4*>(ring);
  for (int cu = u0; cu < u1; cu += ch) {
    const int cn = (u1 - cu) < ch ? (u1 - cu) : ch;
    // this thread's output unit of the second pass: its residual load goes
    // out now and lands while the first pass runs
    uint2 rv = make_uint2(0u, 0u);
    if (a.residual && tid < cn) {
      const int u = cu + tid;
      const int t = u / q4, r = (u - t * q4) * 4;
      rv = __ldg(reinterpret_cast<const uint2*>(a.residual + static_cast<size_t>(t) * a.H + r));
    }
    // y of one (token, 4 rows, pair) by a quad of lanes: lane p sums the
    // slices p, p+4, ... in order, then the quad adds (p0 + p1) + (p2 + p3)
    // (every lane ends with the same bits: each add is commutative); two
    // tasks per quad and round keep 8 loads in flight per lane
    for (int t0 = warp * 16; t0 < cn * nj; t0 += kFfnConsumerWarps * 16) {
      float4 y[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int task = t0 + 8 * h + (lane >> 2), p = lane & 3;
        y[h] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (task < cn * nj) {
          const int ui = task / nj, jj = task - ui * nj;
          const int u = cu + ui;
          const int t = u / q4, r = (u - t * q4) * 4;
          const int row = jj < a.k ? pos_s[t * a.k + jj] : a.P + (jj - a.k) * a.T + t;
          const float* src = a.ypart + static_cast<size_t>(row) * nsl * a.H + r;
#pragma unroll 4
          for (int sl = p; sl < nsl; sl += 4) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(src + static_cast<size_t>(sl) * a.H));
            y[h].x += v.x;
            y[h].y += v.y;
            y[h].z += v.z;
            y[h].w += v.w;
          }
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int m = 1; m <= 2; m <<= 1) {
          y[h].x += __shfl_xor_sync(0xffffffffu, y[h].x, m);
          y[h].y += __shfl_xor_sync(0xffffffffu, y[h].y, m);
          y[h].z += __shfl_xor_sync(0xffffffffu, y[h].z, m);
          y[h].w += __shfl_xor_sync(0xffffffffu, y[h].w, m);
        }
        const int task = t0 + 8 * h + (lane >> 2);
        if ((lane & 3) == 0 && task < cn * nj) ysum[task] = y[h];
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(cbar);
    if (!mbar_wait(cbar, cph, abort_flag, a.status)) return false;
    cph ^= 1u;
    for (int ui = tid; ui < cn; ui += nthr) {
      const int u = cu + ui;
      const int t = u / q4, r = (u - t * q4) * 4;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j = 0; j < a.k; ++j) {
        const float w = w_s[t * a.k + j];
        const float4 y = ysum[ui * nj + j];
        acc.x = fmaf(w, y.x, acc.x);
        acc.y = fmaf(w, y.y, acc.y);
        acc.z = fmaf(w, y.z, acc.z);
        acc.w = fmaf(w, y.w, acc.w);
      }
      for (int s = 0; s < a.S; ++s) {
        const float4 y = ysum[ui * nj + a.k + s];
        acc.x += y.x;
        acc.y += y.y;
        acc.z += y.z;
        acc.w += y.w;
      }
      if (a.residual) {
        if (ui != tid)
          rv = __ldg(reinterpret_cast<const uint2*>(a.residual + static_cast<size_t>(t) * a.H + r));
        acc.x += __uint_as_float(rv.x << 16);
        acc.y += __uint_as_float(rv.x & 0xffff0000u);
        acc.z += __uint_as_float(rv.y << 16);
        acc.w += __uint_as_float(rv.y & 0xffff0000u);
      }
      uint2 o;
      o.x = float_to_bf16_bits(acc.x) | (static_cast<uint32_t>(float_to_bf16_bits(acc.y)) << 16);
      o.y = float_to_bf16_bits(acc.z) | (static_cast<uint32_t>(float_to_bf16_bits(acc.w)) << 16);
      *reinterpret_cast<uint2*>(a.out + static_cast<size_t>(t) * a.H + r) = o;
    }
    // the next chunk overwrites ysum: everyone is done with this one
    __syncwarp();
    if (lane == 0) mbar_arrive(cbar);
    if (!mbar_wait(cbar, cph, abort_flag, a.status)) return false;
    cph ^= 1u;
  }
  return true;
}

// The split-K FFN kernel.  Cooperative launch (the final grid-wide wait needs
// every CTA resident); a.rb_done[0] is the zeroed arrival counter.
template <bool SINGLE, int GROUP, int BITS>
__global__ void __launch_bounds__(kFfnThreads, 1)
    ffn_splitk_kernel(const __grid_constant__ CUtensorMap gq, const __grid_constant__ CUtensorMap uq,
                      const __grid_constant__ CUtensorMap gs, const __grid_constant__ CUtensorMap us,
                      const __grid_constant__ CUtensorMap dq, const __grid_constant__ CUtensorMap ds,
                      const FfnArgs a) {
  using F = SkCfg<GROUP, BITS>;
  constexpr int NS = F::NS, STAGE = F::STAGE, KCG = F::D::KCG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* red = reinterpret_cast<float*>(smem + NS * STAGE);
  int32_t* meta = reinterpret_cast<int32_t*>(smem + NS * STAGE + F::RED_BYTES);
  uint16_t* hbuf = reinterpret_cast<uint16_t*>(smem + NS * STAGE + F::RED_BYTES + F::META_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NS * STAGE + F::RED_BYTES + F::META_BYTES + F::H_BYTES);
  uint64_t* empty = full + NS;
  uint64_t* red_full = empty + NS;
  uint64_t* red_empty = red_full + kRowWarps;
  uint64_t* h_ready = red_empty + kRowWarps;
  uint64_t* h_free = h_ready + 1;
  uint64_t* cbar = h_free + 1;
  uint64_t* gbar = cbar + 1;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + F::NBAR);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int q = 0; q < NS; ++q) {
      mbar_init(&full[q], 1);
      mbar_init(&empty[q], kFfnConsumerWarps);
    }
    for (int r = 0; r < kRowWarps; ++r) {
      mbar_init(&red_full[r], 32);
      mbar_init(&red_empty[r], 32);
    }
    mbar_init(h_ready, kRowWarps);          // the K-half-0 warps write h
    mbar_init(h_free, kFfnConsumerWarps);
    mbar_init(cbar, kFfnConsumerWarps);
    mbar_init(gbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kFfnConsumerWarps && lane == 0) {
    prefetch_tensormap(&gq);
    prefetch_tensormap(&uq);
    prefetch_tensormap(&dq);
  }
  pdl_wait();
  pdl_trigger();
  Meta m;
  {
    const int n_seg = __ldg(a.plan);
    const int U = __ldg(a.n_unique);
    int32_t* mplan = meta;
    int32_t* muniq = meta + kMaxSeg + 2;
    int32_t* mseg = muniq + kMaxSeg;
    for (int i = threadIdx.x; i < n_seg + 3; i += blockDim.x) mplan[i] = __ldg(a.plan + i);
    for (int i = threadIdx.x; i < U; i += blockDim.x) muniq[i] = __ldg(a.unique_ids + i);
    for (int i = threadIdx.x; i <= U; i += blockDim.x) mseg[i] = __ldg(a.seg_off + i);
    m.plan = mplan;
    m.unique = muniq;
    m.seg_off = mseg;
    m.n_seg = n_seg;
    m.U = U;
    m.S = n_seg - U;
    m.total_blocks = __ldg(a.plan + 1);
    m.nrb_gu = a.I / kRowBlock;
    m.nrb_dn = a.H / kRowBlock;
    m.tiles_gu = m.total_blocks * m.nrb_gu;
    m.tiles_all = m.tiles_gu;
  }
  __syncthreads();

  if (warp == kFfnConsumerWarps) {
    // ---------------- producer ----------------
    int s = 0;
    uint32_t ph = 0;
    long issued = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < m.tiles_gu; t += gridDim.x) {
      const TileInfo ti = decode_tile<8>(a, m, t);
      ok = produce_tile<KCG, 1, 2, NS, STAGE, GROUP, BITS>(a, ti, &gq, &uq, &gs, &us, a.gate_s, a.up_s, a.H, a.I,
                                                           m.nrb_gu, smem, full, empty, s, ph, issued, abort_flag,
                                                           lane);
      if (ok) ok = produce_down_slice<NS, STAGE, GROUP, BITS>(a, ti, &dq, &ds, smem, full, empty, s, ph, issued,
                                                              abort_flag, lane);
    }
    if (!ok && lane == 0) {
      // bounded wait (ignoring the abort flag) for the copies still in flight
      int dummy = 0;
      const long n = issued < NS ? issued : NS;
      for (long q = 0; q < n; ++q) {
        const long idx = issued - 1 - q;
        mbar_wait(&full[static_cast<int>(idx % NS)], static_cast<uint32_t>((idx / NS) & 1),
                  reinterpret_cast<volatile int*>(&dummy), a.status);
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  int s = 0;
  uint32_t ph = 0, rph = 0, lu = 0;
  for (int t = blockIdx.x; t < m.tiles_gu; t += gridDim.x, ++lu) {
    const TileInfo ti = decode_tile<8>(a, m, t);
    if (!consume_tile<KCG, 1, 2, SINGLE, NS, STAGE, GROUP, true, BITS>(a, m, ti, a.H, a.I, smem, red, full, empty,
                                                                       red_full, red_empty, s, ph, rph, abort_flag,
                                                                       warp, lane, hbuf, h_free, h_ready, lu))
      return;
    if (!consume_down_slice<SINGLE, NS, STAGE, GROUP, BITS>(a, ti, smem, hbuf, full, empty, h_ready, h_free, s, ph,
                                                            lu, abort_flag, warp, lane))
      return;
  }
  // publish: every warp fences its partials and checks in on the CTA barrier;
  // then one thread per CTA increments the grid counter and waits (bounded)
  // for every CTA, and releases the CTA's warps through gbar
  __threadfence();
  __syncwarp();
  uint32_t cph = 0;
  if (lane == 0) mbar_arrive(cbar);
  if (!mbar_wait(cbar, cph, abort_flag, a.status)) return;
  cph ^= 1u;
  // the h slice buffer is free now: it takes the batch's pair_pos and
  // topk_w for the combine while the grid-wide wait runs
  int32_t* pos_s = reinterpret_cast<int32_t*>(hbuf);
  float* w_s = reinterpret_cast<float*>(pos_s + kSkMaxT * 32);
  for (int i = warp * 32 + lane; i < a.T * a.k; i += kFfnConsumerWarps * 32) {
    pos_s[i] = __ldg(a.pair_pos + i);
    w_s[i] = __ldg(a.topk_w + i);
  }
  if (warp == 0 && lane == 0) {
    __threadfence();
    atomicAdd(a.rb_done, 1);
    if (wait_counter(a.rb_done, static_cast<int>(gridDim.x), abort_flag, a.status)) mbar_arrive(gbar);
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(cbar);
  if (!mbar_wait(cbar, cph, abort_flag, a.status)) return;
  cph ^= 1u;
  if (!mbar_wait(gbar, 0, abort_flag, a.status)) return;
  splitk_combine(a, pos_s, w_s, smem, NS * STAGE, cbar, cph, abort_flag, warp, lane);
}

}  // namespace coli
