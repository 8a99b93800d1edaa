// Decode form of the int4 expert FFN and the routing-weighted combine.
//
// The routed experts are int4 (Colibri README, "L'idea": ~19 MB per expert in
// the int4 container; the three matrices of an expert are the gate, up and
// down projections of a SwiGLU FFN).  For the few tokens per expert of decode,
// the step is bound by reading the int4 weights, so this form streams them
// once at HBM rate:
//   * a persistent CTA per SM walks (segment, token block, 128-row block)
//     tiles from the plan; one producer warp moves 128-row x 256-element
//     chunks of codes (128B-swizzled tensor-map copies) and their fp16 scales
//     into a ring of shared-memory stages;
//   * 8 consumer warps (16 rows each) turn every 32-bit code word into four
//     bf16x2 pairs (two bit operations each: mask + magic exponent, then an
//     exact bf16x2 subtract), feed them as the A operand of m16n8k16 bf16
//     mma.sync against up to 8 tokens per n-tile, and multiply each 32-wide
//     group's fp32 partial by its fp16 scale.  Codes, activations and products
//     are exact; accumulation is fp32.
// Mode 0 runs gate and up together and writes h = bf16(silu(g) * u); mode 1
// runs down and writes y (fp32) per (pair, row); the combine kernel then sums
// each token's k routed y's with its routing weights, its shared experts and
// its residual in a fixed order and rounds once to bf16.
#pragma once
#include "common.cuh"
#include "k_union.cuh"

namespace coli {

constexpr int kFfnConsumerWarps = 8;
constexpr int kFfnThreads = (kFfnConsumerWarps + 1) * 32;
constexpr int kRowBlock = 16 * kFfnConsumerWarps;  // 128 rows per tile

struct FfnArgs {
  const uint16_t* bsrc;      // mode 0: fragment-ordered x [T][K]; mode 1: h [P+S*T][K]
  const uint16_t* scales0;   // 1-D scale copies when a stage spans all of K
  const uint16_t* scales1;
  const int32_t* unique_ids;
  const int32_t* n_unique;
  const int32_t* seg_off;
  const int32_t* perm;
  const int32_t* plan;       // [n_seg, total_blocks, tile_off[0..n_seg]]
  uint16_t* hq;              // mode 0 output, fragment-ordered [P+S*T][R]
  float* ypair;              // mode 1 output [P+S*T][R]
  uint32_t* status;
  int K, R, T, k, E, P;
};

template <int MODE, int KC>
struct FfnCfg {
  static constexpr int NMAT = MODE == 0 ? 2 : 1;
  static constexpr int ROWB = KC / 2;          // code bytes per row per stage
  static constexpr int SROWB = KC / 16;        // scale bytes per row per stage
  static constexpr int CODE_BYTES = kRowBlock * ROWB;
  static constexpr int SC_BYTES = kRowBlock * SROWB;
  static constexpr int STAGE = NMAT * (CODE_BYTES + SC_BYTES);
  static constexpr int NS = MODE == 0 ? 5 : (KC == 256 ? 10 : 8);
  static constexpr bool SWZ = (KC == 256);
  static constexpr size_t SMEM = static_cast<size_t>(NS) * STAGE + 1024 + 2 * NS * 8 + 16;
  static_assert(CODE_BYTES % 1024 == 0 && SC_BYTES % 1024 == 0, "stage regions must stay 1 KiB aligned");
};

// Two code nibbles (e_i, e_{i+4}) of word w -> exact bf16x2 (q_i, q_{i+4}).
// (w >> sh) & 0x000F000F keeps one nibble per half; XOR with 0x4308 sets the
// bf16 exponent of 128 and flips bit 3, giving 128 + (n ^ 8) = 136 + q for the
// two's-complement code q; subtracting 136 leaves q.
__device__ __forceinline__ uint32_t dq_pair(uint32_t w, int sh) {
  uint32_t t = w >> sh, r, q;
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(r) : "r"(t), "r"(0x000F000Fu), "r"(0x43084308u));
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(q) : "r"(r), "r"(0x43084308u));
  return q;
}

__device__ __forceinline__ void mma_16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct TileInfo {
  int u, tb, rb, e, base, cnt;
  bool routed;
};

__device__ __forceinline__ TileInfo decode_tile(const FfnArgs& a, int tile, int nrb, int n_seg, int U) {
  TileInfo ti;
  const int tbg = tile / nrb;
  ti.rb = tile - tbg * nrb;
  int lo = 0, hi = n_seg - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(a.plan + 2 + mid) <= tbg) lo = mid; else hi = mid - 1;
  }
  ti.u = lo;
  ti.tb = tbg - __ldg(a.plan + 2 + lo);
  if (lo < U) {
    ti.routed = true;
    ti.e = __ldg(a.unique_ids + lo);
    ti.base = __ldg(a.seg_off + lo);
    ti.cnt = __ldg(a.seg_off + lo + 1) - ti.base;
  } else {
    ti.routed = false;
    const int s = lo - U;
    ti.e = a.E + s;
    ti.base = a.P + s * a.T;
    ti.cnt = a.T;
  }
  return ti;
}

template <int MODE, int KC>
__global__ void __launch_bounds__(kFfnThreads, 1)
    ffn_decode_kernel(const __grid_constant__ CUtensorMap mapq0, const __grid_constant__ CUtensorMap mapq1,
                      const __grid_constant__ CUtensorMap maps0, const __grid_constant__ CUtensorMap maps1,
                      const FfnArgs a) {
  using C = FfnCfg<MODE, KC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::NS * C::STAGE);
  uint64_t* empty = full + C::NS;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + C::NS);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kFfnConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int n_seg = __ldg(a.plan + 0);
  const int nrb = a.R / kRowBlock;
  const int n_tiles = __ldg(a.plan + 1) * nrb;
  const int U = __ldg(a.n_unique);
  const int nkc = a.K / KC;

  if (warp == kFfnConsumerWarps) {
    // ---------------- producer ----------------
    if (lane == 0) {
      prefetch_tensormap(&mapq0);
      prefetch_tensormap(&maps0);
      if (C::NMAT == 2) {
        prefetch_tensormap(&mapq1);
        prefetch_tensormap(&maps1);
      }
      int s = 0;
      uint32_t ph = 0;
      long issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x) {
        const TileInfo ti = decode_tile(a, tile, nrb, n_seg, U);
        const int row0 = ti.e * a.R + ti.rb * kRowBlock;
        for (int kc = 0; kc < nkc; ++kc) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, a.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], C::STAGE);
          uint8_t* st = smem + s * C::STAGE;
          tma_load_2d(st, &mapq0, &full[s], kc * C::ROWB, row0);
          if (C::NMAT == 2) tma_load_2d(st + C::CODE_BYTES, &mapq1, &full[s], kc * C::ROWB, row0);
          uint8_t* sc = st + C::NMAT * C::CODE_BYTES;
          if (KC == a.K) {
            bulk_load(sc, a.scales0 + static_cast<size_t>(row0) * (a.K / 32), C::SC_BYTES, &full[s]);
            if (C::NMAT == 2)
              bulk_load(sc + C::SC_BYTES, a.scales1 + static_cast<size_t>(row0) * (a.K / 32), C::SC_BYTES, &full[s]);
          } else {
            tma_load_2d(sc, &maps0, &full[s], kc * (KC / 32), row0);
            if (C::NMAT == 2) tma_load_2d(sc + C::SC_BYTES, &maps1, &full[s], kc * (KC / 32), row0);
          }
          ++issued;
          if (++s == C::NS) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        // Wait (bounded, ignoring the abort flag) for the copies still in
        // flight so none lands after this CTA has exited.
        int dummy = 0;
        const long n = issued < C::NS ? issued : C::NS;
        for (long q = 0; q < n; ++q) {
          const long idx = issued - 1 - q;
          const int ss = static_cast<int>(idx % C::NS);
          const uint32_t pp = static_cast<uint32_t>((idx / C::NS) & 1);
          mbar_wait(&full[ss], pp, reinterpret_cast<volatile int*>(&dummy), a.status);
        }
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  const int g = lane >> 2, c = lane & 3;
  const int rl0 = 16 * warp + g, rl1 = rl0 + 8;  // tile-local rows of this thread
  int s = 0;
  uint32_t ph = 0;
  for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const TileInfo ti = decode_tile(a, tile, nrb, n_seg, U);
    const int i0 = ti.tb * kTokBlock;
    const int ntok = min(kTokBlock, ti.cnt - i0);
    const int nnt = (ntok + 7) >> 3;
    int brow[8];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int i = i0 + nt * 8 + g;
      int r = -1;
      if (nt < nnt && i < ti.cnt) {
        if (MODE == 0) r = ti.routed ? __ldg(a.perm + ti.base + i) / a.k : i;
        else r = ti.base + i;
      }
      brow[nt] = r;
    }
    float acc0[8][4], acc1[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc0[nt][q] = 0.f;
        acc1[nt][q] = 0.f;
      }

    for (int kc = 0; kc < nkc; ++kc) {
      if (!mbar_wait(&full[s], ph, abort_flag, a.status)) return;
      const uint32_t st = smem_addr(smem + s * C::STAGE);
      const uint32_t sc = st + C::NMAT * C::CODE_BYTES;
#pragma unroll
      for (int j = 0; j < KC / 32; ++j) {
        const uint32_t o0 = rl0 * C::ROWB + ((C::SWZ ? (j ^ (rl0 & 7)) : j) << 4) + 4 * c;
        const uint32_t o1 = rl1 * C::ROWB + ((C::SWZ ? (j ^ (rl1 & 7)) : j) << 4) + 4 * c;
        const uint32_t w0 = lds32(st + o0), w1 = lds32(st + o1);
        const float s0 = half_bits_to_float(lds16(sc + rl0 * C::SROWB + 2 * j));
        const float s1 = half_bits_to_float(lds16(sc + rl1 * C::SROWB + 2 * j));
        const uint32_t p00 = dq_pair(w0, 0), p01 = dq_pair(w0, 4), p02 = dq_pair(w0, 8), p03 = dq_pair(w0, 12);
        const uint32_t p10 = dq_pair(w1, 0), p11 = dq_pair(w1, 4), p12 = dq_pair(w1, 8), p13 = dq_pair(w1, 12);
        uint32_t u00 = 0, u01 = 0, u02 = 0, u03 = 0, u10 = 0, u11 = 0, u12 = 0, u13 = 0;
        float t0 = 0.f, t1 = 0.f;
        if (C::NMAT == 2) {
          const uint32_t v0 = lds32(st + C::CODE_BYTES + o0), v1 = lds32(st + C::CODE_BYTES + o1);
          t0 = half_bits_to_float(lds16(sc + C::SC_BYTES + rl0 * C::SROWB + 2 * j));
          t1 = half_bits_to_float(lds16(sc + C::SC_BYTES + rl1 * C::SROWB + 2 * j));
          u00 = dq_pair(v0, 0); u01 = dq_pair(v0, 4); u02 = dq_pair(v0, 8); u03 = dq_pair(v0, 12);
          u10 = dq_pair(v1, 0); u11 = dq_pair(v1, 4); u12 = dq_pair(v1, 8); u13 = dq_pair(v1, 12);
        }
        const int kg = kc * KC + 32 * j + 8 * c;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          if (nt < nnt) {
            uint4 b = make_uint4(0u, 0u, 0u, 0u);
            if (brow[nt] >= 0) b = ldg_nc_v4(a.bsrc + static_cast<size_t>(brow[nt]) * a.K + kg);
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            mma_16816(d, p00, p10, p01, p11, b.x, b.y);
            mma_16816(d, p02, p12, p03, p13, b.z, b.w);
            acc0[nt][0] = fmaf(s0, d[0], acc0[nt][0]);
            acc0[nt][1] = fmaf(s0, d[1], acc0[nt][1]);
            acc0[nt][2] = fmaf(s1, d[2], acc0[nt][2]);
            acc0[nt][3] = fmaf(s1, d[3], acc0[nt][3]);
            if (C::NMAT == 2) {
              float e[4] = {0.f, 0.f, 0.f, 0.f};
              mma_16816(e, u00, u10, u01, u11, b.x, b.y);
              mma_16816(e, u02, u12, u03, u13, b.z, b.w);
              acc1[nt][0] = fmaf(t0, e[0], acc1[nt][0]);
              acc1[nt][1] = fmaf(t0, e[1], acc1[nt][1]);
              acc1[nt][2] = fmaf(t1, e[2], acc1[nt][2]);
              acc1[nt][3] = fmaf(t1, e[3], acc1[nt][3]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == C::NS) {
        s = 0;
        ph ^= 1u;
      }
    }

    // epilogue: d0 (row g, col 2c), d1 (row g, col 2c+1), d2 (row g+8, col 2c), d3 (row g+8, col 2c+1)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      if (nt < nnt) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int rloc = (q < 2) ? rl0 : rl1;
          const int i = i0 + nt * 8 + 2 * c + (q & 1);
          if (i < ti.cnt) {
            const size_t orow = static_cast<size_t>(ti.base + i);
            const int r = ti.rb * kRowBlock + rloc;
            if (MODE == 0) {
              const float gv = acc0[nt][q], uv = acc1[nt][q];
              const float hv = gv / (1.0f + expf(-gv)) * uv;
              a.hq[orow * a.R + frag_pos(r)] = float_to_bf16_bits(hv);
            } else {
              a.ypair[orow * a.R + r] = acc0[nt][q];
            }
          }
        }
      }
    }
  }
}

// out[t, n] = bf16( sum_{j<k} w[t,j] * y[pair_pos[t*k+j], n] + sum_s y[P + s*T + t, n]
//                   + residual[t, n] ), fp32, in exactly this order.
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ ypair,
                                                      const int32_t* __restrict__ pair_pos,
                                                      const float* __restrict__ w,
                                                      const uint16_t* __restrict__ residual, int T, int k,
                                                      int S, int H, uint16_t* __restrict__ out) {
  const int per_tok = H / 4;
  const long total = static_cast<long>(T) * per_tok;
  const int P = T * k;
  for (long idx = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(idx / per_tok);
    const int n = static_cast<int>(idx - static_cast<long>(t) * per_tok) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int pp = __ldg(pair_pos + t * k + j);
      if (pp >= 0) {
        const float wt = __ldg(w + t * k + j);
        const float4 y = __ldg(reinterpret_cast<const float4*>(ypair + static_cast<size_t>(pp) * H + n));
        acc.x = fmaf(wt, y.x, acc.x);
        acc.y = fmaf(wt, y.y, acc.y);
        acc.z = fmaf(wt, y.z, acc.z);
        acc.w = fmaf(wt, y.w, acc.w);
      }
    }
    for (int s = 0; s < S; ++s) {
      const float4 y =
          __ldg(reinterpret_cast<const float4*>(ypair + static_cast<size_t>(P + s * T + t) * H + n));
      acc.x += y.x;
      acc.y += y.y;
      acc.z += y.z;
      acc.w += y.w;
    }
    if (residual) {
      const uint2 r = *reinterpret_cast<const uint2*>(residual + static_cast<size_t>(t) * H + n);
      acc.x += __uint_as_float(r.x << 16);
      acc.y += __uint_as_float(r.x & 0xffff0000u);
      acc.z += __uint_as_float(r.y << 16);
      acc.w += __uint_as_float(r.y & 0xffff0000u);
    }
    uint2 o;
    o.x = float_to_bf16_bits(acc.x) | (static_cast<uint32_t>(float_to_bf16_bits(acc.y)) << 16);
    o.y = float_to_bf16_bits(acc.z) | (static_cast<uint32_t>(float_to_bf16_bits(acc.w)) << 16);
    *reinterpret_cast<uint2*>(out + static_cast<size_t>(t) * H + n) = o;
  }
}

}  // namespace coli
