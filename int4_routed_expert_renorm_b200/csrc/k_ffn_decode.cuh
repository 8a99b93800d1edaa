// Decode form of the int4 expert FFN and the routing-weighted combine.
//
// The routed experts are int4 (Colibri README, "L'idea": ~19 MB per expert in
// the int4 container; an expert's three matrices are the gate, up and down
// projections of a SwiGLU FFN).  With few tokens per expert the step is bound
// by reading the int4 weights, so this form streams them once at HBM rate:
//   * a persistent CTA per SM walks (segment, token block, 128-row block)
//     tiles of the device-side plan; one producer warp moves, per stage,
//     128 rows x 256 K of codes (2-D tensor-map copies, 128B swizzle), their
//     fp16 scales, and the stage's slice of each token's activation row
//     (1-D bulk copies) into a ring of shared-memory stages;
//   * 16 consumer warps: warps w and w+8 own the same 16 rows and split every
//     stage's 32-wide groups between them (first and second half), so each SM
//     sub-partition has four warps to hide latency; they sum their partial
//     accumulators once per tile, in a fixed order;
//   * dequantisation of a pair of codes is one mask-and-magic LOP3 (nibble n
//     of two's-complement code q becomes the bf16 value 128 + (n ^ 8) =
//     136 + q) and one exact bf16x2 subtract of 136 (on the FMA pipe, which
//     the rest of the loop leaves idle); m16n8k16 bf16 mma.sync multiplies the
//     codes with up to 8 tokens per n-tile; each 32-wide group's fp32 partial
//     is multiplied by its fp16 scale and accumulated in fp32.
// Mode 0 runs gate and up together and writes h = bf16(silu(g) * u); mode 1
// runs down and writes y (fp32) per (pair, row).  combine_kernel then sums each
// token's k routed y's with its routing weights, its shared experts and its
// residual in a fixed order and rounds once to bf16.
#pragma once
#include "common.cuh"
#include "k_union.cuh"

namespace coli {

constexpr int kRowWarps = 8;                         // 16-row slices per tile
constexpr int kFfnConsumerWarps = 2 * kRowWarps;     // two K-halves per slice
constexpr int kFfnThreads = (kFfnConsumerWarps + 1) * 32;
constexpr int kRowBlock = 16 * kRowWarps;            // 128 rows per tile

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

// MODE 0 gate/up, 1 down; KC elements of K per stage; NT n-tiles of 8 tokens
// per tile; SINGLE: every tile holds exactly one token (T == 1).
template <int MODE, int KC, int NT, bool SINGLE>
struct FfnCfg {
  static constexpr int NMAT = MODE == 0 ? 2 : 1;
  static constexpr int TOKB = 8 * NT;                 // tokens per tile
  static constexpr int GPS = KC / 32;                 // groups per stage
  static constexpr int GPW = GPS / 2;                 // groups per warp per stage
  static constexpr int ROWB = KC / 2;                 // code bytes per row per stage
  static constexpr int SROWB = KC / 16;               // scale bytes per row per stage
  static constexpr int CODE_BYTES = kRowBlock * ROWB;
  static constexpr int SC_BYTES = kRowBlock * SROWB;
  static constexpr int W_BYTES = NMAT * (CODE_BYTES + SC_BYTES);   // weights of one stage
  // activation rows of the tile's tokens for this stage: KC bf16 + 64 B pad, so
  // the 16-byte fragment loads of 8 tokens x 4 lanes fall in distinct banks
  static constexpr int XROW = KC * 2 + 64;
  static constexpr int X_BYTES = TOKB * XROW;
  static constexpr int STAGE = ((W_BYTES + X_BYTES) + 1023) / 1024 * 1024;
  static constexpr int RED_BYTES = kRowWarps * 32 * NT * 4 * NMAT * 4;   // K-half partials
  static constexpr int NS_RAW = (225 * 1024 - RED_BYTES - 2048) / STAGE;
  static constexpr int NS = NS_RAW > 8 ? 8 : NS_RAW;
  static constexpr bool SWZ = (KC == 256);
  static constexpr size_t SMEM =
      static_cast<size_t>(NS) * STAGE + RED_BYTES + 1024 + (2 * NS + 2 * kRowWarps) * 8 + 16;
  static_assert(CODE_BYTES % 1024 == 0 && SC_BYTES % 1024 == 0, "stage regions must stay 1 KiB aligned");
  static_assert(NS >= 2, "pipeline depth");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(!SINGLE || NT == 1, "single-token tiles use one n-tile");
};

// Two code nibbles (e_i, e_{i+4}) of word w -> exact bf16x2 (q_i, q_{i+4}).
// (w >> sh) & 0x000F000F keeps one nibble per 16-bit half; XOR with 0x4308
// puts it under the exponent of 128 and flips bit 3, giving 128 + (n ^ 8) =
// 136 + q; subtracting 136 leaves q.
__device__ __forceinline__ uint32_t dq_pair(uint32_t w, int sh) {
  uint32_t r, q;
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(r) : "r"(w >> sh), "r"(0x000F000Fu), "r"(0x43084308u));
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

__device__ __forceinline__ __half2 u32_as_half2(uint32_t v) {
  __half2 h;
  memcpy(&h, &v, 4);
  return h;
}

struct TileInfo {
  int u, tb, rb, e, base, cnt;
  bool routed;
};

// Tile -> (segment, token block, row block).  Segments 0..S-1 are the shared
// experts (every token), then the U unique routed experts (plan order).
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
  const int S = n_seg - U;
  if (lo >= S) {
    ti.routed = true;
    ti.e = __ldg(a.unique_ids + (lo - S));
    ti.base = __ldg(a.seg_off + (lo - S));
    ti.cnt = __ldg(a.seg_off + (lo - S) + 1) - ti.base;
  } else {
    ti.routed = false;
    ti.e = a.E + lo;
    ti.base = a.P + lo * a.T;
    ti.cnt = a.T;
  }
  return ti;
}

// Accumulate one 32-wide group of one matrix for one n-tile: p[0..3] are the
// bf16x2 code pairs of row g, p[4..7] of row g + 8; b the token fragment.
template <bool SINGLE>
__device__ __forceinline__ void group_acc(float (&acc)[4], const uint32_t (&p)[8], const uint4& b, float s0,
                                          float s1) {
  float d[4] = {0.f, 0.f, 0.f, 0.f};
  mma_16816(d, p[0], p[4], p[1], p[5], b.x, b.y);
  mma_16816(d, p[2], p[6], p[3], p[7], b.z, b.w);
  acc[0] = fmaf(s0, d[0], acc[0]);
  acc[2] = fmaf(s1, d[2], acc[2]);
  if (!SINGLE) {
    acc[1] = fmaf(s0, d[1], acc[1]);
    acc[3] = fmaf(s1, d[3], acc[3]);
  }
}

__device__ __forceinline__ void dq_word_pair(uint32_t (&p)[8], uint32_t w0, uint32_t w1) {
  p[0] = dq_pair(w0, 0); p[1] = dq_pair(w0, 4); p[2] = dq_pair(w0, 8); p[3] = dq_pair(w0, 12);
  p[4] = dq_pair(w1, 0); p[5] = dq_pair(w1, 4); p[6] = dq_pair(w1, 8); p[7] = dq_pair(w1, 12);
}

template <int MODE, int KC, int NT, bool SINGLE>
__global__ void __launch_bounds__(kFfnThreads, 1)
    ffn_decode_kernel(const __grid_constant__ CUtensorMap mapq0, const __grid_constant__ CUtensorMap mapq1,
                      const __grid_constant__ CUtensorMap maps0, const __grid_constant__ CUtensorMap maps1,
                      const FfnArgs a) {
  using C = FfnCfg<MODE, KC, NT, SINGLE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* red = reinterpret_cast<float*>(smem + C::NS * C::STAGE);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::NS * C::STAGE + C::RED_BYTES);
  uint64_t* empty = full + C::NS;
  uint64_t* red_full = empty + C::NS;       // [kRowWarps]: K-half 1 partials written
  uint64_t* red_empty = red_full + kRowWarps;  // [kRowWarps]: K-half 0 has read them
  volatile int* abort_flag = reinterpret_cast<volatile int*>(red_empty + kRowWarps);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kFfnConsumerWarps);
    }
    for (int r = 0; r < kRowWarps; ++r) {
      mbar_init(&red_full[r], 32);
      mbar_init(&red_empty[r], 32);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();

  const int n_seg = __ldg(a.plan + 0);
  const int nrb = a.R / kRowBlock;
  const int n_tiles = __ldg(a.plan + 1) * nrb;
  const int U = __ldg(a.n_unique);
  const int nkc = a.K / KC;

  if (warp == kFfnConsumerWarps) {
    // ---------------- producer ----------------
    if (lane == 0) {
      prefetch_tensormap(&mapq0);
      if (C::NMAT == 2) prefetch_tensormap(&mapq1);
      if (KC != a.K) {
        prefetch_tensormap(&maps0);
        if (C::NMAT == 2) prefetch_tensormap(&maps1);
      }
    }
    int s = 0;
    uint32_t ph = 0;
    long issued = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x) {
      const TileInfo ti = decode_tile(a, tile, nrb, n_seg, U);
      const int row0 = ti.e * a.R + ti.rb * kRowBlock;
      const int i0 = ti.tb * C::TOKB;
      const int ntok = min(C::TOKB, ti.cnt - i0);
      int brow = 0;  // activation row of the token this lane copies (lane < ntok)
      if (lane < ntok) {
        const int i = i0 + lane;
        if (MODE == 0) brow = ti.routed ? __ldg(a.perm + ti.base + i) / a.k : i;
        else brow = ti.base + i;
      }
      const uint16_t* bsrc_row = a.bsrc + static_cast<size_t>(brow) * a.K;
      for (int kc = 0; kc < nkc; ++kc) {
        if (lane == 0) ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, a.status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        uint8_t* st = smem + s * C::STAGE;
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], C::W_BYTES + ntok * KC * 2);
          tma_load_2d(st, &mapq0, &full[s], kc * C::ROWB, row0);
          if (C::NMAT == 2) tma_load_2d(st + C::CODE_BYTES, &mapq1, &full[s], kc * C::ROWB, row0);
          uint8_t* sc = st + C::NMAT * C::CODE_BYTES;
          if (KC == a.K) {
            bulk_load(sc, a.scales0 + static_cast<size_t>(row0) * (a.K / 32), C::SC_BYTES, &full[s]);
            if (C::NMAT == 2)
              bulk_load(sc + C::SC_BYTES, a.scales1 + static_cast<size_t>(row0) * (a.K / 32), C::SC_BYTES,
                        &full[s]);
          } else {
            tma_load_2d(sc, &maps0, &full[s], kc * (KC / 32), row0);
            if (C::NMAT == 2) tma_load_2d(sc + C::SC_BYTES, &maps1, &full[s], kc * (KC / 32), row0);
          }
        }
        __syncwarp();
        if (lane < ntok) bulk_load(st + C::W_BYTES + lane * C::XROW, bsrc_row + kc * KC, KC * 2, &full[s]);
        ++issued;
        if (++s == C::NS) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (!ok && lane == 0) {
      // Wait (bounded, ignoring the abort flag) for the copies still in flight
      // so none lands after this CTA has exited.
      int dummy = 0;
      const long n = issued < C::NS ? issued : C::NS;
      for (long q = 0; q < n; ++q) {
        const long idx = issued - 1 - q;
        mbar_wait(&full[static_cast<int>(idx % C::NS)], static_cast<uint32_t>((idx / C::NS) & 1),
                  reinterpret_cast<volatile int*>(&dummy), a.status);
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  const int rw = warp & (kRowWarps - 1);   // 16-row slice
  const int half = warp / kRowWarps;       // which half of each stage's groups
  const int g = lane >> 2, c = lane & 3;
  const int rl0 = 16 * rw + g;             // tile-local rows rl0 and rl0 + 8
  // Byte offset of this thread's code word in group 0 of row rl0.  With the
  // 128B swizzle the 16-byte chunk j of row r sits at chunk j ^ (r & 7), and
  // rl0 & 7 == (rl0 + 8) & 7 == g; bits 4..6 of cbase hold g, so chunk j is
  // cbase ^ (j << 4).
  const uint32_t cbase = rl0 * C::ROWB + (C::SWZ ? (g << 4) : 0) + 4 * c;
  const uint32_t sbase = rl0 * C::SROWB + half * C::GPW * 2;
  const uint32_t xbase = C::W_BYTES + g * C::XROW + (half * C::GPW * 32 + 8 * c) * 2;
  int s = 0;
  uint32_t ph = 0, rph = 0;
  for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, rph ^= 1u) {
    const TileInfo ti = decode_tile(a, tile, nrb, n_seg, U);
    const int i0 = ti.tb * C::TOKB;
    const int ntok = min(C::TOKB, ti.cnt - i0);
    const int nnt = (ntok + 7) >> 3;
    float acc0[NT][4], acc1[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc0[nt][q] = 0.f;
        acc1[nt][q] = 0.f;
      }

    for (int kc = 0; kc < nkc; ++kc) {
      if (!mbar_wait(&full[s], ph, abort_flag, a.status)) return;
      const uint8_t* st = smem + s * C::STAGE;
      const uint8_t* sc = st + C::NMAT * C::CODE_BYTES + sbase;
      // this warp's fp16 scales for its GPW groups (rows rl0 and rl0 + 8, both matrices)
      __half2 sh0[2], sh1[2], th0[2], th1[2];
      if (C::GPW == 4) {
        const uint2 v0 = *reinterpret_cast<const uint2*>(sc);
        const uint2 v1 = *reinterpret_cast<const uint2*>(sc + 8 * C::SROWB);
        sh0[0] = u32_as_half2(v0.x); sh0[1] = u32_as_half2(v0.y);
        sh1[0] = u32_as_half2(v1.x); sh1[1] = u32_as_half2(v1.y);
        if (C::NMAT == 2) {
          const uint2 u0 = *reinterpret_cast<const uint2*>(sc + C::SC_BYTES);
          const uint2 u1 = *reinterpret_cast<const uint2*>(sc + C::SC_BYTES + 8 * C::SROWB);
          th0[0] = u32_as_half2(u0.x); th0[1] = u32_as_half2(u0.y);
          th1[0] = u32_as_half2(u1.x); th1[1] = u32_as_half2(u1.y);
        }
      } else {
        sh0[0] = u32_as_half2(*reinterpret_cast<const uint32_t*>(sc));
        sh1[0] = u32_as_half2(*reinterpret_cast<const uint32_t*>(sc + 8 * C::SROWB));
        sh0[1] = sh1[1] = sh0[0];
        if (C::NMAT == 2) {
          th0[0] = u32_as_half2(*reinterpret_cast<const uint32_t*>(sc + C::SC_BYTES));
          th1[0] = u32_as_half2(*reinterpret_cast<const uint32_t*>(sc + C::SC_BYTES + 8 * C::SROWB));
          th0[1] = th1[1] = th0[0];
        }
      }
#pragma unroll
      for (int jj = 0; jj < C::GPW; ++jj) {
        const int j = half * C::GPW + jj;                       // group within the stage
        const uint8_t* ca = st + (cbase ^ static_cast<uint32_t>(j << 4));
        const uint32_t w0 = *reinterpret_cast<const uint32_t*>(ca);
        const uint32_t w1 = *reinterpret_cast<const uint32_t*>(ca + 8 * C::ROWB);
        const float s0 = (jj & 1) ? __high2float(sh0[jj >> 1]) : __low2float(sh0[jj >> 1]);
        const float s1 = (jj & 1) ? __high2float(sh1[jj >> 1]) : __low2float(sh1[jj >> 1]);
        uint32_t pg[8], pu[8];
        dq_word_pair(pg, w0, w1);
        float t0 = 0.f, t1 = 0.f;
        if (C::NMAT == 2) {
          const uint32_t v0 = *reinterpret_cast<const uint32_t*>(ca + C::CODE_BYTES);
          const uint32_t v1 = *reinterpret_cast<const uint32_t*>(ca + C::CODE_BYTES + 8 * C::ROWB);
          t0 = (jj & 1) ? __high2float(th0[jj >> 1]) : __low2float(th0[jj >> 1]);
          t1 = (jj & 1) ? __high2float(th1[jj >> 1]) : __low2float(th1[jj >> 1]);
          dq_word_pair(pu, v0, v1);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (NT == 1 || nt < nnt) {
            uint4 b = make_uint4(0u, 0u, 0u, 0u);
            if (nt * 8 + g < ntok) b = *reinterpret_cast<const uint4*>(st + xbase + nt * 8 * C::XROW + jj * 64);
            group_acc<SINGLE>(acc0[nt], pg, b, s0, s1);
            if (C::NMAT == 2) group_acc<SINGLE>(acc1[nt], pu, b, t0, t1);
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

    // Combine the two K-halves of each 16-row slice (fixed order: half 0 + half 1),
    // handing the partials over through shared memory under bounded waits.
    float* rp = red + (rw * 32 + lane) * (NT * 4 * C::NMAT);
    if (half == 1) {
      if (!mbar_wait(&red_empty[rw], rph ^ 1u, abort_flag, a.status)) return;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          rp[nt * 4 + q] = acc0[nt][q];
          if (C::NMAT == 2) rp[NT * 4 + nt * 4 + q] = acc1[nt][q];
        }
      mbar_arrive(&red_full[rw]);
      continue;
    }
    if (!mbar_wait(&red_full[rw], rph, abort_flag, a.status)) return;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc0[nt][q] += rp[nt * 4 + q];
        if (C::NMAT == 2) acc1[nt][q] += rp[NT * 4 + nt * 4 + q];
      }
    mbar_arrive(&red_empty[rw]);
    // epilogue: d0 (row g, col 2c), d1 (row g, col 2c+1), d2 (row g+8, col 2c), d3 (row g+8, col 2c+1)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      if (nt < nnt) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = i0 + nt * 8 + 2 * c + (q & 1);
          if (i < ti.cnt && !(SINGLE && (q & 1))) {
            const size_t orow = static_cast<size_t>(ti.base + i);
            const int r = ti.rb * kRowBlock + rl0 + ((q & 2) ? 8 : 0);
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
  pdl_wait();
  pdl_trigger();
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
