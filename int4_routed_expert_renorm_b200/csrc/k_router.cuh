// Route step kernels: optional pre-norm + fragment-ordered copy of the
// activations, router logits, and the top-k / renormalised-softmax router.
//
// Route is the first step of every layer of every token on the Colibri
// README's per-token path ("Il percorso di ogni token"; getting-started
// guide, "1. Route": the router decides which experts a token activates).
#pragma once
#include "common.cuh"

namespace coli {

constexpr float kRmsEps = 1e-6f;

// Eight consecutive expert-input values of a token from its bf16 row: x, or
// with pre-norm n = bf16(x * r).
__device__ __forceinline__ void input8(const uint16_t* __restrict__ xr, int i, int prenorm, float r, float (&v)[8]) {
  const uint4 q = *reinterpret_cast<const uint4*>(xr + i);
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = __uint_as_float(w[k] << 16);
    v[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
  }
  if (prenorm) {
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = bf16_bits_to_float(float_to_bf16_bits(v[k] * r));
  }
}

// Integer planes of one token's expert input (common.cuh): the largest |v|
// over the row sets the grid exponent (*xe), then the H/32 plane records go
// to xp_row.  Called by every thread of a block of 256 (H % 256 == 0, so each
// warp covers whole groups); `mx` is 8 floats of shared memory.
__device__ __forceinline__ void token_planes(const uint16_t* __restrict__ xr, int H, int prenorm, float r,
                                             uint8_t* __restrict__ xp_row, int32_t* __restrict__ xe, float* mx) {
  float m = 0.f;
  for (int i = threadIdx.x * 8; i < H; i += blockDim.x * 8) {
    float v[8];
    input8(xr, i, prenorm, r, v);
#pragma unroll
    for (int k = 0; k < 8; ++k) m = fmaxf(m, fabsf(v[k]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __syncthreads();   // mx may still be read from the previous token
  if ((threadIdx.x & 31) == 0) mx[threadIdx.x >> 5] = m;
  __syncthreads();
  m = 0.f;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) m = fmaxf(m, mx[w]);
  const int e = plane_exponent(m);
  if (threadIdx.x == 0) *xe = e;
  float f1, f2;
  pow2_split(e, f1, f2);
  const int c = threadIdx.x & 3;
  for (int i = threadIdx.x * 8; i < H; i += blockDim.x * 8) {
    float v[8];
    input8(xr, i, prenorm, r, v);
    uint2 lo, hi;
    int slo, shi;
    planes8(v, f1, f2, lo, hi, slo, shi);
    uint8_t* rec = xp_row + static_cast<size_t>(i >> 5) * kPlaneRec;
    *reinterpret_cast<uint2*>(rec + 8 * c) = lo;
    *reinterpret_cast<uint2*>(rec + 32 + 8 * c) = hi;
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      slo += __shfl_xor_sync(0xffffffffu, slo, o);
      shi += __shfl_xor_sync(0xffffffffu, shi, o);
    }
    if (c == 0) *reinterpret_cast<int2*>(rec + 64) = make_int2(kPlaneMagic - 8 * slo, -8 * shi);
  }
}

// One block per token.  Writes the fragment-ordered copy `xq` of the layer's
// expert input (bf16; with xq_f16, for the prefill form, the fp16 copies of
// those bf16 values, COLI_FLAG_RANGE for one of magnitude 65536 or more), its
// integer planes `xp` / grid exponents `xe` when xp is not NULL (the split-K
// decode form), and, with prenorm, the natural-order normalised copy `xn`:
//   n = bf16( x * (1 / sqrt(mean(x^2) + 1e-6)) ), the sum of squares in fp32
// in a fixed order.  H % 8 == 0.
__global__ void __launch_bounds__(256) prep_kernel(const uint16_t* __restrict__ x, int H, int prenorm,
                                                   uint16_t* __restrict__ xn, uint16_t* __restrict__ xq,
                                                   uint8_t* __restrict__ xp, int32_t* __restrict__ xe, int xq_f16,
                                                   uint32_t* __restrict__ status) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  const uint16_t* xr = x + static_cast<size_t>(t) * H;
  __shared__ float red[8];
  float r = 1.0f;
  bool range = false;
  if (prenorm) {
    float ss = 0.f;
    for (int i = threadIdx.x * 8; i < H; i += blockDim.x * 8) {
      uint4 v = *reinterpret_cast<const uint4*>(xr + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float a = __uint_as_float(w[q] << 16), b = __uint_as_float(w[q] & 0xffff0000u);
        ss = fmaf(a, a, ss);
        ss = fmaf(b, b, ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += red[w];
    r = 1.0f / sqrtf(tot / static_cast<float>(H) + kRmsEps);
  }
  for (int i = threadIdx.x * 8; i < H; i += blockDim.x * 8) {
    uint4 v = *reinterpret_cast<const uint4*>(xr + i);
    uint16_t e[8];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      e[2 * q] = static_cast<uint16_t>(w[q] & 0xffffu);
      e[2 * q + 1] = static_cast<uint16_t>(w[q] >> 16);
    }
    if (prenorm) {
#pragma unroll
      for (int q = 0; q < 8; ++q) e[q] = float_to_bf16_bits(bf16_bits_to_float(e[q]) * r);
      uint4 o;
      o.x = e[0] | (static_cast<uint32_t>(e[1]) << 16);
      o.y = e[2] | (static_cast<uint32_t>(e[3]) << 16);
      o.z = e[4] | (static_cast<uint32_t>(e[5]) << 16);
      o.w = e[6] | (static_cast<uint32_t>(e[7]) << 16);
      *reinterpret_cast<uint4*>(xn + static_cast<size_t>(t) * H + i) = o;
    }
    // fragment order x0 x4 x1 x5 x2 x6 x3 x7 (fp16 copies for the prefill form)
    if (xq_f16) to_f16_8(e, range);
    uint4 o;
    o.x = e[0] | (static_cast<uint32_t>(e[4]) << 16);
    o.y = e[1] | (static_cast<uint32_t>(e[5]) << 16);
    o.z = e[2] | (static_cast<uint32_t>(e[6]) << 16);
    o.w = e[3] | (static_cast<uint32_t>(e[7]) << 16);
    *reinterpret_cast<uint4*>(xq + static_cast<size_t>(t) * H + i) = o;
  }
  if (range) atomicOr(status, COLI_FLAG_RANGE);
  if (xp) {
    __shared__ float mx[8];
    token_planes(xr, H, prenorm, r, xp + static_cast<size_t>(t) * (H / 32) * kPlaneRec, xe + t, mx);
  }
}

// Router logits l[t,e] = sum_h x[t,h] * W_r[e,h] in fp32, for batches of more
// than 8 tokens.  Block = 8 warps, 8 experts (one per warp) and up to `tt`
// tokens whose bf16 rows the block first copies into shared memory (read once
// per block instead of once per expert).  Each (token, expert) is summed in
// front_kernel's order, so that a token's logits are the same bits in a batch
// of any size: H in eight ranges of H/8; in range w, lane l adds the elements
// w*H/8 + 4l + 128j (j ascending, float4 loads of W_r, four in flight); the
// lanes of each range are added in a fixed tree, and the eight range sums in
// turn.  H % 128 == 0; dynamic shared memory tt * H * 2 bytes.
__global__ void __launch_bounds__(256) logits_tile_kernel(const uint16_t* __restrict__ x,
                                                          const float* __restrict__ wr, int T, int E, int H, int tt,
                                                          float* __restrict__ logits) {
  extern __shared__ uint4 xs_raw[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(xs_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.y * tt;
  const int nt = min(tt, T - t0);
  const int e = blockIdx.x * 8 + warp;
  const float* wrow = wr + static_cast<size_t>(e < E ? e : 0) * H;
  const int hw = H >> 3;                 // one range
  const int nch = (hw + 511) / 512;      // chunks of four float4 per lane and range
  const int nall = 8 * nch;
  // chunk c: range c / nch, this lane's elements h0 + 4 lane + 512 (c % nch) + 128 u
  auto load_chunk = [&](int c, float4 (&wv)[4]) {
    const int w8 = c / nch, k = c - w8 * nch;
    const int h0 = w8 * hw, h1 = h0 + hw;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int h = h0 + lane * 4 + 512 * k + 128 * u;
      wv[u] = (e < E && h < h1) ? __ldg(reinterpret_cast<const float4*>(wrow + h)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  // the expert's first W_r loads do not depend on the previous kernel
  float4 wq[4];
  load_chunk(0, wq);
  pdl_wait();
  pdl_trigger();
  const int n16 = nt * H / 8;
  for (int i = threadIdx.x; i < n16; i += blockDim.x)
    xs_raw[i] = *reinterpret_cast<const uint4*>(x + static_cast<size_t>(t0) * H + static_cast<size_t>(i) * 8);
  __syncthreads();
  if (e >= E) return;
  float acc[8], tot[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) acc[q] = tot[q] = 0.f;
  for (int c = 0; c < nall; ++c) {
    const int w8 = c / nch, k = c - w8 * nch;
    const int h0 = w8 * hw, h1 = h0 + hw;
    float4 cur[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) cur[u] = wq[u];
    // the next chunk's loads go out before this chunk's arithmetic
    if (c + 1 < nall) load_chunk(c + 1, wq);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int h = h0 + lane * 4 + 512 * k + 128 * u;
      if (h < h1) {
        const float4 w = cur[u];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (q < nt) {
            const uint2 xv = *reinterpret_cast<const uint2*>(xs + static_cast<size_t>(q) * H + h);
            float a = acc[q];
            a = fmaf(__uint_as_float(xv.x << 16), w.x, a);
            a = fmaf(__uint_as_float(xv.x & 0xffff0000u), w.y, a);
            a = fmaf(__uint_as_float(xv.y << 16), w.z, a);
            a = fmaf(__uint_as_float(xv.y & 0xffff0000u), w.w, a);
            acc[q] = a;
          }
        }
      }
    }
    if (k == nch - 1) {
      // end of a range: its lane tree, then onto the running sum
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float v = acc[q];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        tot[q] += v;
        acc[q] = 0.f;
      }
    }
  }
#pragma unroll
  for (int q = 0; q < 8; ++q)
    if (lane == 0 && q < nt) logits[static_cast<size_t>(t0 + q) * E + e] = tot[q];
}

// Router logits for batches of more than kLogitsMmaMinT - 1 tokens (prefill
// chunks), on the tensor cores.  W_r (fp32) is split on the fly into three
// bf16 pieces, w = w1 + w2 + w3 (w1 = bf16(w), w2 = bf16(w - w1), w3 =
// bf16(w - w1 - w2); each difference is exact in fp32, so the pieces carry all
// 24 bits of w), and l[t,e] = sum over the pieces of x . w_i^T with
// mma.sync m16n8k16 (bf16 x bf16, exact products, fp32 accumulation).  Each
// 256-wide K chunk is accumulated in a fresh accumulator (16 k-steps x 3
// pieces) and added to the running fp32 sum in chunk order, so every (token,
// expert) is summed the same way whatever the batch.  CTA = 64 tokens x 64
// experts, 8 warps as 2 x 4 (32 tokens x 16 experts each); K in chunks of 32,
// double-buffered in shared memory (rows padded to 40 bf16: conflict-free
// fragment loads).  H % 256 == 0.
constexpr int kLogitsMmaMinT = 65;
constexpr int kLgBM = 64, kLgBN = 64, kLgBK = 32, kLgStr = 40;

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The three bf16 pieces of four fp32 values, packed two per word.
__device__ __forceinline__ void split3(float4 v, uint2 (&p)[3]) {
  const float f[4] = {v.x, v.y, v.z, v.w};
  uint16_t q[3][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint16_t b1 = float_to_bf16_bits(f[i]);
    const float r1 = f[i] - bf16_bits_to_float(b1);
    const uint16_t b2 = float_to_bf16_bits(r1);
    const float r2 = r1 - bf16_bits_to_float(b2);
    q[0][i] = b1;
    q[1][i] = b2;
    q[2][i] = float_to_bf16_bits(r2);
  }
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    p[j].x = q[j][0] | (static_cast<uint32_t>(q[j][1]) << 16);
    p[j].y = q[j][2] | (static_cast<uint32_t>(q[j][3]) << 16);
  }
}

__global__ void __launch_bounds__(256) logits_mma_kernel(const uint16_t* __restrict__ x,
                                                         const float* __restrict__ wr, int T, int E, int H,
                                                         float* __restrict__ logits) {
  __shared__ __align__(16) uint16_t xs[2][kLgBM * kLgStr];
  __shared__ __align__(16) uint16_t ws[2][3][kLgBN * kLgStr];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int t0 = blockIdx.y * kLgBM, e0 = blockIdx.x * kLgBN;
  const int wm = warp & 1, wn = warp >> 1;
  // global loads of one K chunk: x row tid / 4, 8 bf16 at column 8 (tid % 4);
  // W_r rows tid / 8 and 32 + tid / 8, 4 fp32 at column 4 (tid % 8)
  const int xr = tid >> 2, xq = tid & 3;
  const int wrw = tid >> 3, wq = tid & 7;
  const bool xin = t0 + xr < T;
  const bool win0 = e0 + wrw < E, win1 = e0 + wrw + 32 < E;
  const uint16_t* xp = x + static_cast<size_t>(xin ? t0 + xr : 0) * H + 8 * xq;
  const float* wp0 = wr + static_cast<size_t>(win0 ? e0 + wrw : 0) * H + 4 * wq;
  const float* wp1 = wr + static_cast<size_t>(win1 ? e0 + wrw + 32 : 0) * H + 4 * wq;
  uint4 xv;
  float4 wv0, wv1;
  auto load = [&](int kc) {
    const int k0 = kc * kLgBK;
    xv = xin ? *reinterpret_cast<const uint4*>(xp + k0) : make_uint4(0u, 0u, 0u, 0u);
    wv0 = win0 ? __ldg(reinterpret_cast<const float4*>(wp0 + k0)) : make_float4(0.f, 0.f, 0.f, 0.f);
    wv1 = win1 ? __ldg(reinterpret_cast<const float4*>(wp1 + k0)) : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  auto store = [&](int b) {
    *reinterpret_cast<uint4*>(&xs[b][xr * kLgStr + 8 * xq]) = xv;
    uint2 p0[3], p1[3];
    split3(wv0, p0);
    split3(wv1, p1);
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      *reinterpret_cast<uint2*>(&ws[b][j][wrw * kLgStr + 4 * wq]) = p0[j];
      *reinterpret_cast<uint2*>(&ws[b][j][(wrw + 32) * kLgStr + 4 * wq]) = p1[j];
    }
  };
  pdl_wait();
  pdl_trigger();
  const int nk = H / kLgBK;
  constexpr int kChunk = 256 / kLgBK;     // K chunks per fresh accumulator
  float tot[2][2][4], acc[2][2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) tot[mt][nt][i] = acc[mt][nt][i] = 0.f;
  load(0);
  store(0);
  __syncthreads();
  for (int kc = 0; kc < nk; ++kc) {
    const int b = kc & 1;
    if (kc + 1 < nk) load(kc + 1);
#pragma unroll
    for (int ks = 0; ks < kLgBK / 16; ++ks) {
      const int kk = ks * 16 + 2 * c;
      uint32_t a[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const uint16_t* r0 = &xs[b][(32 * wm + 16 * mt + g) * kLgStr + kk];
        const uint16_t* r8 = r0 + 8 * kLgStr;
        a[mt][0] = *reinterpret_cast<const uint32_t*>(r0);
        a[mt][1] = *reinterpret_cast<const uint32_t*>(r8);
        a[mt][2] = *reinterpret_cast<const uint32_t*>(r0 + 8);
        a[mt][3] = *reinterpret_cast<const uint32_t*>(r8 + 8);
      }
#pragma unroll
      for (int j = 0; j < 3; ++j) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const uint16_t* wrow = &ws[b][j][(16 * wn + 8 * nt + g) * kLgStr + kk];
          const uint32_t b0 = *reinterpret_cast<const uint32_t*>(wrow);
          const uint32_t b1 = *reinterpret_cast<const uint32_t*>(wrow + 8);
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) mma_bf16_16816(acc[mt][nt], a[mt], b0, b1);
        }
      }
    }
    if ((kc + 1) % kChunk == 0) {
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            tot[mt][nt][i] += acc[mt][nt][i];
            acc[mt][nt][i] = 0.f;
          }
    }
    if (kc + 1 < nk) store(b ^ 1);
    __syncthreads();
  }
  // d0, d1: token row g, experts 2c, 2c + 1; d2, d3: token row g + 8
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = t0 + 32 * wm + 16 * mt + g + 8 * h;
        const int e = e0 + 16 * wn + 8 * nt + 2 * c;
        if (t < T) {
          if (e < E) logits[static_cast<size_t>(t) * E + e] = tot[mt][nt][2 * h];
          if (e + 1 < E) logits[static_cast<size_t>(t) * E + e + 1] = tot[mt][nt][2 * h + 1];
        }
      }
}

// COLI_LAYER_HOST_X: the input rows (and, when b is not NULL, the residual
// rows) from page-locked host memory into the workspace, n 16-byte chunks
// each.  It waits for the previous kernel first, which may still read the
// staging buffers of an earlier call.
__global__ void __launch_bounds__(256) stage_rows_kernel(const uint4* __restrict__ a, uint4* __restrict__ da,
                                                         const uint4* __restrict__ b, uint4* __restrict__ db,
                                                         long n) {
  pdl_wait();
  pdl_trigger();
  for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long>(gridDim.x) * blockDim.x) {
    const uint4 v = a[i];
    if (b) db[i] = b[i];
    da[i] = v;
  }
}

// Small-batch front end (T <= 8), one launch of E + T blocks (T when the
// logits are given, wr == NULL): block e < E computes the router logits of
// expert e for every token; block E + t writes token t's fragment-ordered
// copy of the expert input (and, when xp is not NULL, its integer planes and
// grid exponent), so that no block does both.  With
// prenorm every block normalises its tokens itself (n = bf16(x * r) with
// r = 1/sqrt(mean(x^2) + 1e-6) summed in the same order as prep_kernel), so
// the logits see exactly the normalised input the experts see.  Block 0
// zeroes *zero_ctr when it is not NULL (the arrival counter of a split-K FFN
// kernel that routes the batch itself, so that no routing kernel runs between).
__global__ void __launch_bounds__(256) front_kernel(const uint16_t* __restrict__ x, const float* __restrict__ wr,
                                                    int T, int E, int H, int prenorm, float* __restrict__ logits,
                                                    uint16_t* __restrict__ xn, uint16_t* __restrict__ xq,
                                                    uint8_t* __restrict__ xp, int32_t* __restrict__ xe, int xq_f16,
                                                    uint32_t* __restrict__ status, int32_t* __restrict__ zero_ctr) {
  const int nlog = wr ? E : 0;   // blocks [0, nlog): logits of expert b; then one block per token
  // a logits block's first W_r loads (warp w: range [w H/8, (w+1) H/8), lane l:
  // elements 4 l + 128 it) do not depend on the previous kernel
  constexpr int kIt = 8;                       // float4 per lane per pass (1024 elements per warp)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hw = H >> 3;
  const int h0 = warp * hw, h1 = h0 + hw;
  const float* wrow = wr + static_cast<size_t>(static_cast<int>(blockIdx.x) < nlog ? blockIdx.x : 0) * H;
  float4 w0[kIt];
  if (static_cast<int>(blockIdx.x) < nlog) {
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
      const int h = h0 + lane * 4 + it * 128;
      w0[it] = h < h1 ? __ldg(reinterpret_cast<const float4*>(wrow + h)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  pdl_wait();
  pdl_trigger();
  if (zero_ctr && blockIdx.x == 0 && threadIdx.x == 0) *zero_ctr = 0;
  __shared__ float red[8][8];
  __shared__ float rs[64];
  const int e = blockIdx.x;
  if (prenorm) {
    // every token's sum of squares in one pass (T <= 8 with pre-norm), with
    // prep_kernel's per-thread order, lane reduction and warp order: each
    // token gets the same bits whatever the batch
    float ss[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) ss[t] = 0.f;
    for (int i = threadIdx.x * 8; i < H; i += blockDim.x * 8) {
      uint4 v[8];
#pragma unroll
      for (int t = 0; t < 8; ++t)
        if (t < T) v[t] = *reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H + i);
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (t < T) {
          const uint32_t w[4] = {v[t].x, v[t].y, v[t].z, v[t].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float a = __uint_as_float(w[q] << 16), b = __uint_as_float(w[q] & 0xffff0000u);
            ss[t] = fmaf(a, a, ss[t]);
            ss[t] = fmaf(b, b, ss[t]);
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss[t] += __shfl_xor_sync(0xffffffffu, ss[t], o);
      if ((threadIdx.x & 31) == 0) red[t][threadIdx.x >> 5] = ss[t];
    }
    __syncthreads();
    if (threadIdx.x < T) {
      float tot = 0.f;
      for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) tot += red[threadIdx.x][w];
      rs[threadIdx.x] = 1.0f / sqrtf(tot / static_cast<float>(H) + kRmsEps);
    }
    __syncthreads();
  }
  // fragment-ordered (and normalised) copy and integer planes of this block's token
  if (static_cast<int>(blockIdx.x) >= nlog) {
    const int t = blockIdx.x - nlog;
    const uint16_t* xr = x + static_cast<size_t>(t) * H;
    const float r = prenorm ? rs[t] : 1.0f;
    bool range = false;
    for (int i = threadIdx.x * 8; i < H; i += blockDim.x * 8) {
      const uint4 v = *reinterpret_cast<const uint4*>(xr + i);
      uint16_t q8[8];
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        q8[2 * q] = static_cast<uint16_t>(wv[q] & 0xffffu);
        q8[2 * q + 1] = static_cast<uint16_t>(wv[q] >> 16);
      }
      if (prenorm) {
#pragma unroll
        for (int q = 0; q < 8; ++q) q8[q] = float_to_bf16_bits(bf16_bits_to_float(q8[q]) * r);
        uint4 o;
        o.x = q8[0] | (static_cast<uint32_t>(q8[1]) << 16);
        o.y = q8[2] | (static_cast<uint32_t>(q8[3]) << 16);
        o.z = q8[4] | (static_cast<uint32_t>(q8[5]) << 16);
        o.w = q8[6] | (static_cast<uint32_t>(q8[7]) << 16);
        *reinterpret_cast<uint4*>(xn + static_cast<size_t>(t) * H + i) = o;
      }
      if (xq_f16) to_f16_8(q8, range);
      uint4 o;
      o.x = q8[0] | (static_cast<uint32_t>(q8[4]) << 16);
      o.y = q8[1] | (static_cast<uint32_t>(q8[5]) << 16);
      o.z = q8[2] | (static_cast<uint32_t>(q8[6]) << 16);
      o.w = q8[3] | (static_cast<uint32_t>(q8[7]) << 16);
      *reinterpret_cast<uint4*>(xq + static_cast<size_t>(t) * H + i) = o;
    }
    if (range) atomicOr(status, COLI_FLAG_RANGE);
    if (xp) {
      __shared__ float mx[8];
      token_planes(xr, H, prenorm, r, xp + static_cast<size_t>(t) * (H / 32) * kPlaneRec, xe + t, mx);
    }
  }
  if (static_cast<int>(blockIdx.x) >= nlog) return;
  // logits of expert e for every token, 8 tokens at a time.  Each lane issues
  // all its W_r loads (and a token's x loads) before any arithmetic, so the
  // DRAM round trips overlap instead of following one another; the first
  // pass's W_r values are w0, loaded before the wait.
  __shared__ float part[8][8];
  for (int t0 = 0; t0 < T; t0 += 8) {
    const int nt = min(8, T - t0);
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    for (int hb = h0 + lane * 4; hb < h1; hb += 128 * kIt) {
      float4 w[kIt];
      const bool first = hb == h0 + lane * 4;
#pragma unroll
      for (int it = 0; it < kIt; ++it)
        w[it] = first ? w0[it]
                      : (hb + it * 128 < h1) ? __ldg(reinterpret_cast<const float4*>(wrow + hb + it * 128))
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (q < nt) {
          const uint16_t* xr = x + static_cast<size_t>(t0 + q) * H;
          uint2 xv[kIt];
#pragma unroll
          for (int it = 0; it < kIt; ++it)
            xv[it] = (hb + it * 128 < h1) ? *reinterpret_cast<const uint2*>(xr + hb + it * 128) : make_uint2(0u, 0u);
          float a = acc[q];
#pragma unroll
          for (int it = 0; it < kIt; ++it) {
            float x0 = __uint_as_float(xv[it].x << 16), x1 = __uint_as_float(xv[it].x & 0xffff0000u);
            float x2 = __uint_as_float(xv[it].y << 16), x3 = __uint_as_float(xv[it].y & 0xffff0000u);
            if (prenorm) {
              const float r = rs[t0 + q];
              x0 = bf16_bits_to_float(float_to_bf16_bits(x0 * r));
              x1 = bf16_bits_to_float(float_to_bf16_bits(x1 * r));
              x2 = bf16_bits_to_float(float_to_bf16_bits(x2 * r));
              x3 = bf16_bits_to_float(float_to_bf16_bits(x3 * r));
            }
            a = fmaf(x0, w[it].x, a);
            a = fmaf(x1, w[it].y, a);
            a = fmaf(x2, w[it].z, a);
            a = fmaf(x3, w[it].w, a);
          }
          acc[q] = a;
        }
      }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float v = acc[q];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) part[warp][q] = v;
    }
    __syncthreads();
    if (threadIdx.x < nt) {
      float sacc = 0.f;
#pragma unroll
      for (int w8 = 0; w8 < 8; ++w8) sacc += part[w8][threadIdx.x];
      logits[static_cast<size_t>(t0 + threadIdx.x) * E + e] = sacc;
    }
  }
}

// (value, index) order of the router: larger value first, then lower index.
// Route one token with one warp: top-k over E <= 32*NV logits (+ bias) and
// the renormalised softmax weights.  Lane l holds experts l, l+32, ...
// Slot j receives the j-th expert in (value desc, index asc) order and
// w_j = exp(l_j - l_max) / sum_{i<k} exp(l_i - l_max), summed in slot order.
// NaN ranks as -inf; NaN or +inf anywhere, or a selected -inf, returns bad.
// Lane j < k gets slot j in *id / *w.
// PRELOAD: every logit and bias load is issued before any arithmetic (the
// split-K kernel's own routing, where the logits come from L2); the same
// values and decisions either way.
template <int NV, bool PRELOAD = false>
__device__ __forceinline__ bool route_token(const float* __restrict__ lr, const float* __restrict__ bias, int E,
                                            int k, int lane, int* id, float* w) {
  float v[NV], bq[NV];
  if constexpr (PRELOAD) {
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const int e = lane + 32 * q;
      v[q] = e < E ? lr[e] : 0.f;
      bq[q] = (bias && e < E) ? bias[e] : 0.f;
    }
  }
  uint32_t taken = 0;
  bool bad = false;
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const int e = lane + 32 * q;
    float val = -INFINITY;
    if (e < E) {
      val = PRELOAD ? v[q] : lr[e];
      if (bias) val = val + (PRELOAD ? bq[q] : bias[e]);
      if (isnan(val)) {
        bad = true;
        val = -INFINITY;
      } else if (isinf(val) && val > 0.f) {
        bad = true;
      }
      if (val == 0.f) val = 0.f;   // -0.0 ties +0.0
    } else {
      taken |= 1u << q;  // padding never selected
    }
    v[q] = val;
  }
  // Each round: every lane offers its best untaken value as an order-preserving
  // integer (larger value -> larger key; -0.0 was folded into +0.0 above),
  // the warp takes the maximum key and, among lanes holding it, the lowest
  // expert index -- two redux.sync reductions instead of a shuffle tree.
  uint32_t ord[NV];
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const uint32_t u = __float_as_uint(v[q]);
    ord[q] = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  }
  float l_max = 0.f, my_v = 0.f;
  int my_id = 0;
  for (int j = 0; j < k; ++j) {
    uint32_t lo = 0u;            // below every real key (-inf maps to 0x007FFFFF)
    int le = 0x7fffffff;
#pragma unroll
    for (int q = 0; q < NV; ++q)
      if (!(taken & (1u << q)) && ord[q] > lo) {   // strict: the lower index wins ties inside a lane
        lo = ord[q];
        le = lane + 32 * q;
      }
    const uint32_t m = __reduce_max_sync(0xffffffffu, lo);
    const int bi = __reduce_min_sync(0xffffffffu, lo == m ? le : 0x7fffffff);
    const uint32_t bu = (m & 0x80000000u) ? (m & 0x7fffffffu) : ~m;
    const float bv = __uint_as_float(bu);
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (j == 0) l_max = bv;
    if (lane == j) {
      my_v = bv;
      my_id = bi;
    }
    if (isinf(bv) && bv < 0.f) bad = true;
  }
  const float ej = (lane < k) ? expf(my_v - l_max) : 0.f;
  float sum = 0.f;
  for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, ej, j);
  *id = my_id;
  *w = ej / sum;
  return __any_sync(0xffffffffu, bad);
}

// One warp per token over the whole batch (any T).
template <int NV>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits, const float* __restrict__ bias,
                                                    int T, int E, int k, int32_t* __restrict__ ids,
                                                    float* __restrict__ wout, uint32_t* __restrict__ status) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  int id;
  float w;
  const bool bad = route_token<NV>(logits + static_cast<size_t>(t) * E, bias, E, k, lane, &id, &w);
  if (lane < k) {
    ids[static_cast<size_t>(t) * k + lane] = id;
    wout[static_cast<size_t>(t) * k + lane] = w;
  }
  if (bad && lane == 0) atomicOr(status, COLI_FLAG_NONFINITE);
}

// Values per lane needed for E experts (E <= 1024).
inline int route_nv(int E) {
  const int nv = (E + 31) / 32;
  return nv <= 1 ? 1 : nv <= 2 ? 2 : nv <= 4 ? 4 : nv <= 8 ? 8 : nv <= 16 ? 16 : 32;
}

}  // namespace coli
