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
//
// Arithmetic: integer tensor-core products.  With one to eight tokens the
// step is bound by streaming the codes, and a bf16 product path spends most
// of its instructions turning nibbles into bf16 values.  Here the codes go to
// the tensor cores as bytes: an int4 code word of 8 nibbles becomes two words
// of unsigned bytes (code + 8) with one shift and two LOP3, an int8 word pair
// is regrouped with two PRMT, and mma.sync m16n8k32 (u8/s8 x s8 -> s32)
// multiplies them with the activations' integer planes (common.cuh: each
// token's expert input on a fixed-point grid of its own, as two signed byte
// planes; each MMA column is one plane of one token, so one MMA covers four
// tokens).  The accumulator starts at the value that cancels the +8 and
// carries a magic constant, so 256 * d_hi + d_lo is the group's exact
// integer dot product, read as fp32 with one subtraction; it is scaled by the
// group's fp16 scale and accumulated in fp32, group after group, as before.
//   * gate/up: per stage 128 rows x 256 K of both matrices (int8: 128 K) and
//     the 32-wide groups' plane records of the tile's tokens; warps w and
//     w + 8 own the same 16 rows and split each stage's groups; the K-halves
//     are added once per tile (half 0 + half 1); the epilogue scales g and u
//     back by the token's grid exponent and writes h = bf16(silu(g) * u) of
//     the tile's 128 rows into shared memory, with each token's largest |h|;
//   * h planes: four warps put each token's 128 h values on their own grid
//     (exponent from that largest |h|) and write the plane records of the
//     slice's four groups; every warp then holds its B operands in registers;
//   * down: stages of 512 output rows x 128 K (four 128-row tensor-map boxes
//     of 64 code bytes per row, 64B swizzle, and the rows' 8-scale boxes;
//     int8 codes: 256-row stages of two 128-byte-wide boxes); warp w owns
//     stage rows [32 w, 32 w + 32) (int8: 16 rows) and all 4 groups of the
//     slice; the fp32 result, scaled back by the slice's h exponent, is a
//     partial y per (pair, K slice, row), ypart;
//   * after its last unit every consumer warp fences its partials and checks in
//     on a CTA barrier; one thread per CTA then increments a grid counter;
//     once all CTAs have (a bounded grid-wide wait -- the grid is at most
//     one CTA per SM and one CTA fills an SM's shared memory, so every CTA is
//     resident), each CTA combines a contiguous range of (token, 4 rows):
//     y of every routed and shared pair as the sum of its I/128 partials in
//     slice order (a thread per pair and unit), then the routed y's weighted
//     in slot order, the shared y's and the residual (a thread per unit),
//     rounded once to bf16.
// Every token's arithmetic is the same whatever else is in the batch (its own
// grid, exact integer products, fixed orders everywhere), so the form is
// batch-invariant.
#pragma once
#include "k_ffn_decode.cuh"

namespace coli {

constexpr int kSkMaxT = 8;                       // largest batch this form takes
constexpr int kSkMaxSeg = 264;                   // unique routed + shared segments of such a batch (<= 8*32 + 4)
constexpr int kSkDnScale = kRowBlock * 16;       // the rows' 16-byte (8-scale) boxes
constexpr int kSkHRow = 128 * 2 + 64;            // padded bf16 row of one token's 128-row h slice
constexpr int kSkHGroups = kRowBlock / 32;       // 32-wide groups of one h slice (4)
constexpr int kSkMaxP = kSkMaxT * 32;            // pairs of such a batch (k <= 32)

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
  static constexpr int GPS = D::KCG / 32;                 // 32-wide groups per gate/up stage
  static constexpr int SLOT = GPS * kPlaneRec;            // one token's plane records of a stage
  static constexpr int GU_USED = GU::W_BYTES + kSkMaxT * SLOT;
  static constexpr int DN_USED = D::BOXES * (D::CODE + kSkDnScale);
  static constexpr int STAGE = ((GU_USED > DN_USED ? GU_USED : DN_USED) + 1023) / 1024 * 1024;
  static constexpr int RED_BYTES = kRowWarps * 32 * 8 * 4;             // K-half partials (2 n-tiles)
  static constexpr int META_BYTES = (3 * kSkMaxSeg + 4) * 4;
  static constexpr int H_BYTES = kSkMaxT * kSkHRow;                    // h slice, bf16, natural order
  static constexpr int HP_BYTES = kSkMaxT * kSkHGroups * kPlaneRec;    // its plane records
  static constexpr int HMAX_BYTES = kRowWarps * kSkMaxT * 4 + kSkMaxT * 4;
  static constexpr int ROUTE_BYTES = 4 * kSkMaxP * 4 + 16;   // routing weights, perm, pair_pos, ids; U
  static constexpr int NBAR = 64;
  static constexpr int FIXED =
      RED_BYTES + META_BYTES + H_BYTES + HP_BYTES + HMAX_BYTES + ROUTE_BYTES + 1024 + NBAR * 8 + 64;
  static constexpr int NS_RAW = (227 * 1024 - FIXED) / STAGE;
  static constexpr int NS = NS_RAW > 8 ? 8 : NS_RAW;
  static constexpr size_t SMEM = static_cast<size_t>(NS) * STAGE + FIXED;
  static_assert(NS >= 3, "pipeline depth");
  static_assert(2 * NS + 2 * kRowWarps + 6 <= NBAR, "barrier slots");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(D::CODE % 1024 == 0, "swizzled boxes need 1 KiB alignment");
  static_assert(GU::W_BYTES % 16 == 0 && SLOT % 16 == 0, "bulk copies need 16-byte alignment");
  static_assert(META_BYTES % 16 == 0 && H_BYTES % 16 == 0 && HP_BYTES % 16 == 0, "shared regions stay aligned");
  // the combine stages its pairs' y (k + S <= 36 per 4-row unit) in the stage ring
  static_assert(NS * STAGE >= 36 * 16, "combine staging");
  // the in-kernel routing stages the router bias (E <= 256) in red
  static_assert(RED_BYTES >= 256 * 4, "bias staging");
};

// Integer MMA of one 32-wide group: d = A * B + C with C = {c_lo, c_hi} in
// both row halves.  BITS 4: A unsigned bytes (code + 8); BITS 8: signed codes.
template <int BITS>
__device__ __forceinline__ void mma_i8(int (&d)[4], const uint32_t (&a)[4], uint2 b, int c_lo, int c_hi) {
  if (BITS == 4)
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%10,%11,%12,%13};"
                 : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b.x), "r"(b.y), "r"(c_lo), "r"(c_hi),
                   "r"(c_lo), "r"(c_hi));
  else
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%10,%11,%12,%13};"
                 : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b.x), "r"(b.y), "r"(c_lo), "r"(c_hi),
                   "r"(c_lo), "r"(c_hi));
}

// A operand of one group from the two code words of rows g (w0) and g + 8
// (w1): their even elements at k = 4c .., the odd ones at k = 16 + 4c ..
__device__ __forceinline__ void a_from_int4(uint32_t (&a)[4], uint32_t w0, uint32_t w1) {
  a[0] = (w0 & 0x0F0F0F0Fu) ^ 0x08080808u;
  a[1] = (w1 & 0x0F0F0F0Fu) ^ 0x08080808u;
  a[2] = ((w0 >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
  a[3] = ((w1 >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
}

// The same from the 8 int8 codes of each row (v0: row g, v1: row g + 8).
__device__ __forceinline__ void a_from_int8(uint32_t (&a)[4], uint2 v0, uint2 v1) {
  asm("prmt.b32 %0, %1, %2, 0x6420;" : "=r"(a[0]) : "r"(v0.x), "r"(v0.y));
  asm("prmt.b32 %0, %1, %2, 0x6420;" : "=r"(a[1]) : "r"(v1.x), "r"(v1.y));
  asm("prmt.b32 %0, %1, %2, 0x7531;" : "=r"(a[2]) : "r"(v0.x), "r"(v0.y));
  asm("prmt.b32 %0, %1, %2, 0x7531;" : "=r"(a[3]) : "r"(v1.x), "r"(v1.y));
}

// MMA result of one group -> the exact dot products of rows g and g + 8 for
// the lane's token, scaled by their fp16 group scales into the accumulators.
template <int BITS>
__device__ __forceinline__ void acc_group(float& acc0, float& acc8, const int (&d)[4], float s0, float s8) {
  float v0, v8;
  if (BITS == 4) {
    v0 = __int_as_float(d[0] + (d[1] << 8)) - kPlaneMagicF;
    v8 = __int_as_float(d[2] + (d[3] << 8)) - kPlaneMagicF;
  } else {
    // int8 codes: the two planes' sums read separately (each within 2^22)
    v0 = fmaf(__int_as_float(d[1]) - kPlaneMagicF, 256.f, __int_as_float(d[0]) - kPlaneMagicF);
    v8 = fmaf(__int_as_float(d[3]) - kPlaneMagicF, 256.f, __int_as_float(d[2]) - kPlaneMagicF);
  }
  acc0 = fmaf(s0, v0, acc0);
  acc8 = fmaf(s8, v8, acc8);
}

// The MMA start values of a plane record (int4 codes: they cancel the +8 of
// the unsigned codes; int8 codes only need the magic constant in both columns).
template <int BITS>
__device__ __forceinline__ int2 plane_c(uint32_t rec_addr_c) {
  if (BITS == 4) {
    const uint32_t lo = lds32(rec_addr_c), hi = lds32(rec_addr_c + 4);
    return make_int2(static_cast<int>(lo), static_cast<int>(hi));
  }
  return make_int2(kPlaneMagic, kPlaneMagic);
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// Batch token of slot i of a tile (perm: the union's permutation, in shared memory).
__device__ __forceinline__ int tile_token(const FfnArgs& a, const int32_t* perm, const TileInfo& ti, int i) {
  return ti.routed ? perm[ti.base + ti.i0 + i] / a.k : ti.i0 + i;
}

// Producer, weights of one gate/up stage of a unit: codes and scales of both
// matrices (tensor maps), announced on full[s] together with the plane
// records of the unit's ntok tokens.  One lane.
// The codes are read by this CTA alone, once: evict_first (`cpol`), so that
// they do not push the partial sums, the scales and the down codes (whose
// L2 lines neighbouring CTAs share) out of L2.
template <int STAGE, int GROUP, int BITS>
__device__ __forceinline__ void gu_stage_weights(const FfnArgs& a, int row0, int kc, int ntok, const CUtensorMap* mq0,
                                                 const CUtensorMap* mq1, const CUtensorMap* ms0,
                                                 const CUtensorMap* ms1, uint8_t* st, uint64_t* bar, uint64_t cpol) {
  using F = SkCfg<GROUP, BITS>;
  using C = typename F::GU;
  mbar_arrive_expect_tx(bar, C::W_BYTES + ntok * F::SLOT);
#pragma unroll
  for (int sb = 0; sb < C::SUBS; ++sb)
    tma_load_2d_hint(st + sb * C::SUB_BYTES, mq0, bar, kc * C::ROWB + sb * C::RSTR, row0, cpol);
  tma_load_2d_hint(st + C::CODE_BYTES, mq1, bar, kc * C::ROWB, row0, cpol);
  uint8_t* sc = st + 2 * C::CODE_BYTES;
  if (F::D::KCG == a.H) {
    // one stage spans K: the rows' scales are contiguous and move as 1-D
    // bulk copies (the host encodes no scale maps for this case)
    bulk_load(sc, a.gate_s + static_cast<size_t>(row0) * (a.H / GROUP), C::SC_BYTES, bar);
    bulk_load(sc + C::SC_BYTES, a.up_s + static_cast<size_t>(row0) * (a.H / GROUP), C::SC_BYTES, bar);
  } else {
    const int sx = C::BOX8 ? ((kc * C::SPS) & ~7) : kc * C::SPS;
    tma_load_2d(sc, ms0, bar, sx, row0);
    tma_load_2d(sc + C::SC_BYTES, ms1, bar, sx, row0);
  }
}

// Producer: the gate/up stages of one unit: the stage weights and the plane
// records of the tile's tokens (one 1-D bulk copy per token).  The weights of
// the first `pre` stages were already issued (into stages 0 .. pre-1 of the
// ring's first round) before the kernel waited for its inputs.  Returns false
// on a timeout.
template <int NS, int STAGE, int GROUP, int BITS>
__device__ __forceinline__ bool produce_gu_slice(const FfnArgs& a, const int32_t* perm, const TileInfo& ti,
                                                 const CUtensorMap* mq0, const CUtensorMap* mq1,
                                                 const CUtensorMap* ms0, const CUtensorMap* ms1, uint8_t* smem,
                                                 uint64_t* full, uint64_t* empty, int& s, uint32_t& ph,
                                                 long& issued, int pre, uint64_t cpol, volatile int* abort_flag,
                                                 int lane) {
  using F = SkCfg<GROUP, BITS>;
  using C = typename F::GU;
  const int row0 = ti.e * a.I + ti.rb * kRowBlock;
  const int nkc = a.H / F::D::KCG;
  const uint8_t* xsrc = a.xp;
  if (lane < ti.ntok) xsrc = a.xp + static_cast<size_t>(tile_token(a, perm, ti, lane)) * (a.H / 32) * kPlaneRec;
  for (int kc = 0; kc < nkc; ++kc) {
    uint8_t* st = smem + s * STAGE;
    if (kc >= pre) {
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, a.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) return false;
      if (lane == 0)
        gu_stage_weights<STAGE, GROUP, BITS>(a, row0, kc, ti.ntok, mq0, mq1, ms0, ms1, st, &full[s], cpol);
      ++issued;
    }
    __syncwarp();
    if (lane < ti.ntok)
      bulk_load(st + C::W_BYTES + lane * F::SLOT, xsrc + static_cast<size_t>(kc) * F::SLOT, F::SLOT, &full[s]);
    if (++s == NS) {
      s = 0;
      ph ^= 1u;
    }
  }
  return true;
}

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

// Shared-memory buffers of the h hand-over between a unit's gate/up and down.
struct SkHBufs {
  uint16_t* h;       // [kSkMaxT][kSkHRow / 2] bf16, natural row order
  uint8_t* hp;       // [kSkMaxT][kSkHGroups][kPlaneRec] plane records
  float* hmax;       // [kRowWarps][kSkMaxT] largest |h| per row warp and token
  int* he;           // [kSkMaxT] grid exponent of each token's h slice
  uint64_t *h_ready, *hp_ready, *h_free;
};

// Consumers: the gate/up stages of one unit, then h into shared memory.
// Returns false on a timeout.
template <int NT, int NS, int STAGE, int GROUP, int BITS>
__device__ __forceinline__ bool consume_gu_slice(const FfnArgs& a, const int32_t* perm, const TileInfo& ti,
                                                 uint8_t* smem, float* red,
                                                 uint64_t* full, uint64_t* empty, uint64_t* red_full,
                                                 uint64_t* red_empty, const SkHBufs& hb, int& s, uint32_t& ph,
                                                 uint32_t& rph, uint32_t lu, volatile int* abort_flag, int warp,
                                                 int lane) {
  using F = SkCfg<GROUP, BITS>;
  using C = typename F::GU;
  const int rw = warp & (kRowWarps - 1);   // 16-row slice
  const int half = warp / kRowWarps;       // which half of each stage's groups
  const int g = lane >> 2, c = lane & 3;
  const int rl0 = 16 * rw + g;             // tile-local rows rl0 and rl0 + 8
  // this thread's code bytes of group 0 of row rl0 (128B swizzle: 16-byte
  // chunk j of row r sits at chunk j ^ (r & 7), and rl0 & 7 == g)
  const uint32_t cbase = BITS == 4 ? rl0 * C::RSTR + (g << 4) + 4 * c
                                   : rl0 * C::RSTR + ((g ^ (c >> 1)) << 4) + 8 * (c & 1);
  constexpr int SPH = C::GPW * 32 / GROUP;
  const uint32_t sbase = rl0 * C::SROWB + half * SPH * 2;
  // B operand of this lane: column g = plane (g & 1) of slot nt * 4 + (g >> 1);
  // C values: slot nt * 4 + c
  const uint32_t xb = smem_addr(smem) + C::W_BYTES + (g >> 1) * F::SLOT + (g & 1) * 32 + 8 * c;
  const uint32_t xc = smem_addr(smem) + C::W_BYTES + c * F::SLOT + 64;
  const int nnt = (ti.ntok + 3) >> 2;
  const int nkc = a.H / F::D::KCG;
  // the grid exponents of this lane's tokens, needed after the last stage
  int xe[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int i = nt * 4 + c;
    xe[nt] = i < ti.ntok ? __ldg(a.xe + tile_token(a, perm, ti, i)) : 0;
  }
  float ag[NT][2], au[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) ag[nt][0] = ag[nt][1] = au[nt][0] = au[nt][1] = 0.f;

  for (int kc = 0; kc < nkc; ++kc) {
    if (!mbar_wait(&full[s], ph, abort_flag, a.status)) return false;
    const uint8_t* st = smem + s * STAGE;
    const uint32_t soff = s * STAGE;
    const uint8_t* sc = st + 2 * C::CODE_BYTES + sbase;
    __half2 sh0[4], sh1[4], th0[4], th1[4];
    {
      const uint8_t* sq = sc + (C::BOX8 ? ((kc * C::SPS) & 7) * 2 : 0);
      load_scales<SPH>(sq, sh0);
      load_scales<SPH>(sq + 8 * C::SROWB, sh1);
      load_scales<SPH>(sq + C::SC_BYTES, th0);
      load_scales<SPH>(sq + C::SC_BYTES + 8 * C::SROWB, th1);
    }
#pragma unroll
    for (int jj = 0; jj < C::GPW; ++jj) {
      const int j = half * C::GPW + jj;                       // group within the stage
      const int si = GROUP == 32 ? jj : (jj >> 1);            // this group's scale among the half's
      const float s0 = half2_pick(sh0[si >> 1], si & 1), s1 = half2_pick(sh1[si >> 1], si & 1);
      const float t0 = half2_pick(th0[si >> 1], si & 1), t1 = half2_pick(th1[si >> 1], si & 1);
      uint32_t fg[4], fu[4];
      if (BITS == 4) {
        const uint8_t* ca = st + (cbase ^ static_cast<uint32_t>(j << 4));
        a_from_int4(fg, *reinterpret_cast<const uint32_t*>(ca), *reinterpret_cast<const uint32_t*>(ca + 8 * C::RSTR));
        a_from_int4(fu, *reinterpret_cast<const uint32_t*>(ca + C::CODE_BYTES),
                    *reinterpret_cast<const uint32_t*>(ca + C::CODE_BYTES + 8 * C::RSTR));
      } else {
        const uint8_t* ca = st + (cbase ^ static_cast<uint32_t>((2 * j) << 4));
        a_from_int8(fg, *reinterpret_cast<const uint2*>(ca), *reinterpret_cast<const uint2*>(ca + 8 * C::RSTR));
        a_from_int8(fu, *reinterpret_cast<const uint2*>(ca + C::CODE_BYTES),
                    *reinterpret_cast<const uint2*>(ca + C::CODE_BYTES + 8 * C::RSTR));
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (NT == 1 || nt < nnt) {
          const uint2 b = lds64(xb + soff + nt * 4 * F::SLOT + j * kPlaneRec);
          const int2 cv = plane_c<BITS>(xc + soff + nt * 4 * F::SLOT + j * kPlaneRec);
          int d[4];
          mma_i8<BITS>(d, fg, b, cv.x, cv.y);
          acc_group<BITS>(ag[nt][0], ag[nt][1], d, s0, s1);
          mma_i8<BITS>(d, fu, b, cv.x, cv.y);
          acc_group<BITS>(au[nt][0], au[nt][1], d, t0, t1);
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

  // Add the two K-halves of each 16-row slice (fixed order: half 0 + half 1).
  float* rp = red + (rw * 32 + lane) * 8;
  if (half == 1) {
    if (!mbar_wait(&red_empty[rw], rph ^ 1u, abort_flag, a.status)) return false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      rp[nt * 4 + 0] = ag[nt][0];
      rp[nt * 4 + 1] = ag[nt][1];
      rp[nt * 4 + 2] = au[nt][0];
      rp[nt * 4 + 3] = au[nt][1];
    }
    mbar_arrive(&red_full[rw]);
    rph ^= 1u;
    return true;
  }
  if (!mbar_wait(&red_full[rw], rph, abort_flag, a.status)) return false;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    ag[nt][0] += rp[nt * 4 + 0];
    ag[nt][1] += rp[nt * 4 + 1];
    au[nt][0] += rp[nt * 4 + 2];
    au[nt][1] += rp[nt * 4 + 3];
  }
  mbar_arrive(&red_empty[rw]);
  rph ^= 1u;
  // h = bf16(silu(g) * u) of rows rl0 and rl0 + 8 for slot nt * 4 + c, after
  // g and u are scaled back by the token's grid exponent; then the largest
  // |h| of each token over the warp's 16 rows
  if (lu > 0 && !mbar_wait(hb.h_free, (lu - 1) & 1u, abort_flag, a.status)) return false;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int i = nt * 4 + c;
    float f1, f2;
    pow2_split(-xe[nt], f1, f2);
    float m = 0.f;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float gv = (ag[nt][r] * f1) * f2, uv = (au[nt][r] * f1) * f2;
      const uint16_t hbits = float_to_bf16_bits(gv / (1.0f + expf(-gv)) * uv);
      if (i < ti.ntok) hb.h[i * (kSkHRow / 2) + rl0 + 8 * r] = hbits;
      m = fmaxf(m, fabsf(bf16_bits_to_float(hbits)));
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (g == 0) hb.hmax[rw * kSkMaxT + i] = m;
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(hb.h_ready);
  return true;
}

// Consumers: h slice -> plane records (warps 0..3, one 32-wide group each:
// lane = slot * 4 + c), then every warp's B operands and C values of the
// slice's four groups into registers.  Returns false on a timeout.
template <int NT>
__device__ __forceinline__ bool load_h_planes(const FfnArgs& a, const TileInfo& ti, const SkHBufs& hb, uint32_t lu,
                                              uint2 (&hbv)[kSkHGroups][NT], int2 (&hcv)[kSkHGroups][NT],
                                              int (&he)[NT], volatile int* abort_flag, int warp, int lane) {
  if (!mbar_wait(hb.h_ready, lu & 1u, abort_flag, a.status)) return false;
  if (warp < kSkHGroups) {
    const int slot = lane >> 2, c = lane & 3, jg = warp;
    float m = 0.f;
#pragma unroll
    for (int w = 0; w < kRowWarps; ++w) m = fmaxf(m, hb.hmax[w * kSkMaxT + slot]);
    const int e = plane_exponent(m);
    if (slot < ti.ntok) {
      const uint4 v = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(hb.h) + slot * kSkHRow +
                                                      (jg * 32 + 8 * c) * 2);
      const float vals[8] = {__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                             __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u),
                             __uint_as_float(v.z << 16), __uint_as_float(v.z & 0xffff0000u),
                             __uint_as_float(v.w << 16), __uint_as_float(v.w & 0xffff0000u)};
      float f1, f2;
      pow2_split(e, f1, f2);
      uint2 lo, hi;
      int slo, shi;
      planes8(vals, f1, f2, lo, hi, slo, shi);
      uint8_t* rec = hb.hp + (slot * kSkHGroups + jg) * kPlaneRec;
      *reinterpret_cast<uint2*>(rec + 8 * c) = lo;
      *reinterpret_cast<uint2*>(rec + 32 + 8 * c) = hi;
      slo += __shfl_xor_sync(0x0000000fu << (lane & ~3), slo, 1);
      shi += __shfl_xor_sync(0x0000000fu << (lane & ~3), shi, 1);
      slo += __shfl_xor_sync(0x0000000fu << (lane & ~3), slo, 2);
      shi += __shfl_xor_sync(0x0000000fu << (lane & ~3), shi, 2);
      if (c == 0) *reinterpret_cast<int2*>(rec + 64) = make_int2(kPlaneMagic - 8 * slo, -8 * shi);
      if (jg == 0 && c == 0) hb.he[slot] = e;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(hb.hp_ready);
  }
  if (!mbar_wait(hb.hp_ready, lu & 1u, abort_flag, a.status)) return false;
  const int g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int sb = nt * 4 + (g >> 1), sc = nt * 4 + c;
#pragma unroll
    for (int j = 0; j < kSkHGroups; ++j) {
      hbv[j][nt] = *reinterpret_cast<const uint2*>(hb.hp + (sb * kSkHGroups + j) * kPlaneRec + (g & 1) * 32 + 8 * c);
      if (NT == 1) hcv[j][nt] = *reinterpret_cast<const int2*>(hb.hp + (sc * kSkHGroups + j) * kPlaneRec + 64);
    }
    he[nt] = hb.he[sc];
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(hb.h_free);
  return true;
}

// Consumers: the down stages of one unit, B operand = the unit's h planes in
// registers.  Writes ypart[pair][rb][row].  Returns false on a timeout.
template <int NT, int NS, int STAGE, int GROUP, int BITS>
__device__ __forceinline__ bool consume_down_slice(const FfnArgs& a, const TileInfo& ti, const uint8_t* smem,
                                                   uint64_t* full, uint64_t* empty, const SkHBufs& hb, int& s,
                                                   uint32_t& ph, uint32_t lu, volatile int* abort_flag, int warp,
                                                   int lane) {
  const int g = lane >> 2, c = lane & 3;
  uint2 hbv[kSkHGroups][NT];
  int2 hcv[kSkHGroups][NT];
  int he[NT];
  if (!load_h_planes<NT>(a, ti, hb, lu, hbv, hcv, he, abort_flag, warp, lane)) return false;
  float uf1[NT], uf2[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) pow2_split(-he[nt], uf1[nt], uf2[nt]);
  // the partials are read back by the combine at the end of the kernel
  const uint64_t ppol = l2_policy_evict_last();
  using D = SkDn<BITS>;
  const int nnt = (ti.ntok + 3) >> 2;
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
        float acc[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = 0.f;
#pragma unroll
        for (int j = 0; j < kSkHGroups; ++j) {
          uint32_t fa[4];
          if (BITS == 4) {
            const uint8_t* ca = cb + ((static_cast<uint32_t>(j) ^ sw) << 4);
            a_from_int4(fa, *reinterpret_cast<const uint32_t*>(ca), *reinterpret_cast<const uint32_t*>(ca + 8 * 64));
          } else {
            const uint8_t* ca = stg + bx * D::CODE + (cb8 ^ static_cast<uint32_t>((2 * j) << 4));
            a_from_int8(fa, *reinterpret_cast<const uint2*>(ca), *reinterpret_cast<const uint2*>(ca + 8 * 128));
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            if (NT == 1 || nt < nnt) {
              int d[4];
              // two n-tiles: the start values come from the plane records in
              // shared memory (unchanged until every warp has left this
              // unit's down stages), which saves 16 registers
              const int2 cv = NT == 1 ? hcv[j][nt]
                                      : *reinterpret_cast<const int2*>(hb.hp + ((nt * 4 + c) * kSkHGroups + j) * kPlaneRec + 64);
              mma_i8<BITS>(d, fa, hbv[j][nt], BITS == 4 ? cv.x : kPlaneMagic, BITS == 4 ? cv.y : kPlaneMagic);
              acc_group<BITS>(acc[nt][0], acc[nt][1], d, s0[j], s1[j]);
            }
          }
        }
        // acc[nt]: rows rl and rl + 8 of slot nt * 4 + c
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int i = nt * 4 + c;
          if (i < ti.ntok) {
            const size_t orow = static_cast<size_t>(ti.base + ti.i0 + i);
            float* yp = a.ypart + (orow * a.I / kRowBlock + ti.rb) * a.H + r0 + rl;
            st_f32_hint(yp, (acc[nt][0] * uf1[nt]) * uf2[nt], ppol);
            st_f32_hint(yp + 8, (acc[nt][1] * uf1[nt]) * uf2[nt], ppol);
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
  return true;
}

// Bounded wait of one lane for a global counter to reach `target`.
__device__ __forceinline__ bool wait_counter(const int32_t* cnt, int target, volatile int* abort_flag,
                                             uint32_t* status, uint64_t limit_ns = kWaitLimitNs) {
  if (ld_acquire_gpu(cnt) >= target) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (ld_acquire_gpu(cnt) >= target) return true;
    if ((it & 63u) == 0 && (*abort_flag || globaltimer() - t0 > limit_ns)) {
      if (!*abort_flag) atomicOr(status, COLI_FLAG_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

// The CTA's share of the output after every partial is in: a contiguous
// range of output units (token t, 4 rows r..r+3), in chunks that fit the
// idle stage ring.  Pass 1, one thread per (unit, pair slot j): y of the
// slot's pair (routed slot j < k, then the shared experts) as the sum of its
// I/128 partials in slice order, every load in flight before the first add,
// into the ring.  After a CTA barrier, pass 2, one thread per unit: the
// routed y's weighted in slot order, then the shared y's and the residual,
// rounded once to bf16.  pos / w: shared-memory copies of pair_pos and
// topk_w.  `cbar` (count: consumer warps) separates the passes; returns
// false on a timeout.
__device__ __forceinline__ bool splitk_combine(const FfnArgs& a, const int32_t* pos, const float* w,
                                               const int32_t* ids, uint8_t* ring, int ring_bytes, uint64_t* cbar,
                                               uint32_t& cph, volatile int* abort_flag, int warp, int lane) {
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
    for (int task = tid; task < cn * nj; task += nthr) {
      const int ui = task / nj, j = task - ui * nj;
      const int u = cu + ui;
      const int t = u / q4, r = (u - t * q4) * 4;
      const int row = j < a.k ? pos[t * a.k + j] : a.P + (j - a.k) * a.T + t;
      const float* src = a.ypart + static_cast<size_t>(row) * nsl * a.H + r;
      float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
      // an expert-parallel rank adds only the pairs of its own experts
      bool here = true;
      if (a.topk_ids && j < a.k) {
        const int e = ids ? ids[t * a.k + j] : __ldg(a.topk_ids + t * a.k + j);
        here = e >= a.e_off && e < a.e_end;
      }
      for (int s0 = 0; here && s0 < nsl; s0 += 16) {
        float4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          v[i] = s0 + i < nsl ? __ldcg(reinterpret_cast<const float4*>(src + static_cast<size_t>(s0 + i) * a.H))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          y.x += v[i].x;
          y.y += v[i].y;
          y.z += v[i].z;
          y.w += v[i].w;
        }
      }
      ysum[task] = y;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(cbar);
    if (!mbar_wait(cbar, cph, abort_flag, a.status)) return false;
    cph ^= 1u;
    for (int ui = tid; ui < cn; ui += nthr) {
      const int u = cu + ui;
      const int t = u / q4, r = (u - t * q4) * 4;
      uint2 rv = make_uint2(0u, 0u);
      if (a.residual) rv = __ldg(reinterpret_cast<const uint2*>(a.residual + static_cast<size_t>(t) * a.H + r));
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j = 0; j < a.k; ++j) {
        const float wj = w[t * a.k + j];
        const float4 y = ysum[ui * nj + j];
        acc.x = fmaf(wj, y.x, acc.x);
        acc.y = fmaf(wj, y.y, acc.y);
        acc.z = fmaf(wj, y.z, acc.z);
        acc.w = fmaf(wj, y.w, acc.w);
      }
      for (int s = 0; s < a.S; ++s) {
        const float4 y = ysum[ui * nj + a.k + s];
        acc.x += y.x;
        acc.y += y.y;
        acc.z += y.z;
        acc.w += y.w;
      }
      if (a.residual) {
        acc.x += __uint_as_float(rv.x << 16);
        acc.y += __uint_as_float(rv.x & 0xffff0000u);
        acc.z += __uint_as_float(rv.y << 16);
        acc.w += __uint_as_float(rv.y & 0xffff0000u);
      }
      if (a.out_f32) {
        *reinterpret_cast<float4*>(a.out_f32 + static_cast<size_t>(t) * a.H + r) = acc;
        continue;
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

// The split-K kernel's own routing (a.r_logits not NULL), kept out of line so
// that it does not change the code of the kernel's main loops.  Warp t routes
// token t (top-k, lowest index on ties, renormalised softmax); then warp 0
// sorts the pairs into the union and lays out the plan, all in shared memory.
// Every CTA computes the same from the same logits.
__device__ __noinline__ void splitk_route(const FfnArgs& a, const float* bias_s, int32_t* ids_s, float* w_s,
                                          int32_t* muniq, int32_t* n_unique_s, int32_t* mseg, int32_t* perm_s,
                                          int32_t* pos_s, int32_t* mplan, int warp, int lane) {
  const int P = a.T * a.k;
  __syncthreads();
  if (warp < a.T) {
    int id;
    float wt;
    const bool bad = route_token<8, true>(a.r_logits + static_cast<size_t>(warp) * a.E, a.r_bias ? bias_s : nullptr, a.E,
                                    a.k, lane, &id, &wt);
    if (lane < a.k) {
      ids_s[warp * a.k + lane] = id;
      w_s[warp * a.k + lane] = wt;
    }
    if (bad && blockIdx.x == 0 && lane == 0) atomicOr(a.status, COLI_FLAG_NONFINITE);
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t* st = blockIdx.x == 0 ? a.status : nullptr;
    if (P <= 32)
      warp_union_plan32(ids_s, P, a.E, a.T, a.S, a.tokb, muniq, n_unique_s, mseg, perm_s, pos_s, st, mplan, nullptr,
                        nullptr, 0, lane, a.e_off, a.e_end);
    else
      warp_union_plan(ids_s, P, a.E, a.T, a.S, a.tokb, muniq, n_unique_s, mseg, perm_s, pos_s, st, mplan, nullptr,
                      nullptr, 0, lane, a.e_off, a.e_end);
  }
}

// The split-K FFN kernel.  At most one CTA per SM, all resident (the final
// grid-wide wait needs that); a.rb_done[0] is the zeroed arrival counter.  NT: MMA
// n-tiles of four tokens (1 for T <= 4, 2 for T <= 8).  INROUTE: every CTA
// routes the batch from the router logits (a.r_logits) and builds the union and
// the tile plan itself; otherwise they come from earlier kernels.  Either way
// they are kept in shared memory.
template <int NT, int GROUP, int BITS, bool INROUTE>
__global__ void __launch_bounds__(kFfnThreads, 1)
    ffn_splitk_kernel(const __grid_constant__ CUtensorMap gq, const __grid_constant__ CUtensorMap uq,
                      const __grid_constant__ CUtensorMap gs, const __grid_constant__ CUtensorMap us,
                      const __grid_constant__ CUtensorMap dq, const __grid_constant__ CUtensorMap ds,
                      const FfnArgs a) {
  using F = SkCfg<GROUP, BITS>;
  constexpr int NS = F::NS, STAGE = F::STAGE;
  extern __shared__ uint8_t smem_raw[];
  // 1 KiB-aligned start, as an offset from smem_raw so that the compiler
  // keeps every pointer derived from it in the shared state space (ld.shared
  // / st.shared rather than generic accesses)
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* fixed = smem + NS * STAGE;
  float* red = reinterpret_cast<float*>(fixed);
  int32_t* meta = reinterpret_cast<int32_t*>(fixed + F::RED_BYTES);
  SkHBufs hb;
  hb.h = reinterpret_cast<uint16_t*>(fixed + F::RED_BYTES + F::META_BYTES);
  hb.hp = fixed + F::RED_BYTES + F::META_BYTES + F::H_BYTES;
  hb.hmax = reinterpret_cast<float*>(hb.hp + F::HP_BYTES);
  hb.he = reinterpret_cast<int*>(hb.hmax + kRowWarps * kSkMaxT);
  float* w_s = reinterpret_cast<float*>(hb.hp + F::HP_BYTES + F::HMAX_BYTES);
  int32_t* perm_s = reinterpret_cast<int32_t*>(w_s + kSkMaxP);
  int32_t* pos_s = perm_s + kSkMaxP;
  int32_t* ids_s = pos_s + kSkMaxP;
  int32_t* n_unique_s = ids_s + kSkMaxP;
  uint64_t* full = reinterpret_cast<uint64_t*>(hb.hp + F::HP_BYTES + F::HMAX_BYTES + F::ROUTE_BYTES);
  uint64_t* empty = full + NS;
  uint64_t* red_full = empty + NS;
  uint64_t* red_empty = red_full + kRowWarps;
  hb.h_ready = red_empty + kRowWarps;
  hb.hp_ready = hb.h_ready + 1;
  hb.h_free = hb.hp_ready + 1;
  uint64_t* cbar = hb.h_free + 1;
  uint64_t* gbar = cbar + 1;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + F::NBAR);
  int32_t* mplan = meta;
  int32_t* muniq = meta + kSkMaxSeg + 2;
  int32_t* mseg = muniq + kSkMaxSeg;

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
    mbar_init(hb.h_ready, kRowWarps);        // the K-half-0 warps write h
    mbar_init(hb.hp_ready, kSkHGroups);      // four warps write its planes
    mbar_init(hb.h_free, kFfnConsumerWarps);
    mbar_init(cbar, kFfnConsumerWarps);
    mbar_init(gbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // The tile plan puts the shared experts' units first, independent of the
  // routing: CTA b < S * I/128 starts with row block b % (I/128) of shared
  // expert E + b / (I/128), for all T tokens.  Those weights are no output of
  // an earlier kernel, so their first stages stream in while the kernel still
  // waits for its inputs.
  int pre = 0;
  const int nrb_gu = a.I / kRowBlock;
  if (warp == kFfnConsumerWarps) {
    if (lane == 0) {
      prefetch_tensormap(&gq);
      prefetch_tensormap(&uq);
      prefetch_tensormap(&dq);
    }
    if (static_cast<int>(blockIdx.x) < a.S * nrb_gu) {
      const int nkc = a.H / F::D::KCG;
      pre = nkc < NS ? nkc : NS;
      const int row0 = (a.e_shared + static_cast<int>(blockIdx.x) / nrb_gu) * a.I + (blockIdx.x % nrb_gu) * kRowBlock;
      if (lane == 0) {
        const uint64_t cpol = l2_policy_evict_first();
        for (int kc = 0; kc < pre; ++kc)
          gu_stage_weights<STAGE, GROUP, BITS>(a, row0, kc, a.T, &gq, &uq, &gs, &us, smem + kc * STAGE, &full[kc],
                                               cpol);
      }
    }
  }
  const int P = a.T * a.k;
  // the router bias is no output of an earlier kernel: staged before the wait
  float* bias_s = red;
  if (INROUTE && a.r_bias)
    for (int i = threadIdx.x; i < a.E; i += blockDim.x) bias_s[i] = __ldg(a.r_bias + i);
  pdl_wait();
  pdl_trigger();
  if constexpr (INROUTE) {
    splitk_route(a, bias_s, ids_s, w_s, muniq, n_unique_s, mseg, perm_s, pos_s, mplan, warp, lane);
  } else {
    // every array in one round of loads, up to its allocated size (the union
    // of P pairs has at most Umax = min(E, P) experts), not to the sizes the
    // routing kernel reports, so no load waits on another
    const int Umax = P < a.E ? P : a.E;
    if (threadIdx.x == 0) *n_unique_s = __ldg(a.n_unique);
    for (int i = threadIdx.x; i < Umax + a.S + 3; i += blockDim.x) mplan[i] = __ldg(a.plan + i);
    for (int i = threadIdx.x; i < Umax; i += blockDim.x) muniq[i] = __ldg(a.unique_ids + i);
    for (int i = threadIdx.x; i <= Umax; i += blockDim.x) mseg[i] = __ldg(a.seg_off + i);
    for (int i = threadIdx.x; i < P; i += blockDim.x) {
      perm_s[i] = __ldg(a.perm + i);
      pos_s[i] = __ldg(a.pair_pos + i);
      w_s[i] = __ldg(a.topk_w + i);
    }
  }
  __syncthreads();
  Meta m;
  m.plan = mplan;
  m.unique = muniq;
  m.seg_off = mseg;
  m.n_seg = mplan[0];
  m.U = *n_unique_s;
  m.S = m.n_seg - m.U;
  m.total_blocks = mplan[1];
  m.nrb_gu = nrb_gu;
  m.nrb_dn = a.H / kRowBlock;
  m.tiles_gu = m.total_blocks * m.nrb_gu;
  m.tiles_all = m.tiles_gu;

  if (warp == kFfnConsumerWarps) {
    // ---------------- producer ----------------
    int s = 0;
    uint32_t ph = 0;
    long issued = pre;
    bool ok = true;
    const uint64_t cpol = l2_policy_evict_first();
    for (int t = blockIdx.x; ok && t < m.tiles_gu; t += gridDim.x) {
      const TileInfo ti = decode_tile<8>(a, m, t);
      ok = produce_gu_slice<NS, STAGE, GROUP, BITS>(a, perm_s, ti, &gq, &uq, &gs, &us, smem, full, empty, s, ph,
                                                    issued, t == static_cast<int>(blockIdx.x) ? pre : 0, cpol,
                                                    abort_flag, lane);
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
  if (INROUTE && blockIdx.x == 0) {
    // publish the union and the plan this CTA built (plain stores: nothing
    // in this kernel reads them back)
    const int tid = threadIdx.x, nthr = kFfnConsumerWarps * 32;
    for (int i = tid; i < m.U; i += nthr) a.r_unique[i] = muniq[i];
    for (int i = tid; i <= m.U; i += nthr) a.r_seg_off[i] = mseg[i];
    for (int i = tid; i < m.n_seg + 3; i += nthr) a.r_plan[i] = mplan[i];
    for (int i = tid; i < P; i += nthr) {
      a.r_perm[i] = perm_s[i];
      a.r_pair_pos[i] = pos_s[i];
      a.r_ids[i] = ids_s[i];
      a.r_w[i] = w_s[i];
    }
    if (tid == 0) *a.r_n_unique = m.U;
  }
  int s = 0;
  uint32_t ph = 0, rph = 0, lu = 0;
  for (int t = blockIdx.x; t < m.tiles_gu; t += gridDim.x, ++lu) {
    const TileInfo ti = decode_tile<8>(a, m, t);
    if (!consume_gu_slice<NT, NS, STAGE, GROUP, BITS>(a, perm_s, ti, smem, red, full, empty, red_full, red_empty, hb,
                                                      s, ph, rph, lu, abort_flag, warp, lane))
      return;
    if (!consume_down_slice<NT, NS, STAGE, GROUP, BITS>(a, ti, smem, full, empty, hb, s, ph, lu, abort_flag, warp,
                                                        lane))
      return;
  }
  // publish: every warp fences its partials and checks in on the CTA barrier;
  // then one thread per CTA increments the grid counter and waits (bounded)
  // for every CTA, and releases the CTA's warps through gbar
  __threadfence();
  __syncwarp();
  if (lane == 0) mbar_arrive(cbar);
  if (!mbar_wait(cbar, 0, abort_flag, a.status)) return;
  if (warp == 0 && lane == 0) {
    __threadfence();
    atomicAdd(a.rb_done, 1);
    if (wait_counter(a.rb_done, static_cast<int>(gridDim.x), abort_flag, a.status)) mbar_arrive(gbar);
  }
  if (!mbar_wait(gbar, 0, abort_flag, a.status)) return;
  // (the combine's CTA barriers are cbar's next phases)
  uint32_t cph = 1;
  splitk_combine(a, pos_s, w_s, INROUTE ? ids_s : nullptr, smem, NS * STAGE, cbar, cph, abort_flag, warp, lane);
}

}  // namespace coli
