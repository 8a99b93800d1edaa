// Decode form of the int4 expert FFN and the routing-weighted combine: the
// two-phase kernel, used for batches of more than 8 tokens (and for I = 128);
// smaller batches take the split-K kernel of k_ffn_splitk.cuh, which reuses
// this file's stage configuration, producer and gate/up consumer.
//
// The routed experts are int4 (Colibri README, "L'idea": ~19 MB per expert in
// the int4 container; an expert's three matrices are the gate, up and down
// projections of a SwiGLU FFN).  With few tokens per expert the step is bound
// by reading the int4 weights, so this form streams them once at HBM rate in
// ONE persistent, cooperatively launched kernel (one CTA per SM):
//   * tiles are (segment, token block, 128-row block); every CTA first walks
//     its gate/up tiles, then its down tiles, so all CTAs stream weights
//     without a gap between the two projections;
//   * one producer warp moves, per stage, 128 rows x 256 K of codes (2-D
//     tensor-map copies, 128B swizzle), their fp16 scales and the stage's
//     slice of each token's activation row (1-D bulk copies) into a ring of
//     shared-memory stages;
//   * a down tile needs h of its token block from all gate/up row blocks: the
//     gate/up epilogue publishes each finished (token block, row block) with
//     a fence and an atomic increment; the down producer issues its weight
//     copies at once and waits (bounded) on that counter only before copying
//     the h rows;
//   * 16 consumer warps: warps w and w+8 own the same 16 rows and split every
//     stage's 32-wide groups between them; they add their partials once per
//     tile, in a fixed order;
//   * dequantisation of a pair of codes is one mask-and-magic LOP3 (nibble n
//     of the two's-complement code q becomes the bf16 value 128 + (n ^ 8) =
//     136 + q) and one exact bf16x2 subtract of 136; m16n8k16 bf16 mma.sync
//     multiplies the codes with up to 8 tokens per n-tile; each 32-wide
//     group's fp32 partial is multiplied by its fp16 scale and accumulated in
//     fp32.
// Gate/up writes h = bf16(silu(g) * u); down writes y (fp32) per (pair, row).
// The combine (each token's k routed y's with its routing weights, its shared
// experts and its residual, summed in a fixed order and rounded once to bf16)
// is done by the last down warp to finish a row block when T <= 4, and by
// combine_kernel otherwise.
#pragma once
#include "common.cuh"
#include "k_union.cuh"

namespace coli {

constexpr int kRowWarps = 8;                         // 16-row slices per tile
constexpr int kFfnConsumerWarps = 2 * kRowWarps;     // two K-halves per slice
constexpr int kFfnThreads = (kFfnConsumerWarps + 1) * 32;
constexpr int kRowBlock = 16 * kRowWarps;            // 128 rows per tile
constexpr int kMaxSeg = 1024 + 8;                    // unique routed + shared segments
constexpr int kFusedCombineMaxT = 4;

struct FfnArgs {
  const uint16_t* xq;        // fragment-ordered expert input [T][H]
  const uint8_t* xp;         // split-K form: integer planes of the expert input [T][H/32][kPlaneRec]
  const int32_t* xe;         // split-K form: grid exponent of each token's planes [T]
  uint16_t* hq;              // h, fragment-ordered [P+S*T][I]
  float* ypair;              // y [P+S*T][H]
  float* ypart;              // split-K form: y partials [P+S*T][I/128][H]
  const uint16_t* gate_s;    // scales for 1-D copies when a stage spans all of K
  const uint16_t* up_s;
  const uint16_t* down_s;
  const int32_t* unique_ids;
  const int32_t* n_unique;
  const int32_t* seg_off;
  const int32_t* perm;
  const int32_t* plan;       // [n_seg, total_blocks, tile_off[0..n_seg]]
  int32_t* tb_done;          // [total_blocks] gate/up warps finished per token block
  int32_t* rb_done;          // [H/128] down warps finished per row block (fused combine)
  const int32_t* pair_pos;   // for the fused combine
  const float* topk_w;
  const uint16_t* residual;
  uint16_t* out;
  uint32_t* status;
  int H, I, T, k, E, S, P;
  // expert-parallel rank (split-K form): the weights hold routed experts
  // [e_off, e_off + n) at rows 0.. and the S shared ones from expert e_shared
  // on; pairs whose expert (topk_ids) is not among them add nothing; with
  // out_f32 the output is the unrounded fp32 partial sum (else e_off = 0,
  // e_shared = E, topk_ids and out_f32 NULL)
  int e_off, e_end, e_shared;
  const int32_t* topk_ids;
  float* out_f32;
  // split-K form with the routing in the kernel (r_logits not NULL; T*k <=
  // 128 and E <= 256): the batch's router logits [T][E] and bias; every CTA
  // routes the batch and builds the union and the tile plan (tokb tokens per
  // block) in shared memory, and CTA 0 also writes them, the ids and the
  // weights to the arrays below.  With r_logits NULL they come from an
  // earlier kernel through the const pointers above.
  const float* r_logits;
  const float* r_bias;
  int32_t* r_ids;
  float* r_w;
  int32_t* r_unique;
  int32_t* r_n_unique;
  int32_t* r_seg_off;
  int32_t* r_perm;
  int32_t* r_pair_pos;
  int32_t* r_plan;
  int tokb;
};

// Shared-memory layout constants.  KC elements of K per stage; NT n-tiles of 8
// tokens per tile; NMAT matrices per stage (2 = gate+up, 1 = down).
// GROUP: K elements per fp16 scale (32, or 64 for the gs64 container).  BITS:
// 4 (int4 codes, two per byte) or 8 (int8 codes).  A stage with fewer than 8
// scales per row loads them as one 16-byte box of 8 (the smallest aligned TMA
// box): consecutive stages load the same box (the later ones from L2) and each
// reads its own part (BOX8).
template <int KC, int NT, int NMAT, int GROUP = 32, int BITS = 4>
struct StageCfg {
  static constexpr int TOKB = 8 * NT;
  static constexpr int GPW = KC / 64;                 // groups per warp per stage (two K-halves)
  static constexpr int ROWB = KC * BITS / 8;          // code bytes per row
  static constexpr int SUBS = ROWB >= 256 ? ROWB / 128 : 1;   // 128-byte-wide code sub-tiles per stage
  static constexpr int RSTR = ROWB / SUBS;            // row stride inside a code sub-tile
  static constexpr int SUB_BYTES = kRowBlock * RSTR;
  static constexpr int SPS = KC / GROUP;              // scales per row per stage
  static constexpr int SROWB = (GROUP == 32 && BITS == 4) ? KC / 16 : 16;   // scale bytes per row
  static constexpr bool BOX8 = SROWB == 16 && SPS < 8;
  static constexpr int CODE_BYTES = kRowBlock * ROWB;
  static constexpr int SC_BYTES = kRowBlock * SROWB;
  static constexpr int W_BYTES = NMAT * (CODE_BYTES + SC_BYTES);
  static constexpr int XROW = KC * 2 + 64;            // padded activation row (bank-conflict free)
  static constexpr int STAGE_USED = W_BYTES + TOKB * XROW;
  static constexpr bool SWZ = (ROWB >= 128);
  static_assert(CODE_BYTES % 1024 == 0 && SC_BYTES % 1024 == 0, "stage regions must stay 1 KiB aligned");
  static_assert(NMAT == 1 || KC <= 256, "wide stages are for the down projection only");
  static_assert(GROUP == 32 || (GROUP == 64 && KC >= 128), "64-wide groups need stages of 128 K or more");
  static_assert(BITS == 4 || (BITS == 8 && KC == 128 && NT == 1), "int8 stages: 128 K, one n-tile");
};

template <int NT, int KCD, int GROUP = 32>
struct FusedCfg {
  using GU = StageCfg<256, NT, 2, GROUP>;
  using DN = StageCfg<KCD, NT, 1, GROUP>;
  static constexpr int STAGE = ((GU::STAGE_USED > DN::STAGE_USED ? GU::STAGE_USED : DN::STAGE_USED) + 1023) / 1024 * 1024;
  static constexpr int RED_BYTES = kRowWarps * 32 * NT * 4 * 2 * 4;   // K-half partials (2 matrices)
  static constexpr int META_BYTES = (3 * kMaxSeg + 4) * 4;            // cached plan / unique / seg_off
  static constexpr int FIXED = RED_BYTES + META_BYTES + 1024 + 64 * 8 + 64;
  static constexpr int NS_RAW = (227 * 1024 - FIXED) / STAGE;
  static constexpr int NS = NS_RAW > 8 ? 8 : NS_RAW;
  static constexpr size_t SMEM = static_cast<size_t>(NS) * STAGE + FIXED;
  static_assert(NS >= 3, "pipeline depth");
  static_assert(SMEM <= 232448, "shared memory budget");
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

__device__ __forceinline__ void dq_word_pair(uint32_t (&p)[8], uint32_t w0, uint32_t w1) {
  p[0] = dq_pair(w0, 0); p[1] = dq_pair(w0, 4); p[2] = dq_pair(w0, 8); p[3] = dq_pair(w0, 12);
  p[4] = dq_pair(w1, 0); p[5] = dq_pair(w1, 4); p[6] = dq_pair(w1, 8); p[7] = dq_pair(w1, 12);
}

// int8 codes: q = 16 * hi + lo with hi the signed high nibble and lo the
// unsigned low nibble.  One word of 4 codes gives two bf16x2 pairs of each:
// (w >> sh) & 0x000F000F puts one nibble in each 16-bit half; under the
// exponent of 2048 (0x4500) the nibble n ^ 8 is worth 16 * (n ^ 8), and
// subtracting 2048 + 128 leaves 16 * hi exactly; under 128 (0x4300) the plain
// nibble is worth n, and subtracting 128 leaves lo.
__device__ __forceinline__ uint32_t dq_hi16(uint32_t w, int sh) {
  uint32_t r, q;
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(r) : "r"(w >> sh), "r"(0x000F000Fu), "r"(0x45084508u));
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(q) : "r"(r), "r"(0x45084508u));
  return q;
}

__device__ __forceinline__ uint32_t dq_lo(uint32_t w, int sh) {
  uint32_t r, q;
  asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(r) : "r"(w >> sh), "r"(0x000F000Fu), "r"(0x43004300u));
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(q) : "r"(r), "r"(0x43004300u));
  return q;
}

// 8 int8 codes c0..c7 of one row (two words) -> the pairs (c0,c4), (c1,c5),
// (c2,c6), (c3,c7) of 16 * hi and of lo, the same pairing (and activation
// fragment order) as the int4 codes of dq_word_pair.
__device__ __forceinline__ void dq8_row(uint32_t (&hi)[4], uint32_t (&lo)[4], uint2 v) {
  uint32_t w1, w2;
  asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(w1) : "r"(v.x), "r"(v.y));   // c0 c1 c4 c5
  asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(w2) : "r"(v.x), "r"(v.y));   // c2 c3 c6 c7
  hi[0] = dq_hi16(w1, 4);  lo[0] = dq_lo(w1, 0);
  hi[1] = dq_hi16(w1, 12); lo[1] = dq_lo(w1, 8);
  hi[2] = dq_hi16(w2, 4);  lo[2] = dq_lo(w2, 0);
  hi[3] = dq_hi16(w2, 12); lo[3] = dq_lo(w2, 8);
}

__device__ __forceinline__ void mma_16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
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

// One 32-wide group of int8 codes: rows g (h0, l0) and g + 8 (h1, l1); the
// 16*hi and lo parts of every code meet the same activation fragment.
template <bool SINGLE>
__device__ __forceinline__ void group_acc8(float (&acc)[4], const uint32_t (&h0)[4], const uint32_t (&h1)[4],
                                           const uint32_t (&l0)[4], const uint32_t (&l1)[4], const uint4& b,
                                           float s0, float s1) {
  float d[4] = {0.f, 0.f, 0.f, 0.f};
  mma_16816(d, h0[0], h1[0], h0[1], h1[1], b.x, b.y);
  mma_16816(d, h0[2], h1[2], h0[3], h1[3], b.z, b.w);
  mma_16816(d, l0[0], l1[0], l0[1], l1[1], b.x, b.y);
  mma_16816(d, l0[2], l1[2], l0[3], l1[3], b.z, b.w);
  acc[0] = fmaf(s0, d[0], acc[0]);
  acc[2] = fmaf(s1, d[2], acc[2]);
  if (!SINGLE) {
    acc[1] = fmaf(s0, d[1], acc[1]);
    acc[3] = fmaf(s1, d[3], acc[3]);
  }
}

__device__ __forceinline__ __half2 u32_as_half2(uint32_t v) {
  __half2 h;
  memcpy(&h, &v, 4);
  return h;
}

// N fp16 scales at p (N = 1, 2, 4, 8; p aligned to 2N bytes) as half2 pairs.
template <int N>
__device__ __forceinline__ void load_scales(const uint8_t* p, __half2 (&h)[4]) {
  if (N == 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    h[0] = u32_as_half2(v.x); h[1] = u32_as_half2(v.y); h[2] = u32_as_half2(v.z); h[3] = u32_as_half2(v.w);
  } else if (N == 4) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    h[0] = u32_as_half2(v.x); h[1] = u32_as_half2(v.y);
  } else if (N == 2) {
    h[0] = u32_as_half2(*reinterpret_cast<const uint32_t*>(p));
  } else {
    const uint32_t x = *reinterpret_cast<const uint16_t*>(p);
    h[0] = u32_as_half2(x | (x << 16));
  }
}

__device__ __forceinline__ float half2_pick(const __half2& h, int hi) {
  return hi ? __high2float(h) : __low2float(h);
}

__device__ __forceinline__ int ld_acquire_gpu(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Tile geometry shared by producer and consumers.
struct Meta {
  const int32_t* plan;      // shared copy: [n_seg, total_blocks, tile_off...]
  const int32_t* unique;    // shared copy
  const int32_t* seg_off;   // shared copy
  int n_seg, U, S, total_blocks, nrb_gu, nrb_dn, tiles_gu, tiles_all;
};

struct TileInfo {
  int tbg, rb, e, base, cnt, i0, ntok;
  bool routed, down;
};

template <int TOKB>
__device__ __forceinline__ TileInfo decode_tile(const FfnArgs& a, const Meta& m, int tile) {
  TileInfo ti;
  ti.down = tile >= m.tiles_gu;
  const int t = ti.down ? tile - m.tiles_gu : tile;
  const int nrb = ti.down ? m.nrb_dn : m.nrb_gu;
  ti.tbg = t / nrb;
  ti.rb = t - ti.tbg * nrb;
  int lo = 0, hi = m.n_seg - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (m.plan[2 + mid] <= ti.tbg) lo = mid; else hi = mid - 1;
  }
  const int tb = ti.tbg - m.plan[2 + lo];
  if (lo >= m.S) {
    const int u = lo - m.S;
    ti.routed = true;
    ti.e = m.unique[u] - a.e_off;
    ti.base = m.seg_off[u];
    ti.cnt = m.seg_off[u + 1] - ti.base;
  } else {
    ti.routed = false;
    ti.e = a.e_shared + lo;
    ti.base = a.P + lo * a.T;
    ti.cnt = a.T;
  }
  ti.i0 = tb * TOKB;
  ti.ntok = min(TOKB, ti.cnt - ti.i0);
  return ti;
}

// Bounded wait of the producer lane for a token block's h to be complete.
__device__ __forceinline__ bool wait_h_ready(const FfnArgs& a, int tbg, int target, volatile int* abort_flag) {
  const int32_t* cnt = a.tb_done + tbg;
  bool ok = true;
  if (ld_acquire_gpu(cnt) < target) {
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
      if (ld_acquire_gpu(cnt) >= target) break;
      if ((it & 63u) == 0 && (*abort_flag || globaltimer() - t0 > kWaitLimitNs)) {
        if (!*abort_flag) atomicOr(a.status, COLI_FLAG_TIMEOUT);
        *abort_flag = 1;
        ok = false;
        break;
      }
      __nanosleep(64);
    }
  }
  // h was written through the generic proxy; the bulk copies read it through the async proxy
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return ok;
}

// Producer: fills the stages of one tile.  For a down tile the weight copies
// go out immediately; the h rows wait (bounded) for the tile's token block to
// be complete in gate/up.  Returns false on a timeout.
template <int KC, int NT, int NMAT, int NS, int STAGE, int GROUP, int BITS = 4>
__device__ __forceinline__ bool produce_tile(const FfnArgs& a, const TileInfo& ti, const CUtensorMap* mq0,
                                             const CUtensorMap* mq1, const CUtensorMap* ms0, const CUtensorMap* ms1,
                                             const uint16_t* s0_1d, const uint16_t* s1_1d, int K, int R, int nrb_gu,
                                             uint8_t* smem, uint64_t* full, uint64_t* empty, int& s, uint32_t& ph,
                                             long& issued, volatile int* abort_flag, int lane) {
  using C = StageCfg<KC, NT, NMAT, GROUP, BITS>;
  const int row0 = ti.e * R + ti.rb * kRowBlock;
  const int nkc = K / KC;
  const uint16_t* bsrc = a.xq;
  if (lane < ti.ntok) {
    const int i = ti.i0 + lane;
    if (!ti.down) {
      const int tok = ti.routed ? __ldg(a.perm + ti.base + i) / a.k : i;
      bsrc = a.xq + static_cast<size_t>(tok) * K;
    } else {
      bsrc = a.hq + static_cast<size_t>(ti.base + i) * K;
    }
  }
  const int target = nrb_gu * kRowWarps;
  bool b_ready = !ti.down;
  int pend_s[8], pend_kc[8];
  int npend = 0;
  for (int kc = 0; kc < nkc; ++kc) {
    // a slot still in use would only free up once the consumers have the
    // pending h rows: resolve them before blocking on it
    if (!b_ready && npend > 0) {
      bool free_now = false;
      if (lane == 0) free_now = mbar_try_wait(&empty[s], ph ^ 1u);
      free_now = __shfl_sync(0xffffffffu, free_now, 0);
      if (!free_now || npend == 8) {
        bool ok = true;
        if (lane == 0) ok = wait_h_ready(a, ti.tbg, target, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) return false;
        b_ready = true;
        __syncwarp();
        for (int q = 0; q < npend; ++q)
          if (lane < ti.ntok)
            bulk_load(smem + pend_s[q] * STAGE + C::W_BYTES + lane * C::XROW, bsrc + pend_kc[q] * KC, KC * 2,
                      &full[pend_s[q]]);
        npend = 0;
      }
    }
    bool ok = true;
    if (lane == 0) ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, a.status);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) return false;
    uint8_t* st = smem + s * STAGE;
    if (lane == 0) {
      mbar_arrive_expect_tx(&full[s], C::W_BYTES + ti.ntok * KC * 2);
#pragma unroll
      for (int sb = 0; sb < C::SUBS; ++sb)
        tma_load_2d(st + sb * C::SUB_BYTES, mq0, &full[s], kc * C::ROWB + sb * C::RSTR, row0);
      if (NMAT == 2) tma_load_2d(st + C::CODE_BYTES, mq1, &full[s], kc * C::ROWB, row0);
      uint8_t* sc = st + NMAT * C::CODE_BYTES;
      if (KC == K) {
        bulk_load(sc, s0_1d + static_cast<size_t>(row0) * (K / GROUP), C::SC_BYTES, &full[s]);
        if (NMAT == 2)
          bulk_load(sc + C::SC_BYTES, s1_1d + static_cast<size_t>(row0) * (K / GROUP), C::SC_BYTES, &full[s]);
      } else {
        const int sx = C::BOX8 ? ((kc * C::SPS) & ~7) : kc * C::SPS;
        tma_load_2d(sc, ms0, &full[s], sx, row0);
        if (NMAT == 2) tma_load_2d(sc + C::SC_BYTES, ms1, &full[s], sx, row0);
      }
    }
    __syncwarp();
    if (b_ready) {
      if (lane < ti.ntok) bulk_load(st + C::W_BYTES + lane * C::XROW, bsrc + kc * KC, KC * 2, &full[s]);
    } else {
      pend_s[npend] = s;
      pend_kc[npend] = kc;
      ++npend;
    }
    ++issued;
    if (++s == NS) {
      s = 0;
      ph ^= 1u;
    }
  }
  if (npend > 0) {
    // every stage of the tile is out: wait for h and send the pending rows
    bool ok = true;
    if (lane == 0) ok = wait_h_ready(a, ti.tbg, target, abort_flag);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) return false;
    __syncwarp();
    for (int q = 0; q < npend; ++q)
      if (lane < ti.ntok)
        bulk_load(smem + pend_s[q] * STAGE + C::W_BYTES + lane * C::XROW, bsrc + pend_kc[q] * KC, KC * 2,
                  &full[pend_s[q]]);
  }
  return true;
}

// Combine of one 128-row block for all T tokens by one warp (T <= 4):
// out[t, r] = bf16( sum_j w[t,j] * y[pair_pos[t*k+j], r] + sum_s y[P+s*T+t, r] + residual[t, r] ).
__device__ __forceinline__ void warp_combine_rows(const FfnArgs& a, int rb, int lane) {
  const int r = rb * kRowBlock + lane * 4;
  for (int t = 0; t < a.T; ++t) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    // issue the loads of up to 8 routed slots at once, then add them in slot order
    for (int j0 = 0; j0 < a.k; j0 += 8) {
      int pp[8];
      float wt[8];
      float4 y[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int j = j0 + q;
        pp[q] = j < a.k ? a.pair_pos[t * a.k + j] : -1;
        wt[q] = j < a.k ? a.topk_w[t * a.k + j] : 0.f;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q)
        y[q] = pp[q] >= 0 ? __ldcg(reinterpret_cast<const float4*>(a.ypair + static_cast<size_t>(pp[q]) * a.H + r))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (pp[q] >= 0) {
          acc.x = fmaf(wt[q], y[q].x, acc.x);
          acc.y = fmaf(wt[q], y[q].y, acc.y);
          acc.z = fmaf(wt[q], y[q].z, acc.z);
          acc.w = fmaf(wt[q], y[q].w, acc.w);
        }
      }
    }
    for (int s = 0; s < a.S; ++s) {
      const float4 y =
          __ldcg(reinterpret_cast<const float4*>(a.ypair + static_cast<size_t>(a.P + s * a.T + t) * a.H + r));
      acc.x += y.x;
      acc.y += y.y;
      acc.z += y.z;
      acc.w += y.w;
    }
    if (a.residual) {
      const uint2 rv = *reinterpret_cast<const uint2*>(a.residual + static_cast<size_t>(t) * a.H + r);
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
}

// Consumers: one tile.  Returns false on a timeout.
template <int KC, int NT, int NMAT, bool SINGLE, int NS, int STAGE, int GROUP, int BITS = 4>
__device__ __forceinline__ bool consume_tile(const FfnArgs& a, const Meta& m, const TileInfo& ti, int K, int R,
                                             uint8_t* smem, float* red, uint64_t* full, uint64_t* empty,
                                             uint64_t* red_full, uint64_t* red_empty, int& s, uint32_t& ph,
                                             uint32_t& rph, volatile int* abort_flag, int warp, int lane) {
  using C = StageCfg<KC, NT, NMAT, GROUP, BITS>;
  const int rw = warp & (kRowWarps - 1);   // 16-row slice
  const int half = warp / kRowWarps;       // which half of each stage's groups
  const int g = lane >> 2, c = lane & 3;
  const int rl0 = 16 * rw + g;             // tile-local rows rl0 and rl0 + 8
  // Byte offset of this thread's code word in group 0 of row rl0.  With the
  // 128B swizzle the 16-byte chunk j of row r sits at chunk j ^ (r & 7), and
  // rl0 & 7 == (rl0 + 8) & 7 == g; bits 4..6 of cbase hold g, so chunk j is
  // cbase ^ (j << 4).
  // int8: thread c's 8 bytes of a group (codes 8c .. 8c+7, the int4 codes'
  // ownership) are 16-byte chunk 2j + (c >> 1), bytes 8 (c & 1) ..; with the
  // swizzle that chunk is (2j) ^ (g ^ (c >> 1)).
  const uint32_t cbase = BITS == 4 ? rl0 * C::RSTR + (C::SWZ ? (g << 4) : 0) + 4 * c
                                   : rl0 * C::RSTR + ((g ^ (c >> 1)) << 4) + 8 * (c & 1);
  // this half's scales: SPH fp16 values (its GPW 32-wide sub-groups share
  // them when GROUP is 64)
  constexpr int SPH = C::GPW * 32 / GROUP;
  const uint32_t sbase = rl0 * C::SROWB + half * SPH * 2;
  const uint32_t xbase = C::W_BYTES + g * C::XROW + (half * C::GPW * 32 + 8 * c) * 2;
  const int nnt = (ti.ntok + 7) >> 3;
  const int nkc = K / KC;
  float acc0[NT][4], acc1[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc0[nt][q] = 0.f;
      acc1[nt][q] = 0.f;
    }

  for (int kc = 0; kc < nkc; ++kc) {
    if (!mbar_wait(&full[s], ph, abort_flag, a.status)) return false;
    const uint8_t* st = smem + s * STAGE;
    const uint8_t* sc = st + NMAT * C::CODE_BYTES + sbase;
    // this warp's fp16 scales for its GPW groups (rows rl0 and rl0 + 8, both matrices)
    __half2 sh0[4], sh1[4], th0[4], th1[4];
    {
      const uint8_t* sq = sc + (C::BOX8 ? ((kc * C::SPS) & 7) * 2 : 0);
      load_scales<SPH>(sq, sh0);
      load_scales<SPH>(sq + 8 * C::SROWB, sh1);
      if (NMAT == 2) {
        load_scales<SPH>(sq + C::SC_BYTES, th0);
        load_scales<SPH>(sq + C::SC_BYTES + 8 * C::SROWB, th1);
      }
    }
#pragma unroll
    for (int jj = 0; jj < C::GPW; ++jj) {
      const int j = half * C::GPW + jj;                       // group within the stage
      const int si = GROUP == 32 ? jj : (jj >> 1);            // this sub-group's scale among the half's
      const float s0 = half2_pick(sh0[si >> 1], si & 1);
      const float s1 = half2_pick(sh1[si >> 1], si & 1);
      float t0 = 0.f, t1 = 0.f;
      if (NMAT == 2) {
        t0 = half2_pick(th0[si >> 1], si & 1);
        t1 = half2_pick(th1[si >> 1], si & 1);
      }
      if (BITS == 4) {
        const int jc = C::SUBS == 1 ? j : (j & 7);            // 16-byte chunk within the sub-tile row
        const uint8_t* ca = st + (C::SUBS == 1 ? 0 : (j >> 3) * C::SUB_BYTES) + (cbase ^ static_cast<uint32_t>(jc << 4));
        const uint32_t w0 = *reinterpret_cast<const uint32_t*>(ca);
        const uint32_t w1 = *reinterpret_cast<const uint32_t*>(ca + 8 * C::RSTR);
        uint32_t pg[8], pu[8];
        dq_word_pair(pg, w0, w1);
        if (NMAT == 2) {
          const uint32_t v0 = *reinterpret_cast<const uint32_t*>(ca + C::CODE_BYTES);
          const uint32_t v1 = *reinterpret_cast<const uint32_t*>(ca + C::CODE_BYTES + 8 * C::RSTR);
          dq_word_pair(pu, v0, v1);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (NT == 1 || nt < nnt) {
            uint4 b = make_uint4(0u, 0u, 0u, 0u);
            if (nt * 8 + g < ti.ntok) b = *reinterpret_cast<const uint4*>(st + xbase + nt * 8 * C::XROW + jj * 64);
            group_acc<SINGLE>(acc0[nt], pg, b, s0, s1);
            if (NMAT == 2) group_acc<SINGLE>(acc1[nt], pu, b, t0, t1);
          }
        }
      } else {
        const uint8_t* ca = st + (cbase ^ static_cast<uint32_t>((2 * j) << 4));
        uint32_t h0[4], h1[4], l0[4], l1[4];
        dq8_row(h0, l0, *reinterpret_cast<const uint2*>(ca));
        dq8_row(h1, l1, *reinterpret_cast<const uint2*>(ca + 8 * C::RSTR));
        uint4 b = make_uint4(0u, 0u, 0u, 0u);
        if (g < ti.ntok) b = *reinterpret_cast<const uint4*>(st + xbase + jj * 64);
        group_acc8<SINGLE>(acc0[0], h0, h1, l0, l1, b, s0, s1);
        if (NMAT == 2) {
          dq8_row(h0, l0, *reinterpret_cast<const uint2*>(ca + C::CODE_BYTES));
          dq8_row(h1, l1, *reinterpret_cast<const uint2*>(ca + C::CODE_BYTES + 8 * C::RSTR));
          group_acc8<SINGLE>(acc1[0], h0, h1, l0, l1, b, t0, t1);
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

  // Add the two K-halves of each 16-row slice (fixed order: half 0 + half 1),
  // handing the partials over through shared memory under bounded waits.
  float* rp = red + (rw * 32 + lane) * (NT * 4 * 2);
  if (half == 1) {
    if (!mbar_wait(&red_empty[rw], rph ^ 1u, abort_flag, a.status)) return false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        rp[nt * 4 + q] = acc0[nt][q];
        if (NMAT == 2) rp[NT * 4 + nt * 4 + q] = acc1[nt][q];
      }
    mbar_arrive(&red_full[rw]);
    rph ^= 1u;
    return true;
  }
  if (!mbar_wait(&red_full[rw], rph, abort_flag, a.status)) return false;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc0[nt][q] += rp[nt * 4 + q];
      if (NMAT == 2) acc1[nt][q] += rp[NT * 4 + nt * 4 + q];
    }
  mbar_arrive(&red_empty[rw]);
  rph ^= 1u;
  // epilogue: d0 (row g, col 2c), d1 (row g, col 2c+1), d2 (row g+8, col 2c), d3 (row g+8, col 2c+1)
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    if (nt < nnt) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = ti.i0 + nt * 8 + 2 * c + (q & 1);
        if (i < ti.cnt && !(SINGLE && (q & 1))) {
          const size_t orow = static_cast<size_t>(ti.base + i);
          const int r = ti.rb * kRowBlock + rl0 + ((q & 2) ? 8 : 0);
          if (NMAT == 2) {
            const float gv = acc0[nt][q], uv = acc1[nt][q];
            const float hv = gv / (1.0f + expf(-gv)) * uv;
            a.hq[orow * R + frag_pos(r)] = float_to_bf16_bits(hv);
          } else {
            a.ypair[orow * R + r] = acc0[nt][q];
          }
        }
      }
    }
  }
  // publish: every lane's stores, then one increment per warp
  __threadfence();
  __syncwarp();
  if (NMAT == 2) {
    if (lane == 0) atomicAdd(a.tb_done + ti.tbg, 1);
  } else if (a.T <= kFusedCombineMaxT) {
    int old = 0;
    if (lane == 0) old = atomicAdd(a.rb_done + ti.rb, 1);
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old + 1 == m.total_blocks * kRowWarps) {   // last warp of this row block
      __threadfence();
      warp_combine_rows(a, ti.rb, lane);
    }
  }
  return true;
}

// The persistent FFN kernel (gate/up tiles, then down tiles).  Launched
// cooperatively so that every CTA is resident: a down tile only waits for
// gate/up tiles, which every CTA processes before any of its down tiles.
template <int NT, bool SINGLE, int KCD, int GROUP>
__global__ void __launch_bounds__(kFfnThreads, 1)
    ffn_fused_kernel(const __grid_constant__ CUtensorMap gq, const __grid_constant__ CUtensorMap uq,
                     const __grid_constant__ CUtensorMap gs, const __grid_constant__ CUtensorMap us,
                     const __grid_constant__ CUtensorMap dq, const __grid_constant__ CUtensorMap ds,
                     const FfnArgs a) {
  using F = FusedCfg<NT, KCD, GROUP>;
  constexpr int NS = F::NS, STAGE = F::STAGE;
  extern __shared__ uint8_t smem_raw[];
  // 1 KiB-aligned start, as an offset from smem_raw so that the compiler
  // keeps every pointer derived from it in the shared state space (ld.shared
  // / st.shared rather than generic accesses)
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  float* red = reinterpret_cast<float*>(smem + NS * STAGE);
  int32_t* meta = reinterpret_cast<int32_t*>(smem + NS * STAGE + F::RED_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NS * STAGE + F::RED_BYTES + F::META_BYTES);
  uint64_t* empty = full + NS;
  uint64_t* red_full = empty + NS;
  uint64_t* red_empty = red_full + kRowWarps;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(red_empty + kRowWarps);

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
  // cache the plan, the unique experts and their segment offsets
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
    m.tiles_all = m.tiles_gu + m.total_blocks * m.nrb_dn;
  }
  __syncthreads();
  constexpr int TOKB = 8 * NT;

  if (warp == kFfnConsumerWarps) {
    // ---------------- producer ----------------
    int s = 0;
    uint32_t ph = 0;
    long issued = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < m.tiles_all; tile += gridDim.x) {
      const TileInfo ti = decode_tile<TOKB>(a, m, tile);
      if (!ti.down)
        ok = produce_tile<256, NT, 2, NS, STAGE, GROUP>(a, ti, &gq, &uq, &gs, &us, a.gate_s, a.up_s, a.H, a.I, m.nrb_gu,
                                                 smem, full, empty, s, ph, issued, abort_flag, lane);
      else
        ok = produce_tile<KCD, NT, 1, NS, STAGE, GROUP>(a, ti, &dq, &dq, &ds, &ds, a.down_s, a.down_s, a.I, a.H, m.nrb_gu,
                                                 smem, full, empty, s, ph, issued, abort_flag, lane);
    }
    if (!ok && lane == 0) {
      // Wait (bounded, ignoring the abort flag) for the copies still in flight
      // so none lands after this CTA has exited.
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
  uint32_t ph = 0, rph = 0;
  for (int tile = blockIdx.x; tile < m.tiles_all; tile += gridDim.x) {
    const TileInfo ti = decode_tile<TOKB>(a, m, tile);
    bool ok;
    if (!ti.down)
      ok = consume_tile<256, NT, 2, SINGLE, NS, STAGE, GROUP>(a, m, ti, a.H, a.I, smem, red, full, empty, red_full,
                                                        red_empty, s, ph, rph, abort_flag, warp, lane);
    else
      ok = consume_tile<KCD, NT, 1, SINGLE, NS, STAGE, GROUP>(a, m, ti, a.I, a.H, smem, red, full, empty, red_full,
                                                        red_empty, s, ph, rph, abort_flag, warp, lane);
    if (!ok) return;
  }
}

// out[t, n] = bf16( sum_{j<k} w[t,j] * y[pair_pos[t*k+j], n] + sum_s y[P + s*T + t, n]
//                   + residual[t, n] ), fp32, in exactly this order.  With ids (an
// expert-parallel rank) only the slots whose expert is in [eb, ee) are added;
// with out_f32 the fp32 sum is written there, unrounded, instead of out.
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ ypair,
                                                      const int32_t* __restrict__ pair_pos,
                                                      const float* __restrict__ w,
                                                      const uint16_t* __restrict__ residual, int T, int k,
                                                      int S, int H, uint16_t* __restrict__ out,
                                                      const int32_t* __restrict__ ids, int eb, int ee,
                                                      float* __restrict__ out_f32) {
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
    // issue the loads of up to 8 routed slots at once, then add them in slot order
    for (int j0 = 0; j0 < k; j0 += 8) {
      int pp[8];
      float wt[8];
      float4 y[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int j = j0 + q;
        pp[q] = j < k ? __ldg(pair_pos + t * k + j) : -1;
        wt[q] = j < k ? __ldg(w + t * k + j) : 0.f;
        if (ids && j < k) {
          // an expert-parallel rank adds only the pairs of its own experts
          const int e = __ldg(ids + t * k + j);
          if (e < eb || e >= ee) pp[q] = -1;
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q)
        y[q] = pp[q] >= 0 ? __ldg(reinterpret_cast<const float4*>(ypair + static_cast<size_t>(pp[q]) * H + n))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (pp[q] >= 0) {
          acc.x = fmaf(wt[q], y[q].x, acc.x);
          acc.y = fmaf(wt[q], y[q].y, acc.y);
          acc.z = fmaf(wt[q], y[q].z, acc.z);
          acc.w = fmaf(wt[q], y[q].w, acc.w);
        }
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
    if (out_f32) {
      *reinterpret_cast<float4*>(out_f32 + static_cast<size_t>(t) * H + n) = acc;
      continue;
    }
    uint2 o;
    o.x = float_to_bf16_bits(acc.x) | (static_cast<uint32_t>(float_to_bf16_bits(acc.y)) << 16);
    o.y = float_to_bf16_bits(acc.z) | (static_cast<uint32_t>(float_to_bf16_bits(acc.w)) << 16);
    *reinterpret_cast<uint2*>(out + static_cast<size_t>(t) * H + n) = o;
  }
}

}  // namespace coli
