// Prefill form of the int4 expert FFN: a tcgen05 grouped GEMM per projection.
//
// With many tokens per expert (a prefill chunk: ~128 tokens on each of the
// 256 experts) the expert matmuls are dense contractions and belong on the
// 5th-generation tensor cores.  One persistent CTA per SM walks tiles of
// (segment, token block of <= 160 tokens, 128 weight rows); segments are the
// union's experts followed by the shared ones.  Per tile and 64-wide K chunk:
//   * the producer warp copies the chunk's codes and fp16 group scales
//     (2-D tensor maps, 4 chunks per copy) and the token rows (fp16, 128B
//     swizzle) into two shared-memory rings;
//   * 16 dequantisation warps, one weight row per thread, turn the codes into
//     fp16 q*s (one mask-and-magic LOP3, one f16x2 subtract, one f16x2
//     multiply per pair of codes: q exact, q*s rounded once to 11 bits) and
//     store them straight into tensor memory with tcgen05.st: the weights are
//     the MMA's A operand *in TMEM*, so they never pass through shared memory;
//   * one thread issues tcgen05.mma (kind::f16, M = 128 weight rows, N =
//     the tile's tokens rounded up to 16, K = 16) from A in TMEM and the
//     token tile in shared memory into fp32 accumulators in TMEM, and
//     releases A buffers and token stages with tcgen05.commit;
//   * the same 16 warps read the accumulators back (tcgen05.ld) and write
//     h = bf16(silu(g) * u) (gate/up launch; stored as the fp16 of that bf16
//     value, which is exact) or y in fp32 (down launch).
// Both MMA operands are fp16 (kind::f16 takes one type for A and B): the
// expert input rows are the fp16 copies of their bf16 values (exact from
// 2^-17 up; COLI_FLAG_RANGE marks a value of 65536 or more, which fp16
// cannot hold), and h likewise.
// A tile of the gate/up launch holds the same 128 rows of both matrices; a
// tile of the down launch holds two neighbouring 128-row blocks of W_down.
// Either way two weight blocks share each token tile, which halves the
// token-tile traffic per MMA (one block per tile would need ~60 B/cycle of
// TMA per SM for a 160-token tile, above what the TMA engine delivers).
// The activations are gathered into pair order first, so a token tile is a
// plain row range of a 2-D tensor map.  Both operands use the same
// permutation of K inside every 8-element block (x0 x4 x1 x5 ...), which
// leaves every dot product unchanged.
#pragma once
#include "common.cuh"
#include "k_ffn_decode.cuh"

namespace coli {

constexpr int kPfTeams = 2;       // dequantisation teams of 8 warps; team t takes chunks t, t+2, ...
constexpr int kPfDqWarps = 8 * kPfTeams;
constexpr int kPfThreads = (4 + kPfDqWarps) * 32;   // warp 0 weight TMA, warp 1 MMA + TMEM owner, warp 2 token
                                                    // TMA, warps 4.. dequant + epilogue
constexpr int kPfMaxN = 160;      // tokens per tile (MMA N is this rounded up to 16)
constexpr int kPfAutoMinT = 32;   // smallest batch for which the form is chosen by default
constexpr int kPfTmemCols = 512;

struct PfArgs {
  const int32_t* plan;        // [n_seg, total_blocks, blk_off[0..n_seg]]
  const int32_t* unique_ids;
  const int32_t* n_unique;
  const int32_t* seg_off;
  const uint16_t* s0;         // scales of matrix 0 / 1, for 1-D copies when one stage spans K
  const uint16_t* s1;
  uint16_t* hq;               // gate/up output: h, fragment-ordered [P+S*T][I]
  float* ypair;               // down output: y [P+S*T][H]
  uint32_t* status;
  int H, I, T, k, E, S, P;
  // expert-parallel rank: the weights hold routed experts [e_off, ...) at rows
  // 0.. and the S shared ones from expert e_shared on (else 0 and E)
  int e_off, e_shared;
};

// Shared-memory / TMEM plan of one launch.  NMAT weight blocks per tile share
// the token tile: gate and up, or two row blocks of down (NMAT = 1: one down
// row block).
template <int NMAT>
struct PfCfg {
  static constexpr int CODE_SLOT = kRowBlock * 128;                 // codes of one matrix, 4 chunks
  static constexpr int SC_SLOT = kRowBlock * 16;                    // scales of one matrix, 4 chunks
  static constexpr int CSTAGE = NMAT * (CODE_SLOT + SC_SLOT);
  static constexpr int BSTAGE = kPfMaxN * 128;                      // token tile of one chunk
  // A chunk slot = one A buffer in TMEM + one token-tile stage in shared
  // memory, released together by one tcgen05.commit.
  static constexpr int NSC = 4;
  static constexpr int NBUF = NMAT == 2 ? 3 : 6;                    // chunk slots
  static constexpr int NSB = NBUF;
  // Accumulator buffers: two for the down GEMM, so that the epilogue of one
  // tile overlaps the MMAs of the next; gate/up needs both of its matrices'
  // accumulators and has room for one set only.
  static constexpr int ACC_BUFS = NMAT == 1 ? 2 : 1;
  static constexpr int ACOL = ACC_BUFS * NMAT * kPfMaxN;            // first A column
  static constexpr int META_INTS = 3 * kMaxSeg + 4;
  static constexpr int NBAR = 2 * NSC + NSB + 2 * NBUF + 2 * ACC_BUFS + 1;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(NSC) * CSTAGE + static_cast<size_t>(NSB) * BSTAGE +
                                 META_INTS * 4 + NBAR * 8 + 16;
  static_assert(CSTAGE % 1024 == 0 && BSTAGE % 1024 == 0, "stage alignment");
  static_assert(ACOL + NBUF * 32 * NMAT <= kPfTmemCols, "tensor memory budget");
  static_assert(SMEM <= 232448, "shared memory budget");
};

// ---------------------------------------------------------------- tcgen05 --

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Warp-wide: allocate `ncols` TMEM columns, base address written to smem.
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols) : "memory");
}

// The mbarrier receives one arrival once every tcgen05.mma issued so far by
// this thread has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// D[128 x N] (+)= A[128 x 16] * B[N x 16]^T; A in TMEM, B K-major in smem.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Shared-memory matrix descriptor: K-major rows of 128 bytes, 128-byte
// swizzle, 8-row groups 1024 bytes apart, descriptor version 1.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor of kind::f16: fp16 A and B (both K-major; type
// fields 0), fp32 accumulate, M = 128, N = n.
__device__ __forceinline__ uint32_t idesc_f16_m128(int n) {
  return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr)
               : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Two code nibbles (e_i, e_{i+4}) of word w -> exact f16x2 (q_i, q_{i+4}):
// (w >> sh) & 0x000F000F keeps one nibble per 16-bit half; XOR with 0x6408
// puts it under the exponent of 1024 and flips bit 3, giving 1024 + (n ^ 8)
// = 1032 + q; subtracting 1032 leaves q.
__device__ __forceinline__ uint32_t dq_pair_f16(uint32_t w, int sh) {
  uint32_t r, q;
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(r) : "r"(w >> sh), "r"(0x000F000Fu), "r"(0x64086408u));
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(q) : "r"(r), "r"(0x64086408u));
  return q;
}

// f16x2 a * b, rounded to nearest even.
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}


// ------------------------------------------------------------- tile plan --

struct PfTile {
  int e;        // expert id (shared experts E..E+S-1)
  int rblk;     // 128-row block of the output
  int ntok;     // tokens in the tile
  int npad;     // ntok rounded up to 16 (MMA N)
  int brow;     // first row of the tile's B operand rows
  int orow;     // first output row (pair order)
};

// Tile t of a launch with `mb` row blocks.  plan/unique/seg_off are the
// shared-memory copies.
template <bool DOWN>
__device__ __forceinline__ PfTile pf_decode(const PfArgs& a, const int32_t* blk_off, int n_seg, const int32_t* uniq,
                                            const int32_t* seg, int U, int mb, int t) {
  PfTile ti;
  const int blk = t / mb;
  ti.rblk = t - blk * mb;
  int lo = 0, hi = n_seg - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (blk_off[mid] <= blk) lo = mid; else hi = mid - 1;
  }
  const int j = blk - blk_off[lo], nb = blk_off[lo + 1] - blk_off[lo];
  int cnt, sbase, obase;
  if (lo < U) {
    ti.e = uniq[lo] - a.e_off;
    sbase = seg[lo];
    cnt = seg[lo + 1] - sbase;
    obase = sbase;
  } else {
    ti.e = a.e_shared + (lo - U);
    cnt = a.T;
    obase = a.P + (lo - U) * a.T;
    sbase = DOWN ? obase : a.P;   // gate/up: every shared segment reads the token-order rows
  }
  const int start = static_cast<int>(static_cast<int64_t>(cnt) * j / nb);
  const int end = static_cast<int>(static_cast<int64_t>(cnt) * (j + 1) / nb);
  ti.ntok = end - start;
  ti.npad = (ti.ntok + 15) & ~15;
  ti.brow = sbase + start;
  ti.orow = obase + start;
  return ti;
}

// Blocks of the prefill form: every segment (union experts, then shared
// experts) split into ceil(cnt / 160) near-equal token blocks; with `uniq`
// (an expert-parallel rank) routed segments of experts outside [eb, ee) get
// none.  plan = [n_seg, total_blocks, blk_off[0..n_seg]].  One CTA of 1024
// threads.
__global__ void __launch_bounds__(1024) pf_plan_kernel(const int32_t* __restrict__ n_unique,
                                                       const int32_t* __restrict__ seg_off, int T, int S,
                                                       int32_t* __restrict__ plan, const int32_t* __restrict__ uniq,
                                                       int eb, int ee) {
  pdl_wait();
  pdl_trigger();
  __shared__ int scratch[33];
  const int U = *n_unique;
  const int n_seg = U + S;
  auto nblk = [&](int s) -> int {
    if (s >= n_seg) return 0;
    if (uniq && s < U && (uniq[s] < eb || uniq[s] >= ee)) return 0;
    const int cnt = s < U ? seg_off[s + 1] - seg_off[s] : T;
    return (cnt + kPfMaxN - 1) / kPfMaxN;
  };
  const int s0 = 2 * threadIdx.x;
  const int b0 = nblk(s0), b1 = nblk(s0 + 1);
  int total = 0;
  const int off = block_exclusive_scan(b0 + b1, scratch, &total);
  if (s0 < n_seg) plan[2 + s0] = off;
  if (s0 + 1 < n_seg) plan[2 + s0 + 1] = off + b0;
  if (threadIdx.x == 0) {
    plan[0] = n_seg;
    plan[1] = total;
    plan[2 + n_seg] = total;
  }
}

// xg[i] = xq[perm[i] / k] for the P routed pairs: one warp per row, 16-byte moves.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ xq,
                                                          const int32_t* __restrict__ perm, int k, int P, int H,
                                                          uint16_t* __restrict__ xg) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_row = H / 8;
  for (int i = blockIdx.x * 8 + warp; i < P; i += gridDim.x * 8) {
    const uint4* src = reinterpret_cast<const uint4*>(xq + static_cast<size_t>(__ldg(perm + i) / k) * H);
    uint4* dst = reinterpret_cast<uint4*>(xg + static_cast<size_t>(i) * H);
    for (int c = lane; c < per_row; c += 32) dst[c] = __ldg(src + c);
  }
}

// ------------------------------------------------------------ the kernel --

// Warp-uniform bounded wait: every lane waits, the warp proceeds only if all did.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status) {
  const bool ok = mbar_wait(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}

// GROUP: K elements per fp16 scale.  GROUP 32: a 64-wide chunk has two scales,
// one per 32-wide K half.  GROUP 64: one scale per chunk; a stage's 4 scales
// are half of a 16-byte box of 8 (the scale map's box), so two consecutive
// stages load the same box and each reads its own half (K a multiple of 512).
// DOWN: the down projection (NMAT row blocks of W_down per tile, y out);
// otherwise gate/up (NMAT = 2, h out).
template <int NMAT, int GROUP, bool DOWN>
__global__ void __launch_bounds__(kPfThreads, 1)
    ffn_prefill_kernel(const __grid_constant__ CUtensorMap mq0, const __grid_constant__ CUtensorMap mq1,
                       const __grid_constant__ CUtensorMap ms0, const __grid_constant__ CUtensorMap ms1,
                       const __grid_constant__ CUtensorMap mb128, const __grid_constant__ CUtensorMap mb64,
                       const __grid_constant__ CUtensorMap mb32, const __grid_constant__ CUtensorMap mb16, PfArgs a) {
  using C = PfCfg<NMAT>;
  extern __shared__ uint8_t smem_raw[];
  // 1 KiB-aligned start, as an offset from smem_raw so that the compiler
  // keeps every pointer derived from it in the shared state space (ld.shared
  // / st.shared rather than generic accesses)
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint8_t* cst_base = smem;
  uint8_t* bst_base = smem + C::NSC * C::CSTAGE;
  int32_t* meta = reinterpret_cast<int32_t*>(bst_base + C::NSB * C::BSTAGE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(meta + C::META_INTS);
  uint64_t* code_full = bars;
  uint64_t* code_empty = code_full + C::NSC;
  uint64_t* b_full = code_empty + C::NSC;
  uint64_t* a_full = b_full + C::NSB;
  uint64_t* slot_empty = a_full + C::NBUF;   // chunk slot consumed by the MMAs (A buffer + token stage)
  uint64_t* acc_full = slot_empty + C::NBUF;
  uint64_t* acc_empty = acc_full + C::ACC_BUFS;
  uint64_t* mma_done = acc_empty + C::ACC_BUFS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int q = 0; q < C::NSC; ++q) {
      mbar_init(&code_full[q], 1);
      mbar_init(&code_empty[q], kPfDqWarps);
    }
    for (int q = 0; q < C::NSB; ++q) {
      mbar_init(&b_full[q], 1);
    }
    for (int q = 0; q < C::NBUF; ++q) {
      mbar_init(&a_full[q], 8);
      mbar_init(&slot_empty[q], 1);
    }
    for (int q = 0; q < C::ACC_BUFS; ++q) {
      mbar_init(&acc_full[q], 1);
      mbar_init(&acc_empty[q], kPfDqWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&mq0);
    if (NMAT == 2 && !DOWN) prefetch_tensormap(&mq1);
  }
  if (warp == 2 && lane == 0) {
    prefetch_tensormap(&mb128);
    prefetch_tensormap(&mb16);
  }
  if (warp == 1) tmem_alloc(tmem_slot, kPfTmemCols);
  pdl_wait();
  pdl_trigger();

  // shared copies of the plan, the unique experts and their segment offsets
  int32_t* blk_off = meta;
  int32_t* uniq = meta + kMaxSeg + 3;
  int32_t* seg = uniq + kMaxSeg;
  const int n_seg = __ldg(a.plan);
  const int total_blocks = __ldg(a.plan + 1);
  const int U = __ldg(a.n_unique);
  for (int i = threadIdx.x; i <= n_seg; i += blockDim.x) blk_off[i] = __ldg(a.plan + 2 + i);
  for (int i = threadIdx.x; i < U; i += blockDim.x) uniq[i] = __ldg(a.unique_ids + i);
  for (int i = threadIdx.x; i <= U; i += blockDim.x) seg[i] = __ldg(a.seg_off + i);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  const int K = DOWN ? a.I : a.H;
  const int R = DOWN ? a.H : a.I;
  constexpr int ROWS = DOWN ? NMAT * kRowBlock : kRowBlock;   // weight rows a tile spans
  const int mbk = R / ROWS;
  const int nk = K / 64;
  const int cps = (K % 256 == 0) ? 4 : 2;            // 64-wide chunks per code stage
  const bool one_stage = GROUP == 32 && (K == cps * 64);   // scales then move by one 1-D copy
  const int tiles = total_blocks * mbk;

  if (warp == 0) {
    // -------------------------------------------------- weight producer
    // Codes and scales run up to NSC stages (4 chunks each) ahead, paced only
    // by the dequantisation warps -- never by the MMA's token stages.
    if (lane == 0) {
      uint32_t cst = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        const PfTile ti = pf_decode<DOWN>(a, blk_off, n_seg, uniq, seg, U, mbk, t);
        const int row0 = ti.e * R + ti.rblk * ROWS;
        // weight block m: gate / up rows row0 (maps 0 / 1), or down rows row0 + 128 m (map 0)
        const int row1 = DOWN ? row0 + kRowBlock : row0;
        const CUtensorMap* q1 = DOWN ? &mq0 : &mq1;
        const CUtensorMap* s1 = DOWN ? &ms0 : &ms1;
        const uint16_t* s1p = DOWN ? a.s0 : a.s1;
        for (int kb = 0; ok && kb < nk; kb += cps) {
          const int cs = static_cast<int>(cst % C::NSC);
          if (!(ok = mbar_wait(&code_empty[cs], ((cst / C::NSC) & 1u) ^ 1u, abort_flag, a.status))) break;
          uint8_t* dst = cst_base + cs * C::CSTAGE;
          mbar_arrive_expect_tx(&code_full[cs], NMAT * kRowBlock * cps * 36);
          tma_load_2d(dst, &mq0, &code_full[cs], kb * 32, row0);
          if (NMAT == 2) tma_load_2d(dst + C::CODE_SLOT, q1, &code_full[cs], kb * 32, row1);
          uint8_t* sdst = dst + NMAT * C::CODE_SLOT;
          if (one_stage) {
            bulk_load(sdst, a.s0 + static_cast<size_t>(row0) * (K / 32), kRowBlock * cps * 4, &code_full[cs]);
            if (NMAT == 2)
              bulk_load(sdst + C::SC_SLOT, s1p + static_cast<size_t>(row1) * (K / 32), kRowBlock * cps * 4,
                        &code_full[cs]);
          } else {
            const int sx = GROUP == 32 ? kb * 2 : (kb & ~7);
            tma_load_2d(sdst, &ms0, &code_full[cs], sx, row0);
            if (NMAT == 2) tma_load_2d(sdst + C::SC_SLOT, s1, &code_full[cs], sx, row1);
          }
          ++cst;
        }
      }
      if (!ok) {
        // bounded wait (ignoring the abort flag) for the copies still in flight
        int dummy = 0;
        for (uint32_t q = cst > C::NSC ? cst - C::NSC : 0; q < cst; ++q)
          mbar_wait(&code_full[q % C::NSC], (q / C::NSC) & 1u, reinterpret_cast<volatile int*>(&dummy), a.status);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------- token-tile producer
    if (lane == 0) {
      uint32_t bit = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        const PfTile ti = pf_decode<DOWN>(a, blk_off, n_seg, uniq, seg, U, mbk, t);
        for (int kb = 0; ok && kb < nk; ++kb) {
          const int s = static_cast<int>(bit % C::NSB);
          if (!(ok = mbar_wait(&slot_empty[s], ((bit / C::NSB) & 1u) ^ 1u, abort_flag, a.status))) break;
          uint8_t* dst = bst_base + s * C::BSTAGE;
          mbar_arrive_expect_tx(&b_full[s], ti.npad * 128);
          // the token tile in as few boxes as possible (128/64/32/16 rows): the TMA
          // engine's cost per box is large next to its cost per row
          int row = ti.brow, rem = ti.npad;
          uint8_t* d = dst;
          for (; rem >= 128; rem -= 128, row += 128, d += 128 * 128) tma_load_2d(d, &mb128, &b_full[s], kb * 64, row);
          if (rem >= 64) { tma_load_2d(d, &mb64, &b_full[s], kb * 64, row); rem -= 64; row += 64; d += 64 * 128; }
          if (rem >= 32) { tma_load_2d(d, &mb32, &b_full[s], kb * 64, row); rem -= 32; row += 32; d += 32 * 128; }
          if (rem >= 16) tma_load_2d(d, &mb16, &b_full[s], kb * 64, row);
          ++bit;
        }
      }
      if (!ok) {
        int dummy = 0;
        for (uint32_t q = bit > C::NSB ? bit - C::NSB : 0; q < bit; ++q)
          mbar_wait(&b_full[q % C::NSB], (q / C::NSB) & 1u, reinterpret_cast<volatile int*>(&dummy), a.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      uint32_t it = 0, bit = 0, tt = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        const PfTile ti = pf_decode<DOWN>(a, blk_off, n_seg, uniq, seg, U, mbk, t);
        const uint32_t idesc = idesc_f16_m128(ti.npad);
        const int ab = static_cast<int>(tt % C::ACC_BUFS);
        const uint32_t dbase = tbase + ab * NMAT * kPfMaxN;
        if (!(ok = mbar_wait(&acc_empty[ab], ((tt / C::ACC_BUFS) & 1u) ^ 1u, abort_flag, a.status))) break;
        tc_fence_after();
        for (int kb = 0; kb < nk; ++kb) {
          const int b = static_cast<int>(it % C::NBUF);
          const int s = static_cast<int>(bit % C::NSB);
          if (!(ok = mbar_wait(&a_full[b], (it / C::NBUF) & 1u, abort_flag, a.status))) break;
          if (!(ok = mbar_wait(&b_full[s], (bit / C::NSB) & 1u, abort_flag, a.status))) break;
          tc_fence_after();
          const uint32_t bs = smem_addr(bst_base + s * C::BSTAGE);
          const uint32_t acol = tbase + C::ACOL + b * 32 * NMAT;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bdesc = sw128_kmajor_desc(bs + kk * 32);
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
              mma_bf16_ts(dbase + m * kPfMaxN, acol + m * 32 + kk * 8, bdesc, idesc, (kb | kk) != 0);
          }
          tc_commit(&slot_empty[b]);   // b == s: the slot's A buffer and token stage
          ++it;
          ++bit;
        }
        if (!ok) break;
        tc_commit(&acc_full[ab]);
        ++tt;
      }
      // every MMA of this CTA has completed before TMEM is released
      int dummy = 0;
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, reinterpret_cast<volatile int*>(&dummy), a.status);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------- dequantisation + epilogue
    // Team t dequantises the chunks whose running index is t mod kPfTeams, so
    // kPfTeams chunks are in flight at once; inside a team, warps with the
    // same lane quarter split each chunk into two 32-wide K halves.
    const int dw = warp - 4;
    const int q = warp & 3;                   // TMEM lane quarter of this warp
    const int g = (dw >> 2) & 1;              // 32-wide K half of every chunk
    const int team = dw >> 3;
    const int r = 32 * q + lane;              // weight row within the tile
    const uint32_t lane_bits = static_cast<uint32_t>(32 * q) << 16;
    uint32_t it = 0, tt = 0;
    uint32_t scl[NMAT][4];                    // this row's fp16 scales of the current code stage
    bool ok = true;
    bool range = false;                       // an h value fp16 cannot hold
    // epilogue of one tile: accumulators -> h (gate/up) or y (down)
    auto epilogue = [&](const PfTile& et, uint32_t ett) -> bool {
      const int ab = static_cast<int>(ett % C::ACC_BUFS);
      if (!warp_wait(&acc_full[ab], (ett / C::ACC_BUFS) & 1u, abort_flag, a.status)) return false;
      tc_fence_after();
      const uint32_t dbase = tbase + lane_bits + ab * NMAT * kPfMaxN;
      const int grow = et.rblk * ROWS + r;          // output row within the expert (weight block 0)
      const int hpos = frag_pos(grow);
      for (int c8 = dw >> 2; c8 < (et.npad >> 3); c8 += kPfDqWarps / 4) {
        uint32_t d0[8], d1[8];
        tmem_ld8(dbase + c8 * 8, d0);
        if (NMAT == 2) tmem_ld8(dbase + kPfMaxN + c8 * 8, d1);
        tmem_wait_ld();
#pragma unroll
        for (int n = 0; n < 8; ++n) {
          const int i = c8 * 8 + n;
          if (i < et.ntok) {
            if (!DOWN) {
              const float gv = __uint_as_float(d0[n]), uv = __uint_as_float(d1[n]);
              const float hv = gv / (1.0f + expf(-gv)) * uv;
              a.hq[static_cast<size_t>(et.orow + i) * a.I + hpos] = bf16_to_f16_bits(float_to_bf16_bits(hv), range);
            } else {
              float* yrow = a.ypair + static_cast<size_t>(et.orow + i) * a.H + grow;
              yrow[0] = __uint_as_float(d0[n]);
              if (NMAT == 2) yrow[kRowBlock] = __uint_as_float(d1[n]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
      return true;
    };
    // with two accumulator buffers a tile's epilogue waits until the first
    // kDefer chunks of the next tile are dequantised, so those MMAs run under it
    constexpr int kDefer = C::NBUF;
    PfTile pend{};
    uint32_t pend_tt = 0;
    bool has_pend = false;
    for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
      const PfTile ti = pf_decode<DOWN>(a, blk_off, n_seg, uniq, seg, U, mbk, t);
      for (int kb = 0; kb < nk; ++kb, ++it) {
        if (C::ACC_BUFS > 1 && has_pend && kb == (kDefer < nk ? kDefer : nk - 1)) {
          if (!(ok = epilogue(pend, pend_tt))) break;
          has_pend = false;
        }
        if (static_cast<int>(it % kPfTeams) != team) continue;
        const int ci = kb % cps;                       // chunks are stage-aligned: it % cps == kb % cps
        const uint32_t stage = it / cps;
        const int cs = static_cast<int>(stage % C::NSC);
        const uint8_t* stg = cst_base + cs * C::CSTAGE;
        if (ci < kPfTeams) {                           // this team's first chunk of the stage
          if (!(ok = warp_wait(&code_full[cs], (stage / C::NSC) & 1u, abort_flag, a.status))) break;
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            const uint8_t* sp = stg + NMAT * C::CODE_SLOT + m * C::SC_SLOT + r * cps * 4;
            if (GROUP == 64) {                         // 4 scales at element (kb - ci) & 7 of the 8-scale row
              const uint2 v = *reinterpret_cast<const uint2*>(sp + ((kb - ci) & 7) * 2);
              scl[m][0] = v.x; scl[m][1] = v.y; scl[m][2] = 0u; scl[m][3] = 0u;
            } else if (cps == 4) {
              const uint4 v = *reinterpret_cast<const uint4*>(sp);
              scl[m][0] = v.x; scl[m][1] = v.y; scl[m][2] = v.z; scl[m][3] = v.w;
            } else {
              const uint2 v = *reinterpret_cast<const uint2*>(sp);
              scl[m][0] = v.x; scl[m][1] = v.y; scl[m][2] = 0u; scl[m][3] = 0u;
            }
          }
        }
        // this thread's 16 code bytes (32 codes) of each matrix
        const int c16 = ci * 2 + g;
        const uint32_t coff = cps == 4 ? static_cast<uint32_t>(r * 128 + ((c16 ^ (r & 7)) << 4))
                                       : static_cast<uint32_t>(r * 64 + ((c16 ^ ((r >> 1) & 3)) << 4));
        uint4 cw[NMAT];
#pragma unroll
        for (int m = 0; m < NMAT; ++m) cw[m] = *reinterpret_cast<const uint4*>(stg + m * C::CODE_SLOT + coff);
        if (ci >= cps - kPfTeams) {                    // this team's last chunk of the stage
          __syncwarp();
          if (lane == 0) mbar_arrive(&code_empty[cs]);
        }
        const int b = static_cast<int>(it % C::NBUF);
        if (!(ok = warp_wait(&slot_empty[b], ((it / C::NBUF) & 1u) ^ 1u, abort_flag, a.status))) break;
        tc_fence_after();
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          uint32_t sh;
          if (GROUP == 64) {                           // chunk ci's one scale, for both K halves
            sh = (ci < 2 ? scl[m][0] : scl[m][1]) >> ((ci & 1) * 16);
          } else {
            const uint32_t sw = ci == 0 ? scl[m][0] : ci == 1 ? scl[m][1] : ci == 2 ? scl[m][2] : scl[m][3];
            sh = sw >> (g * 16);
          }
          const uint32_t s2 = (sh & 0xFFFFu) | (sh << 16);
          const uint32_t wd[4] = {cw[m].x, cw[m].y, cw[m].z, cw[m].w};
          uint32_t v[16];
#pragma unroll
          for (int w = 0; w < 4; ++w)
#pragma unroll
            for (int i = 0; i < 4; ++i) v[4 * w + i] = hmul2(dq_pair_f16(wd[w], 4 * i), s2);
          tmem_st16(tbase + lane_bits + C::ACOL + b * 32 * NMAT + m * 32 + g * 16, v);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[b]);
      }
      if (!ok) break;
      if (C::ACC_BUFS == 1) {
        if (!(ok = epilogue(ti, tt))) break;
      } else {
        pend = ti;
        pend_tt = tt;
        has_pend = true;
      }
      ++tt;
    }
    if (ok && has_pend) ok = epilogue(pend, pend_tt);
    if (range) atomicOr(a.status, COLI_FLAG_RANGE);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kPfTmemCols);
  }
}

}  // namespace coli
