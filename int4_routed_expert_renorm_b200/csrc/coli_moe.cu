// libcolimoe: host side of the C ABI declared in include/coli_moe.h.
//
// Argument checking, workspace layout, tensor-map encoding and the launch
// sequence of one routed-expert MoE layer (Colibri README, "Il percorso di
// ogni token": Route -> Union -> expert matmuls, every layer of every token).
// All device work is enqueued on the caller's stream; nothing here allocates
// or synchronises, except coli_moe_get_status.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "k_ffn_decode.cuh"
#include "k_ffn_prefill.cuh"
#include "k_ffn_splitk.cuh"
#include "k_router.cuh"
#include "k_tier.cuh"
#include "k_union.cuh"

using namespace coli;

// Scratch of coli_moe_layer_noalloc (see include/coli_moe.h): device memory
// owned by the library for callers that cannot allocate.  Host code must not
// use this name as a pointer; its device address comes from
// cudaGetSymbolAddress, once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[COLI_NOALLOC_SCRATCH_BYTES];

namespace {

__device__ uint32_t g_status_word;

// A counter nothing ever increments: the grid-counter wait of the timeout hook.
__device__ int32_t g_never_counted;

// Test hook of the bounded waits (coli_moe_test_wait_timeout): one thread waits
// with a limit of limit_ns on an mbarrier nothing arrives on, then on a
// counter nothing increments -- the same helpers every pipeline wait of the
// FFN kernels uses.  Each wait gives up, sets COLI_FLAG_TIMEOUT and returns;
// elapsed[0..1] (may be NULL) receive the time each one took.
__global__ void wait_timeout_kernel(uint64_t limit_ns, uint64_t* elapsed, uint32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  abort_flag = 0;
  fence_mbar_init();
  const uint64_t t0 = globaltimer();
  const bool got_bar = mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
  const uint64_t t1 = globaltimer();
  abort_flag = 0;
  const bool got_cnt = wait_counter(&g_never_counted, 1, &abort_flag, status, limit_ns);
  const uint64_t t2 = globaltimer();
  if (elapsed) {
    elapsed[0] = got_bar ? 0 : t1 - t0;
    elapsed[1] = got_cnt ? 0 : t2 - t1;
  }
}

thread_local uint64_t t_launches = 0;

// Stage events of the timing hook (coli_moe_set_stage_events); consumed by one call.
constexpr int kMaxStageEvents = 16;
thread_local cudaEvent_t t_stage_ev[kMaxStageEvents];
thread_local int t_stage_n = 0;

struct StageRecorder {
  cudaEvent_t ev[kMaxStageEvents];
  int n;
  cudaStream_t st;
  explicit StageRecorder(cudaStream_t s) : n(t_stage_n), st(s) {
    for (int i = 0; i < n; ++i) ev[i] = t_stage_ev[i];
    t_stage_n = 0;
  }
  void mark(int i) const {
    if (i < n) cudaEventRecord(ev[i], st);
  }
  void mark_through(int i0, int i1) const {
    for (int i = i0; i <= i1; ++i) mark(i);
  }
};

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint32_t* g_status_ptr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};
bool g_attr_done[kMaxDevices] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

struct DevInfo {
  uint32_t* status;
  int sms;
};

coli_status dev_info(DevInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return COLI_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return COLI_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return COLI_ERR_CUDA;
    g_status_ptr[dev] = static_cast<uint32_t*>(p);
    g_num_sms[dev] = sms;
  }
  if (!g_attr_done[dev]) {
    bool ok = true;
#define COLI_SET_SMEM(NT, SG, KCD, GR)                                                                   \
  ok &= cudaFuncSetAttribute(ffn_fused_kernel<NT, SG, KCD, GR>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             static_cast<int>(FusedCfg<NT, KCD, GR>::SMEM)) == cudaSuccess;
    COLI_SET_SMEM(1, true, 128, 32)
    COLI_SET_SMEM(1, false, 128, 32)
    COLI_SET_SMEM(2, false, 128, 32)
    COLI_SET_SMEM(4, false, 128, 32)
    COLI_SET_SMEM(2, false, 256, 32)
    COLI_SET_SMEM(4, false, 256, 32)
    COLI_SET_SMEM(2, false, 256, 64)
    COLI_SET_SMEM(4, false, 256, 64)
#undef COLI_SET_SMEM
#define COLI_SET_PF_SMEM(NMAT, GR, DN)                                                                      \
  ok &= cudaFuncSetAttribute(ffn_prefill_kernel<NMAT, GR, DN>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             static_cast<int>(PfCfg<NMAT>::SMEM)) == cudaSuccess;
    COLI_SET_PF_SMEM(2, 32, false)
    COLI_SET_PF_SMEM(2, 32, true)
    COLI_SET_PF_SMEM(2, 64, false)
    COLI_SET_PF_SMEM(2, 64, true)
#undef COLI_SET_PF_SMEM
#define COLI_SET_SK_SMEM(NT, GR, B)                                                                           \
  ok &= cudaFuncSetAttribute(ffn_splitk_kernel<NT, GR, B, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             static_cast<int>(SkCfg<GR, B>::SMEM)) == cudaSuccess;                           \
  ok &= cudaFuncSetAttribute(ffn_splitk_kernel<NT, GR, B, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                             static_cast<int>(SkCfg<GR, B>::SMEM)) == cudaSuccess;
    COLI_SET_SK_SMEM(1, 32, 4)
    COLI_SET_SK_SMEM(2, 32, 4)
    COLI_SET_SK_SMEM(1, 64, 4)
    COLI_SET_SK_SMEM(2, 64, 4)
    COLI_SET_SK_SMEM(1, 32, 8)
    COLI_SET_SK_SMEM(2, 32, 8)
    COLI_SET_SK_SMEM(1, 64, 8)
    COLI_SET_SK_SMEM(2, 64, 8)
#undef COLI_SET_SK_SMEM
    ok &= cudaFuncSetAttribute(logits_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) ==
          cudaSuccess;
    ok &= cudaFuncSetAttribute(union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kUnionWarps * 1024 * 4) == cudaSuccess;
    ok &= cudaFuncSetAttribute(union_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kUnionWarps * 1024 * 4) == cudaSuccess;
    const int ru_smem = (kUnionWarps * 1024 + kFusedRouteMaxT * 32) * 4;
    ok &= cudaFuncSetAttribute(route_union_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, ru_smem) == cudaSuccess;
    ok &= cudaFuncSetAttribute(route_union_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, ru_smem) == cudaSuccess;
    ok &= cudaFuncSetAttribute(route_union_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, ru_smem) == cudaSuccess;
    ok &= cudaFuncSetAttribute(route_union_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, ru_smem) == cudaSuccess;
    ok &= cudaFuncSetAttribute(route_union_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, ru_smem) == cudaSuccess;
    ok &= cudaFuncSetAttribute(route_union_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, ru_smem) == cudaSuccess;
    if (!ok) return COLI_ERR_CUDA;
    if (!g_encode) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return COLI_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    g_attr_done[dev] = true;
  }
  out->status = g_status_ptr[dev];
  out->sms = g_num_sms[dev];
  return COLI_OK;
}

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// Every kernel is launched with programmatic stream serialization: its CTAs
// may become resident while the previous kernel drains, and each kernel
// executes griddepcontrol.wait before touching any input.
template <typename... KArgs, typename... Args>
bool launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  ++t_launches;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess;
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

coli_status check_dims(const coli_moe_dims* d) {
  if (!d) return COLI_ERR_INVALID_ARG;
  if (d->group != 32 && d->group != 64) return COLI_ERR_UNSUPPORTED;
  if (d->code_bits != 0 && d->code_bits != 4 && d->code_bits != 8) return COLI_ERR_UNSUPPORTED;
  // int8 codes run in the split-K decode form only: whole 16-byte down scale rows
  if (d->code_bits == 8 && d->inter % 256 != 0) return COLI_ERR_UNSUPPORTED;
  if (d->hidden <= 0 || d->hidden % 256 != 0) return COLI_ERR_UNSUPPORTED;
  if (d->inter <= 0 || !(d->inter % 256 == 0 || d->inter == 128)) return COLI_ERR_UNSUPPORTED;
  // 64-wide groups: scale rows are read in 16-byte boxes of 8 scales (512 K)
  if (d->group == 64 && (d->hidden % 512 != 0 || d->inter % 512 != 0)) return COLI_ERR_UNSUPPORTED;
  if (d->n_experts < 1 || d->n_experts > 1024) return COLI_ERR_UNSUPPORTED;
  if (d->top_k < 1 || d->top_k > 32 || d->top_k > d->n_experts) return COLI_ERR_UNSUPPORTED;
  if (d->n_shared < 0 || d->n_shared > 4) return COLI_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(d->n_experts + d->n_shared) * d->hidden > (int64_t(1) << 31)) return COLI_ERR_UNSUPPORTED;
  return COLI_OK;
}

coli_status check_weights(const coli_moe_weights* w, bool need_router) {
  if (!w || !w->gate_q || !w->up_q || !w->down_q || !w->gate_s || !w->up_s || !w->down_s)
    return COLI_ERR_INVALID_ARG;
  if (need_router && !w->router_w) return COLI_ERR_INVALID_ARG;
  const void* ps[6] = {w->gate_q, w->up_q, w->down_q, w->gate_s, w->up_s, w->down_s};
  for (const void* p : ps)
    if (!aligned(p, 16)) return COLI_ERR_INVALID_ARG;
  if (need_router && !aligned(w->router_w, 16)) return COLI_ERR_INVALID_ARG;
  return COLI_OK;
}

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Workspace layout for T tokens (every region 256-byte aligned).
struct Ws {
  uint16_t* xg;      // [P][H] expert input gathered into pair order (prefill form), directly followed by xq
  uint16_t* xq;      // [T][H] fragment-ordered expert input
  uint16_t* xn;      // [T][H] normalised input (prenorm)
  uint8_t* xp;       // split-K form: [T][H/32][kPlaneRec] integer planes of the expert input
  int32_t* xe;       // split-K form: [T] their grid exponents
  float* logits;     // [T][E]
  int32_t* ids;      // [T*k]
  float* w;          // [T*k]
  int32_t* unique;   // [min(E,P)]
  int32_t* n_unique; // [1]
  int32_t* seg_off;  // [min(E,P)+1]
  int32_t* perm;     // [P]
  int32_t* pair_pos; // [P]
  int32_t* ucnt;     // [ceil(P / union_chunk(P))][E] per-chunk expert counts of the many-CTA union
  int32_t* plan;     // [min(E,P)+S+3]
  int32_t* tb_done;  // [token blocks upper bound] gate/up completion per token block
  int32_t* rb_done;  // [H/128] down completion per output row block
  uint16_t* hq;      // [P+S*T][I]
  float* ypair;      // [P+S*T][H]
  uint16_t* xin;     // [T][H] the input rows copied from host memory (COLI_LAYER_HOST_X)
  uint16_t* rin;     // [T][H] the residual rows copied from host memory
  int32_t* sunique;  // [min(E,P)] device slot of each unique expert (host-RAM tier)
  size_t bytes;
};

// Split-K form: batches of <= kSkMaxT tokens whose down scale rows are whole
// 16-byte units (I a multiple of 256; of 512 with 64-wide groups, as always).
inline bool use_splitk(const coli_moe_dims* d, int T) { return T <= kSkMaxT && d->inter % 256 == 0; }

inline int code_bits(const coli_moe_dims* d) { return d->code_bits == 8 ? 8 : 4; }

// Tokens per block of logits_tile_kernel: up to 8, their bf16 rows in at most
// 200 KB of shared memory.
inline int logits_tokens_per_block(int H) {
  const int t = static_cast<int>((200 * 1024) / (static_cast<long>(H) * 2));
  return t < 1 ? 1 : t > 8 ? 8 : t;
}

// Tokens per token block of the two-phase decode form: 8 for T <= 8 (I = 128
// only; other shapes take the split-K form), 16 up to 64 tokens, 32 above.
// 16-token blocks leave room for a fourth pipeline stage, which outweighs the
// extra weight reads of experts with more than 16 tokens (decode b64 Zipf:
// 1.11x instead of 1.03x the union's bytes, 19 % less time).
inline int tok_block(int T) { return T <= 8 ? 8 : T <= 64 ? 16 : 32; }

Ws layout(const coli_moe_dims* d, int T, void* base) {
  Ws ws{};
  const size_t H = d->hidden, I = d->inter, E = d->n_experts, k = d->top_k, S = d->n_shared;
  const size_t P = static_cast<size_t>(T) * k;
  const size_t Umax = P < E ? P : E;
  const size_t rows = P + S * static_cast<size_t>(T);
  uint8_t* b = static_cast<uint8_t*>(base);
  size_t o = 0;
  auto take = [&](size_t bytes) -> void* {
    void* p = b ? b + o : nullptr;
    o += align256(bytes);
    return p;
  };
  ws.xg = static_cast<uint16_t*>(take((P + static_cast<size_t>(T)) * H * 2));
  ws.xq = ws.xg ? ws.xg + P * H : nullptr;
  ws.xn = static_cast<uint16_t*>(take(T * H * 2));
  {
    const size_t tsk = use_splitk(d, T) ? static_cast<size_t>(T) : 0;
    // NULL when the batch takes another form: the front kernels then write no planes
    uint8_t* xp = static_cast<uint8_t*>(take(tsk * (H / 32) * kPlaneRec));
    int32_t* xe = static_cast<int32_t*>(take(tsk * 4));
    ws.xp = tsk ? xp : nullptr;
    ws.xe = tsk ? xe : nullptr;
  }
  ws.logits = static_cast<float*>(take(T * E * 4));
  ws.ids = static_cast<int32_t*>(take(P * 4));
  ws.w = static_cast<float*>(take(P * 4));
  ws.unique = static_cast<int32_t*>(take(Umax * 4));
  ws.n_unique = static_cast<int32_t*>(take(4));
  ws.seg_off = static_cast<int32_t*>(take((Umax + 1) * 4));
  ws.perm = static_cast<int32_t*>(take(P * 4));
  ws.pair_pos = static_cast<int32_t*>(take(P * 4));
  {
    const size_t chunk = static_cast<size_t>(union_chunk(static_cast<int>(P)));
    ws.ucnt = static_cast<int32_t*>(take((P + chunk - 1) / chunk * E * 4));
  }
  ws.plan = static_cast<int32_t*>(take((Umax + S + 3) * 4));
  {
    const size_t tokb = static_cast<size_t>(tok_block(T));
    const size_t blocks_ub = Umax + P / tokb + S * ((static_cast<size_t>(T) + tokb - 1) / tokb);
    ws.tb_done = static_cast<int32_t*>(take(blocks_ub * 4));
    ws.rb_done = static_cast<int32_t*>(take(H / 128 * 4));
  }
  ws.hq = static_cast<uint16_t*>(take(rows * I * 2));
  {
    // the split-K form keeps y as I/128 partials per (pair, row) in the same region
    const size_t yb = rows * H * 4, pb = use_splitk(d, T) ? rows * (I / 128) * H * 4 : 0;
    ws.ypair = static_cast<float*>(take(yb > pb ? yb : pb));
  }
  ws.xin = static_cast<uint16_t*>(take(static_cast<size_t>(T) * H * 2));
  ws.rin = static_cast<uint16_t*>(take(static_cast<size_t>(T) * H * 2));
  ws.sunique = static_cast<int32_t*>(take(Umax * 4));
  ws.bytes = o;
  return ws;
}

bool encode_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor maps of one matrix kind: codes [rows_total][K*bits/8] bytes and
// scales [rows_total][K/group] fp16, tiles of 128 rows x KC elements; the
// scale box is KC/32 scales (int4, group 32) or 8 scales (otherwise; K a
// multiple of 512 with group 64).
bool matrix_maps(const uint8_t* q, const uint16_t* s, uint64_t rows_total, int K, int KC, int group, int bits,
                 CUtensorMap* mq, CUtensorMap* ms) {
  // stage rows of 256 bytes move as two 128-byte-wide boxes
  const int rowb = KC * bits / 8;
  const CUtensorMapSwizzle swz = rowb >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
  if (!encode_2d(mq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, static_cast<uint64_t>(K) * bits / 8, rows_total,
                 static_cast<uint64_t>(K) * bits / 8, rowb >= 128 ? 128 : rowb, kRowBlock, swz))
    return false;
  if (KC < K) {
    if (!encode_2d(ms, CU_TENSOR_MAP_DATA_TYPE_UINT16, s, K / group, rows_total, (K / group) * 2,
                   (group == 32 && bits == 4) ? KC / 32 : 8, kRowBlock, CU_TENSOR_MAP_SWIZZLE_NONE))
      return false;
  } else {
    std::memset(ms, 0, sizeof(*ms));  // scales move by 1-D bulk copies when a stage spans K
  }
  return true;
}

// The persistent FFN kernels are launched cooperatively (all CTAs resident,
// so the counter waits between CTAs always make progress).
using FfnKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, FfnArgs);

bool launch_cooperative(FfnKernel kernel, size_t smem, const CUtensorMap* m, const FfnArgs& a, int grid,
                        cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kFfnThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  ++t_launches;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, m[0], m[1], m[2], m[3], m[4], m[5], a);
  if (e != cudaSuccess) {
    // without overlap with the previous kernel
    cudaGetLastError();
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kernel, m[0], m[1], m[2], m[3], m[4], m[5], a);
  }
  return e == cudaSuccess;
}

// The split-K kernel as a plain launch with programmatic dependent launch:
// its grid is at most one CTA per SM and its shared memory admits one CTA
// per SM, so every CTA becomes resident without a cooperative launch (a CTA
// that finds its SM still busy with the preceding kernel's CTAs -- the routing
// kernel's one CTA, the front kernel's, or a tier's copies -- starts when they
// end; none of them waits on anything of this kernel).  The plain launch lets
// the CTAs start their prologue and the shared experts' weight stream while
// the preceding kernel still runs, which a cooperative launch does not.  Every
// wait in the kernel is bounded.
bool launch_splitk(FfnKernel kernel, size_t smem, const CUtensorMap* m, const FfnArgs& a, int grid, int sms,
                   cudaStream_t st) {
  if (grid > sms) return false;
  return launch(kernel, dim3(grid), dim3(kFfnThreads), smem, st, m[0], m[1], m[2], m[3], m[4], m[5], a);
}

template <int NT, bool SG, int KCD, int GR>
bool launch_ffn_fused(const CUtensorMap* m, const FfnArgs& a, int grid, cudaStream_t st) {
  return launch_cooperative(ffn_fused_kernel<NT, SG, KCD, GR>, FusedCfg<NT, KCD, GR>::SMEM, m, a, grid, st);
}

// Two-phase decode-form variant for this batch: tiles of tok_block(T) tokens
// (T <= 8 only with I = 128, KCD = 128).
template <int KCD, int GR>
bool launch_ffn_for(int T, const CUtensorMap* m, const FfnArgs& a, int grid, cudaStream_t st) {
  if (tok_block(T) == 8) {
    if (KCD != 128 || GR != 32) return false;   // other shapes take the split-K form at T <= 8
    return T == 1 ? launch_ffn_fused<1, true, 128, 32>(m, a, grid, st)
                  : launch_ffn_fused<1, false, 128, 32>(m, a, grid, st);
  }
  if (tok_block(T) == 16) return launch_ffn_fused<2, false, KCD, GR>(m, a, grid, st);
  return launch_ffn_fused<4, false, KCD, GR>(m, a, grid, st);
}

bool launch_route(const float* lg, const float* bias, int T, int E, int k, int32_t* ids, float* w, uint32_t* status,
                  cudaStream_t st) {
  const dim3 g((T + 7) / 8), b(256);
  switch (route_nv(E)) {
    case 1: return launch(route_kernel<1>, g, b, 0, st, lg, bias, T, E, k, ids, w, status);
    case 2: return launch(route_kernel<2>, g, b, 0, st, lg, bias, T, E, k, ids, w, status);
    case 4: return launch(route_kernel<4>, g, b, 0, st, lg, bias, T, E, k, ids, w, status);
    case 8: return launch(route_kernel<8>, g, b, 0, st, lg, bias, T, E, k, ids, w, status);
    case 16: return launch(route_kernel<16>, g, b, 0, st, lg, bias, T, E, k, ids, w, status);
    default: return launch(route_kernel<32>, g, b, 0, st, lg, bias, T, E, k, ids, w, status);
  }
}

// Route + union + plan in one CTA (T <= kFusedRouteMaxT); one warp does the
// union when T*k <= kWarpUnionMaxP.
bool launch_route_union(const float* lg, const float* bias, int T, int E, int k, int S, int tokb, int n_rb,
                        int32_t* ids, float* w, const Ws& ws, uint32_t* status, cudaStream_t st, int eb = 0,
                        int ee = -1) {
  if (ee < 0) ee = E;
  if (T * k <= kWarpUnionMaxP) {
    const dim3 g(1), b(32 * (T < 8 ? T : 8));
#define COLI_RUS(NV)                                                                                             \
  launch(route_union_small_kernel<NV>, g, b, 0, st, lg, bias, T, E, k, ids, w, ws.unique, ws.n_unique, ws.seg_off, \
         ws.perm, ws.pair_pos, status, S, tokb, ws.plan, ws.tb_done, ws.rb_done, n_rb, eb, ee)
    switch (route_nv(E)) {
      case 1: return COLI_RUS(1);
      case 2: return COLI_RUS(2);
      case 4: return COLI_RUS(4);
      case 8: return COLI_RUS(8);
      case 16: return COLI_RUS(16);
      default: return COLI_RUS(32);
    }
#undef COLI_RUS
  }
  const size_t smem = static_cast<size_t>(kUnionWarps * E + T * k) * 4;
  const dim3 g(1), b(kUnionThreads);
#define COLI_RU(NV)                                                                                            \
  launch(route_union_kernel<NV>, g, b, smem, st, lg, bias, T, E, k, ids, w, ws.unique, ws.n_unique, ws.seg_off, \
         ws.perm, ws.pair_pos, status, S, tokb, ws.plan, ws.tb_done, ws.rb_done, n_rb, eb, ee)
  switch (route_nv(E)) {
    case 1: return COLI_RU(1);
    case 2: return COLI_RU(2);
    case 4: return COLI_RU(4);
    case 8: return COLI_RU(8);
    case 16: return COLI_RU(16);
    default: return COLI_RU(32);
  }
#undef COLI_RU
}

// FFN form for this call: the tcgen05 grouped GEMM when forced, or by default
// once the batch averages >= 32 tokens per expert of the union's upper bound.
enum class Form { kDecode, kPrefill, kInvalid, kUnsupported };

Form choose_form(uint32_t flags, int T, const coli_moe_dims* d) {
  const int E = d->n_experts, k = d->top_k;
  const bool fd = (flags & COLI_PATH_DECODE) != 0, fp = (flags & COLI_PATH_PREFILL) != 0;
  if (fd && fp) return Form::kInvalid;
  // int8 codes: the split-K decode form, batches above 8 tokens in 8-token passes
  if (code_bits(d) == 8) return (fp || d->inter % 256 != 0) ? Form::kUnsupported : Form::kDecode;
  if (fd) return Form::kDecode;
  if (fp) return Form::kPrefill;
  const long P = static_cast<long>(T) * k;
  const long U = P < E ? P : E;
  return (T >= kPfAutoMinT && P >= 32 * U) ? Form::kPrefill : Form::kDecode;
}

// Tensor maps of the prefill form: codes [rows][K/2] bytes in boxes of 128
// rows x cps*32 bytes (128B / 64B swizzle), scales [rows][K/32] fp16 in boxes
// of 128 rows x cps*2 (unless one stage spans K), token rows [rows][K] bf16 in
// boxes of 128/64/32/16 rows x 64 elements (128B swizzle).
bool pf_weight_maps(const uint8_t* q, const uint16_t* s, uint64_t rows_total, int K, int group, CUtensorMap* mq,
                    CUtensorMap* ms) {
  const int cps = (K % 256 == 0) ? 4 : 2;
  const CUtensorMapSwizzle swz = cps == 4 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!encode_2d(mq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, K / 2, rows_total, K / 2, cps * 32, kRowBlock, swz))
    return false;
  if (group == 64)   // boxes of 8 scales (two code stages); K is a multiple of 512
    return encode_2d(ms, CU_TENSOR_MAP_DATA_TYPE_UINT16, s, K / 64, rows_total, (K / 64) * 2, 8, kRowBlock,
                     CU_TENSOR_MAP_SWIZZLE_NONE);
  if (K == cps * 64) {
    std::memset(ms, 0, sizeof(*ms));
    return true;
  }
  return encode_2d(ms, CU_TENSOR_MAP_DATA_TYPE_UINT16, s, K / 32, rows_total, (K / 32) * 2, cps * 2, kRowBlock,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
}

template <int NMAT, int GR, bool DN>
bool launch_prefill(const CUtensorMap* m, const PfArgs& a, int grid, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kPfThreads);
  cfg.dynamicSmemBytes = PfCfg<NMAT>::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  ++t_launches;
  return cudaLaunchKernelEx(&cfg, ffn_prefill_kernel<NMAT, GR, DN>, m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7], a) ==
         cudaSuccess;
}

// The experts one call computes: all of them, or an expert-parallel rank's
// share (routed experts [begin, end), the shared ones when shared != 0), whose
// weights then hold only those experts, and whose output is the unrounded
// fp32 partial sum `out_f32`.
struct EpRange {
  bool on = false;
  int begin = 0, end = 0, shared = 0;
  const int32_t* ids = nullptr;
  float* out_f32 = nullptr;
};

// Prefill form: gather the expert input into pair order, plan the token
// blocks, gate/up GEMM (h), down GEMM (y), combine.
coli_status run_ffn_prefill(const coli_moe_dims* d, const coli_moe_weights* w, int T, const int32_t* unique,
                            const int32_t* n_unique, const int32_t* seg_off, const int32_t* perm,
                            const int32_t* pair_pos, const float* topk_w, const uint16_t* residual, uint16_t* out,
                            const Ws& ws, const DevInfo& di, cudaStream_t st, const StageRecorder& rec,
                            const EpRange& ep = EpRange()) {
  const int H = d->hidden, I = d->inter, E = d->n_experts, k = d->top_k;
  const int S = ep.on ? ep.shared : d->n_shared;
  const int E_w = ep.on ? ep.end - ep.begin : E;   // routed experts held by the weights
  const int P = T * k;
  const uint64_t rows_gu = static_cast<uint64_t>(E_w + S) * I;
  const uint64_t rows_dn = static_cast<uint64_t>(E_w + S) * H;
  CUtensorMap mg[8], md[8];   // q0, q1, s0, s1, token rows in boxes of 128, 64, 32, 16 rows
  const int G = d->group;
  if (!pf_weight_maps(w->gate_q, w->gate_s, rows_gu, H, G, &mg[0], &mg[2]) ||
      !pf_weight_maps(w->up_q, w->up_s, rows_gu, H, G, &mg[1], &mg[3]) ||
      !pf_weight_maps(w->down_q, w->down_s, rows_dn, I, G, &md[0], &md[2]))
    return COLI_ERR_CUDA;
  for (int j = 0; j < 4; ++j) {
    const uint32_t box = 128u >> j;
    if (!encode_2d(&mg[4 + j], CU_TENSOR_MAP_DATA_TYPE_UINT16, ws.xg, H, static_cast<uint64_t>(P) + T,
                   static_cast<uint64_t>(H) * 2, 64, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&md[4 + j], CU_TENSOR_MAP_DATA_TYPE_UINT16, ws.hq, I,
                   static_cast<uint64_t>(P) + static_cast<uint64_t>(S) * T, static_cast<uint64_t>(I) * 2, 64, box,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return COLI_ERR_CUDA;
  }
  md[1] = md[0];
  md[3] = md[2];

  {
    long blocks = (P + 7) / 8;
    if (blocks > 8L * di.sms) blocks = 8L * di.sms;
    if (!launch(gather_rows_kernel, dim3(static_cast<int>(blocks)), dim3(256), 0, st,
                static_cast<const uint16_t*>(ws.xq), perm, k, P, H, ws.xg))
      return COLI_ERR_CUDA;
  }
  if (!launch(pf_plan_kernel, dim3(1), dim3(1024), 0, st, n_unique, seg_off, T, S, ws.plan,
              ep.on ? unique : static_cast<const int32_t*>(nullptr), ep.on ? ep.begin : 0, ep.on ? ep.end : E))
    return COLI_ERR_CUDA;
  rec.mark(5);

  PfArgs a{};
  a.plan = ws.plan;
  a.unique_ids = unique;
  a.n_unique = n_unique;
  a.seg_off = seg_off;
  a.hq = ws.hq;
  a.ypair = ws.ypair;
  a.status = di.status;
  a.H = H;
  a.I = I;
  a.T = T;
  a.k = k;
  a.E = E;
  a.S = S;
  a.P = P;
  a.e_off = ep.on ? ep.begin : 0;
  a.e_shared = E_w;
  const int Umax = P < E ? P : E;
  const long blocks_ub = static_cast<long>(Umax) + P / kPfMaxN + static_cast<long>(S) * (T / kPfMaxN + 1);
  auto grid_for = [&](int mb) {
    const long tiles = blocks_ub * mb;
    return static_cast<int>(tiles < di.sms ? tiles : di.sms);
  };
  a.s0 = w->gate_s;
  a.s1 = w->up_s;
  if (!(G == 32 ? launch_prefill<2, 32, false>(mg, a, grid_for(I / kRowBlock), st)
                : launch_prefill<2, 64, false>(mg, a, grid_for(I / kRowBlock), st)))
    return COLI_ERR_CUDA;
  rec.mark(6);
  a.s0 = w->down_s;
  a.s1 = w->down_s;
  // two 128-row blocks of W_down per tile (H is a multiple of 256)
  if (!(G == 32 ? launch_prefill<2, 32, true>(md, a, grid_for(H / (2 * kRowBlock)), st)
                : launch_prefill<2, 64, true>(md, a, grid_for(H / (2 * kRowBlock)), st)))
    return COLI_ERR_CUDA;
  rec.mark(7);
  {
    const long work = static_cast<long>(T) * (H / 4);
    long blocks = (work + 255) / 256;
    // enough blocks in flight for the combine to stream its 4 (k + S) H bytes
    // per token at the memory's rate (4 x SMs left it ~10 % short at 4096 tokens)
    if (blocks > 16L * di.sms) blocks = 16L * di.sms;
    if (!launch(combine_kernel, dim3(static_cast<int>(blocks)), dim3(256), 0, st, static_cast<const float*>(ws.ypair),
                pair_pos, topk_w, residual, T, k, S, H, out, ep.on ? ep.ids : static_cast<const int32_t*>(nullptr),
                ep.on ? ep.begin : 0, ep.on ? ep.end : E, ep.on ? ep.out_f32 : static_cast<float*>(nullptr)))
      return COLI_ERR_CUDA;
  }
  rec.mark(8);
  return COLI_OK;
}

// The split-K kernel's own routing (logits not NULL): the batch's router
// logits and bias, and where the ids and weights go; the union and the plan
// go to the workspace arrays as a routing kernel would write them.
struct InRoute {
  const float* logits = nullptr;
  const float* bias = nullptr;
  int32_t* ids = nullptr;
  float* w = nullptr;
};

// The split-K kernel routes the batch itself for 2 to 8 tokens when one warp
// can sort the pairs and route a token (T*k <= 128, E <= 256).  A single token
// is routed by its own kernel: measured on the GLM-5.2-shaped layer, the
// in-kernel routing made the batch-1 step slower (about 2 us of 65) and the
// 4-token stack faster (about 3 %).
inline bool splitk_routes(const coli_moe_dims* d, int T) {
  return T >= 2 && use_splitk(d, T) && T * d->top_k <= kWarpUnionMaxP && d->n_experts <= 256;
}

// The decode-form FFN + combine part shared by coli_moe_expert_ffn and
// coli_moe_layer; the tile plan (ws.plan) must already be on the stream.
coli_status run_ffn(const coli_moe_dims* d, const coli_moe_weights* w, int T, const int32_t* unique,
                    const int32_t* n_unique, const int32_t* seg_off, const int32_t* perm, const int32_t* pair_pos,
                    const float* topk_w, const uint16_t* residual, uint16_t* out, const Ws& ws, const DevInfo& di,
                    cudaStream_t st, const StageRecorder& rec, const EpRange& ep = EpRange(),
                    const InRoute& ir = InRoute(), int slots = 0) {
  const int H = d->hidden, I = d->inter, E = d->n_experts, k = d->top_k;
  const int S = ep.on ? ep.shared : d->n_shared;
  // routed experts held by the weights: all, an expert-parallel rank's range,
  // or the slots of a host-RAM tier (the union then holds slot numbers)
  const int E_w = slots > 0 ? slots : ep.on ? ep.end - ep.begin : E;
  const int P = T * k;
  const uint64_t rows_gu = static_cast<uint64_t>(E_w + S) * I;
  const uint64_t rows_dn = static_cast<uint64_t>(E_w + S) * H;
  const int tokb = tok_block(T);

  // upper bound on tiles: every segment contributes ceil(cnt/64) <= cnt/64 + 1 blocks
  const int Umax = P < E ? P : E;
  const long blocks_ub = static_cast<long>(Umax) + P / tokb + static_cast<long>(S) * ((T + tokb - 1) / tokb);

  CUtensorMap maps[6];   // gate q, up q, gate s, up s, down q, down s
  // gate/up stages of 256 K (int8: 128 K); down stages of the two-phase form
  // 256 K (128 K when I = 128); the split-K form builds its own down maps
  const int G = d->group, B = code_bits(d);
  const int kc_dn = (I % 256 == 0) ? 256 : 128;   // two-phase form: T > 8, or I = 128
  const int kc_gu = B == 4 ? 256 : 128;
  if (!matrix_maps(w->gate_q, w->gate_s, rows_gu, H, kc_gu, G, B, &maps[0], &maps[2]) ||
      !matrix_maps(w->up_q, w->up_s, rows_gu, H, kc_gu, G, B, &maps[1], &maps[3]) ||
      (B == 4 && !matrix_maps(w->down_q, w->down_s, rows_dn, I, kc_dn, G, B, &maps[4], &maps[5])))
    return COLI_ERR_CUDA;

  FfnArgs a{};
  a.xq = ws.xq;
  a.hq = ws.hq;
  a.ypair = ws.ypair;
  a.gate_s = w->gate_s;
  a.up_s = w->up_s;
  a.down_s = w->down_s;
  a.unique_ids = unique;
  a.n_unique = n_unique;
  a.seg_off = seg_off;
  a.perm = perm;
  a.plan = ws.plan;
  a.tb_done = ws.tb_done;
  a.rb_done = ws.rb_done;
  a.pair_pos = pair_pos;
  a.topk_w = topk_w;
  a.residual = residual;
  a.out = out;
  a.status = di.status;
  a.H = H;
  a.I = I;
  a.T = T;
  a.k = k;
  a.E = E;
  a.S = S;
  a.P = P;
  a.e_off = ep.on ? ep.begin : 0;
  a.e_end = ep.on ? ep.end : E;
  a.e_shared = E_w;
  a.topk_ids = ep.on ? ep.ids : nullptr;
  a.out_f32 = ep.on ? ep.out_f32 : nullptr;
  a.tokb = tokb;
  if (ir.logits) {
    a.r_logits = ir.logits;
    a.r_bias = ir.bias;
    a.r_ids = ir.ids;
    a.r_w = ir.w;
    a.r_unique = ws.unique;
    a.r_n_unique = ws.n_unique;
    a.r_seg_off = ws.seg_off;
    a.r_perm = ws.perm;
    a.r_pair_pos = ws.pair_pos;
    a.r_plan = ws.plan;
  }
  if (use_splitk(d, T)) {
    // down maps of the split-K form: codes in boxes of 128 rows x one
    // 128-wide K slice (64 bytes, 64B swizzle; int8: 128 bytes, 128B
    // swizzle), scales in boxes of 8 x 128 rows
    const uint64_t drow = static_cast<uint64_t>(I) * B / 8;
    if (!encode_2d(&maps[4], CU_TENSOR_MAP_DATA_TYPE_UINT8, w->down_q, drow, rows_dn, drow, 16 * B, kRowBlock,
                   B == 4 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&maps[5], CU_TENSOR_MAP_DATA_TYPE_UINT16, w->down_s, I / G, rows_dn, (I / G) * 2, 8, kRowBlock,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
      return COLI_ERR_CUDA;
    a.ypart = ws.ypair;
    a.xp = ws.xp;
    a.xe = ws.xe;
    const long tiles = blocks_ub * (I / kRowBlock);
    const int grid = static_cast<int>(tiles < di.sms ? tiles : di.sms);
    // MMA n-tiles of four tokens each
    const bool nt2 = T > 4;
    FfnKernel k;
    size_t smem;
#define COLI_SK(NT, GR, B) (ir.logits ? ffn_splitk_kernel<NT, GR, B, true> : ffn_splitk_kernel<NT, GR, B, false>)
    if (B == 4) {
      k = nt2 ? (G == 32 ? COLI_SK(2, 32, 4) : COLI_SK(2, 64, 4)) : (G == 32 ? COLI_SK(1, 32, 4) : COLI_SK(1, 64, 4));
      smem = G == 32 ? SkCfg<32, 4>::SMEM : SkCfg<64, 4>::SMEM;
    } else {
      k = nt2 ? (G == 32 ? COLI_SK(2, 32, 8) : COLI_SK(2, 64, 8)) : (G == 32 ? COLI_SK(1, 32, 8) : COLI_SK(1, 64, 8));
      smem = G == 32 ? SkCfg<32, 8>::SMEM : SkCfg<64, 8>::SMEM;
    }
#undef COLI_SK
    if (!launch_splitk(k, smem, maps, a, grid, di.sms, st)) return COLI_ERR_CUDA;
    rec.mark_through(6, 7);
    rec.mark(8);
    return COLI_OK;
  }
  {
    const long tiles = blocks_ub * (I / kRowBlock + H / kRowBlock);
    const int grid = static_cast<int>(tiles < di.sms ? tiles : di.sms);
    bool ok;
    if (G == 64)   // I % 512 == 0, T > 8
      ok = launch_ffn_for<256, 64>(T, maps, a, grid, st);
    else
      ok = kc_dn == 256 ? launch_ffn_for<256, 32>(T, maps, a, grid, st) : launch_ffn_for<128, 32>(T, maps, a, grid, st);
    if (!ok) return COLI_ERR_CUDA;
  }
  rec.mark_through(6, 7);
  if (T > kFusedCombineMaxT) {
    const long work = static_cast<long>(T) * (H / 4);
    long blocks = (work + 255) / 256;
    if (blocks > 4L * di.sms) blocks = 4L * di.sms;
    if (!launch(combine_kernel, dim3(static_cast<int>(blocks)), dim3(256), 0, st, static_cast<const float*>(ws.ypair),
                pair_pos, topk_w, residual, T, k, S, H, out, ep.on ? ep.ids : static_cast<const int32_t*>(nullptr),
                ep.on ? ep.begin : 0, ep.on ? ep.end : E, ep.on ? ep.out_f32 : static_cast<float*>(nullptr)))
      return COLI_ERR_CUDA;
  }
  rec.mark(8);
  return COLI_OK;
}

}  // namespace

extern "C" {

int coli_moe_version(void) { return 100; }

uint64_t coli_moe_launch_count(int reset) {
  const uint64_t v = t_launches;
  if (reset) t_launches = 0;
  return v;
}

coli_status coli_moe_set_stage_events(void* const* events, int n) {
  if (n < 0 || n > kMaxStageEvents || (n > 0 && !events)) return COLI_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) t_stage_ev[i] = static_cast<cudaEvent_t>(events[i]);
  t_stage_n = events ? n : 0;
  return COLI_OK;
}

const char* coli_status_str(coli_status s) {
  switch (s) {
    case COLI_OK: return "ok";
    case COLI_ERR_INVALID_ARG: return "invalid argument";
    case COLI_ERR_UNSUPPORTED: return "unsupported shape";
    case COLI_ERR_WORKSPACE: return "workspace too small";
    case COLI_ERR_CUDA: return "CUDA runtime error";
    case COLI_ERR_NONFINITE: return "non-finite router logits";
    case COLI_ERR_DEVICE: return "device-side error";
  }
  return "unknown status";
}

size_t coli_moe_workspace_bytes(const coli_moe_dims* dims, int T_max) {
  if (check_dims(dims) != COLI_OK || T_max < 0) return 0;
  // Enough for every batch of up to T_max tokens.  The layout grows with T
  // within each decode form, but the split-K form's partials at 8 tokens can
  // outweigh what the two-phase form needs for somewhat larger batches.
  size_t n = layout(dims, T_max, nullptr).bytes;
  if (T_max > kSkMaxT) {
    const size_t n_sk = layout(dims, kSkMaxT, nullptr).bytes;
    if (n_sk > n) n = n_sk;
  }
  return n;
}

coli_status coli_moe_union_offsets(const coli_moe_dims* dims, int T, size_t* off) {
  if (!off) return COLI_ERR_INVALID_ARG;
  const coli_status st = check_dims(dims);
  if (st != COLI_OK) return st;
  if (T < 0) return COLI_ERR_INVALID_ARG;
  if (static_cast<int64_t>(T) * dims->top_k > (int64_t(1) << 24)) return COLI_ERR_UNSUPPORTED;
  // the layout of a workspace based at address 0 gives the offsets (256-byte
  // aligned, so any workspace the calls accept has the same ones)
  uint8_t* const base = reinterpret_cast<uint8_t*>(uintptr_t(256));
  // int8 batches above 8 tokens run in 8-token passes: the last pass's union
  const Ws w = layout(dims, code_bits(dims) == 8 && T > kSkMaxT ? kSkMaxT : T, base);
  auto rel = [&](const void* p) { return static_cast<size_t>(static_cast<const uint8_t*>(p) - base); };
  off[0] = rel(w.unique);
  off[1] = rel(w.n_unique);
  off[2] = rel(w.seg_off);
  off[3] = rel(w.perm);
  off[4] = rel(w.pair_pos);
  return COLI_OK;
}

coli_status coli_moe_ffn_form(const coli_moe_dims* dims, int T, uint32_t flags, int* form) {
  if (!form) return COLI_ERR_INVALID_ARG;
  *form = 0;
  const coli_status st = check_dims(dims);
  if (st != COLI_OK) return st;
  if (T < 0) return COLI_ERR_INVALID_ARG;
  if (static_cast<int64_t>(T) * dims->top_k > (int64_t(1) << 24)) return COLI_ERR_UNSUPPORTED;
  if (T == 0) return COLI_OK;
  switch (choose_form(flags, T, dims)) {
    case Form::kInvalid: return COLI_ERR_INVALID_ARG;
    case Form::kUnsupported: return COLI_ERR_UNSUPPORTED;
    case Form::kPrefill: *form = COLI_FORM_PREFILL; return COLI_OK;
    case Form::kDecode:
      *form = (use_splitk(dims, T) || code_bits(dims) == 8) ? COLI_FORM_DECODE_SPLITK : COLI_FORM_DECODE_TWOPHASE;
      return COLI_OK;
  }
  return COLI_ERR_INVALID_ARG;
}

coli_status coli_moe_route(const float* logits, const float* bias, int T, int E, int k, int32_t* topk_ids,
                           float* topk_w, void* stream) {
  if (T < 0 || E < 1 || k < 1) return COLI_ERR_INVALID_ARG;
  if (E > 1024 || k > 32 || k > E) return COLI_ERR_UNSUPPORTED;
  if (T == 0) return COLI_OK;
  if (!logits || !topk_ids || !topk_w) return COLI_ERR_INVALID_ARG;
  DevInfo di;
  if (dev_info(&di) != COLI_OK) return COLI_ERR_CUDA;
  return launch_route(logits, bias, T, E, k, topk_ids, topk_w, di.status, as_stream(stream)) ? COLI_OK
                                                                                           : COLI_ERR_CUDA;
}

coli_status coli_moe_union(const int32_t* topk_ids, int T, int k, int E, int32_t* unique_ids, int32_t* n_unique,
                           int32_t* seg_off, int32_t* perm, int32_t* pair_pos, void* stream) {
  if (T < 0 || k < 1 || E < 1) return COLI_ERR_INVALID_ARG;
  if (E > 1024 || k > 32 || static_cast<int64_t>(T) * k > (int64_t(1) << 24)) return COLI_ERR_UNSUPPORTED;
  if (!n_unique || !seg_off) return COLI_ERR_INVALID_ARG;
  if (T > 0 && (!topk_ids || !unique_ids || !perm || !pair_pos)) return COLI_ERR_INVALID_ARG;
  DevInfo di;
  if (dev_info(&di) != COLI_OK) return COLI_ERR_CUDA;
  return launch(union_kernel, dim3(1), dim3(kUnionThreads), static_cast<size_t>(kUnionWarps) * E * 4,
                as_stream(stream), topk_ids, T * k, E, unique_ids, n_unique, seg_off, perm, pair_pos, di.status, T, 0, 8,
                static_cast<int32_t*>(nullptr), static_cast<int32_t*>(nullptr), static_cast<int32_t*>(nullptr), 0)
             ? COLI_OK
             : COLI_ERR_CUDA;
}

coli_status coli_moe_expert_ffn(const coli_moe_dims* dims, const coli_moe_weights* w, const uint16_t* x, int T,
                                const int32_t* topk_ids, const float* topk_w, const int32_t* unique_ids,
                                const int32_t* n_unique, const int32_t* seg_off, const int32_t* perm,
                                const int32_t* pair_pos, const uint16_t* residual, uint16_t* out, uint32_t flags,
                                void* ws, size_t ws_bytes, void* stream) {
  coli_status st = check_dims(dims);
  if (st != COLI_OK) return st;
  if (T < 0) return COLI_ERR_INVALID_ARG;
  if (static_cast<int64_t>(T) * dims->top_k > (int64_t(1) << 24)) return COLI_ERR_UNSUPPORTED;
  if ((st = check_weights(w, false)) != COLI_OK) return st;
  if (flags & (COLI_LAYER_HOST_X | COLI_LAYER_HOST_OUT)) return COLI_ERR_UNSUPPORTED;   // device buffers only
  if (T == 0) return COLI_OK;
  if (!x || !topk_ids || !topk_w || !unique_ids || !n_unique || !seg_off || !perm || !pair_pos || !out || !ws)
    return COLI_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(out, 16) || (residual && !aligned(residual, 16)) || !aligned(ws, 256))
    return COLI_ERR_INVALID_ARG;
  if (x == out) return COLI_ERR_INVALID_ARG;
  const Form form = choose_form(flags, T, dims);
  if (form == Form::kInvalid) return COLI_ERR_INVALID_ARG;
  if (form == Form::kUnsupported) return COLI_ERR_UNSUPPORTED;
  const Ws lay = layout(dims, T, ws);
  if (ws_bytes < lay.bytes) return COLI_ERR_WORKSPACE;
  DevInfo di;
  if (dev_info(&di) != COLI_OK) return COLI_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  const StageRecorder rec(s);
  rec.mark(0);
  if (!launch(prep_kernel, dim3(T), dim3(256), 0, s, x, dims->hidden, 0, static_cast<uint16_t*>(nullptr), lay.xq,
              lay.xp, lay.xe, form == Form::kPrefill ? 1 : 0, di.status))
    return COLI_ERR_CUDA;
  rec.mark_through(1, 4);
  if (form == Form::kPrefill)
    return run_ffn_prefill(dims, w, T, unique_ids, n_unique, seg_off, perm, pair_pos, topk_w, residual, out, lay, di,
                           s, rec);
  if (!launch(plan_kernel, dim3(1), dim3(1024), 0, s, n_unique, seg_off, T, dims->n_shared, tok_block(T), lay.plan,
              lay.tb_done, lay.rb_done, dims->hidden / kRowBlock))
    return COLI_ERR_CUDA;
  rec.mark(5);
  return run_ffn(dims, w, T, unique_ids, n_unique, seg_off, perm, pair_pos, topk_w, residual, out, lay, di, s, rec);
}

// A host-RAM tier as the kernels see it: the slot count, the device state and
// the copy description (host sources through their device addresses).
struct TierArgs {
  int slots;
  void* state;
  TierCopy cp;
};

namespace {

// The device address of page-locked, mapped host memory, or NULL for any
// other pointer (device memory, or host memory the device cannot reach).
const void* host_mapped(const void* p) {
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
}

coli_status layer_impl(const coli_moe_dims* dims, const coli_moe_weights* w, const uint16_t* x, int T,
                       const float* logits_in, const uint16_t* residual, uint32_t flags, uint16_t* out,
                       float* logits_out, int32_t* topk_ids_out, float* topk_w_out, void* ws, size_t ws_bytes,
                       void* stream, EpRange ep, const TierArgs* tier = nullptr) {
  coli_status st = check_dims(dims);
  if (st != COLI_OK) return st;
  if (T < 0) return COLI_ERR_INVALID_ARG;
  if (static_cast<int64_t>(T) * dims->top_k > (int64_t(1) << 24)) return COLI_ERR_UNSUPPORTED;
  if (ep.on && (ep.begin < 0 || ep.end > dims->n_experts || ep.begin >= ep.end)) return COLI_ERR_INVALID_ARG;
  if ((st = check_weights(w, logits_in == nullptr)) != COLI_OK) return st;
  if (T == 0) return COLI_OK;
  if (!x || !ws || (ep.on ? !ep.out_f32 : !out)) return COLI_ERR_INVALID_ARG;
  if (!aligned(x, 16) || (out && !aligned(out, 16)) || (ep.out_f32 && !aligned(ep.out_f32, 16)) ||
      (residual && !aligned(residual, 16)) || !aligned(ws, 256))
    return COLI_ERR_INVALID_ARG;
  if (x == out || x == reinterpret_cast<const void*>(ep.out_f32)) return COLI_ERR_INVALID_ARG;
  const Form form = choose_form(flags, T, dims);
  if (form == Form::kInvalid) return COLI_ERR_INVALID_ARG;
  if (form == Form::kUnsupported) return COLI_ERR_UNSUPPORTED;
  // int8 codes above 8 tokens: consecutive passes of up to 8 tokens through
  // the split-K form, each a whole layer call on its rows (every token's output
  // is the bits of its batch-1 output; the weights are read once per pass)
  if (code_bits(dims) == 8 && T > kSkMaxT) {
    const int H = dims->hidden, E = dims->n_experts, k = dims->top_k;
    for (int t0 = 0; t0 < T; t0 += kSkMaxT) {
      const int tc = std::min(kSkMaxT, T - t0);
      const size_t oh = static_cast<size_t>(t0) * H, oe = static_cast<size_t>(t0) * E, ok = static_cast<size_t>(t0) * k;
      EpRange epc = ep;
      if (ep.out_f32) epc.out_f32 = ep.out_f32 + oh;
      const coli_status sc = layer_impl(dims, w, x + oh, tc, logits_in ? logits_in + oe : nullptr,
                                        residual ? residual + oh : nullptr, flags, out ? out + oh : nullptr,
                                        logits_out ? logits_out + oe : nullptr, topk_ids_out ? topk_ids_out + ok : nullptr,
                                        topk_w_out ? topk_w_out + ok : nullptr, ws, ws_bytes, stream, epc, tier);
      if (sc != COLI_OK) return sc;
    }
    return COLI_OK;
  }
  // a host-RAM tier: decode form, no expert-parallel share, and every batch's
  // union must fit the slots
  if (tier && (form != Form::kDecode || ep.on ||
               std::min<int64_t>(dims->n_experts, static_cast<int64_t>(T) * dims->top_k) > tier->slots))
    return COLI_ERR_UNSUPPORTED;
  // host-memory input and output: page-locked and mapped, used through their
  // device addresses (an expert-parallel share writes an fp32 partial instead)
  const bool host_x = (flags & COLI_LAYER_HOST_X) != 0, host_out = (flags & COLI_LAYER_HOST_OUT) != 0;
  if ((host_x || host_out) && ep.on) return COLI_ERR_UNSUPPORTED;
  const uint16_t* xh = nullptr;
  const uint16_t* rh = nullptr;
  if (host_x) {
    xh = static_cast<const uint16_t*>(host_mapped(x));
    rh = residual ? static_cast<const uint16_t*>(host_mapped(residual)) : nullptr;
    if (!xh || (residual && !rh)) return COLI_ERR_INVALID_ARG;
  }
  if (host_out) {
    out = static_cast<uint16_t*>(const_cast<void*>(host_mapped(out)));
    if (!out) return COLI_ERR_INVALID_ARG;
  }
  // an expert-parallel share runs in the prefill form, or in the decode forms
  // with route, union and plan in one kernel (T <= 128) and not through the
  // two-phase kernel's own combine (T <= 4 with I = 128)
  if (ep.on && !(form == Form::kPrefill || (form == Form::kDecode && T <= kFusedRouteMaxT &&
                                            (use_splitk(dims, T) || T > kFusedCombineMaxT))))
    return COLI_ERR_UNSUPPORTED;
  const Ws lay = layout(dims, T, ws);
  if (ws_bytes < lay.bytes) return COLI_ERR_WORKSPACE;
  DevInfo di;
  if (dev_info(&di) != COLI_OK) return COLI_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  const int H = dims->hidden, E = dims->n_experts, k = dims->top_k;
  const bool prenorm = (flags & COLI_LAYER_PRENORM) != 0;
  const StageRecorder rec(s);
  rec.mark(0);
  if (host_x) {
    // the rows into the workspace (a residual that is x itself is copied once)
    const bool rsep = rh && rh != xh;
    const long n16 = static_cast<long>(T) * H / 8;
    long blocks = (n16 + 255) / 256;
    if (blocks > 4L * di.sms) blocks = 4L * di.sms;
    if (!launch(stage_rows_kernel, dim3(static_cast<int>(blocks)), dim3(256), 0, s, reinterpret_cast<const uint4*>(xh),
                reinterpret_cast<uint4*>(lay.xin), rsep ? reinterpret_cast<const uint4*>(rh) : nullptr,
                rsep ? reinterpret_cast<uint4*>(lay.rin) : nullptr, n16))
      return COLI_ERR_CUDA;
    x = lay.xin;
    residual = rh ? (rsep ? lay.rin : lay.xin) : nullptr;
  }
  const int S = dims->n_shared, tokb = tok_block(T);
  // the split-K kernel routes the batch itself: no routing kernel runs
  const bool inroute = form == Form::kDecode && splitk_routes(dims, T) && !tier;

  // 1. expert input (fragment order, optional pre-norm) and router logits
  float* lo = logits_out ? logits_out : lay.logits;
  const float* lg = logits_in;
  const bool fused_front = T <= 8;
  if (fused_front) {
    const float* wr = logits_in ? nullptr : w->router_w;
    const int grid = (logits_in ? 0 : E) + T;
    if (!launch(front_kernel, dim3(grid), dim3(256), 0, s, x, wr, T, E, H, prenorm ? 1 : 0, lo, lay.xn, lay.xq,
                lay.xp, lay.xe, form == Form::kPrefill ? 1 : 0, di.status, inroute ? lay.rb_done : nullptr))
      return COLI_ERR_CUDA;
    rec.mark_through(1, 2);
    if (!logits_in) lg = lo;
  } else {
    if (!launch(prep_kernel, dim3(T), dim3(256), 0, s, x, H, prenorm ? 1 : 0, lay.xn, lay.xq,
                static_cast<uint8_t*>(nullptr), static_cast<int32_t*>(nullptr), form == Form::kPrefill ? 1 : 0,
                di.status))
      return COLI_ERR_CUDA;
    rec.mark(1);
    if (!logits_in) {
      const uint16_t* xr = prenorm ? lay.xn : x;
      if (T >= kLogitsMmaMinT) {
        // prefill-sized batches: tensor cores (bf16 pieces of W_r)
        if (!launch(logits_mma_kernel, dim3((E + kLgBN - 1) / kLgBN, (T + kLgBM - 1) / kLgBM), dim3(256), 0, s,
                    xr, w->router_w, T, E, H, lo))
          return COLI_ERR_CUDA;
      } else {
        const int tt = logits_tokens_per_block(H);
        if (!launch(logits_tile_kernel, dim3((E + 7) / 8, (T + tt - 1) / tt), dim3(256),
                    static_cast<size_t>(tt) * H * 2, s, xr, w->router_w, T, E, H, tt, lo))
          return COLI_ERR_CUDA;
      }
      lg = lo;
    }
    rec.mark(2);
  }
  if (logits_in && logits_out && logits_out != logits_in) {
    if (cudaMemcpyAsync(logits_out, logits_in, static_cast<size_t>(T) * E * 4, cudaMemcpyDeviceToDevice, s) !=
        cudaSuccess)
      return COLI_ERR_CUDA;
  }
  // 2. route, union and the FFN tile plan
  int32_t* ids = topk_ids_out ? topk_ids_out : lay.ids;
  float* tw = topk_w_out ? topk_w_out : lay.w;
  if (inroute) {
    rec.mark_through(3, 5);
  } else if (T <= kFusedRouteMaxT) {
    if (!launch_route_union(lg, w->router_bias, T, E, k, ep.on ? ep.shared : S, tokb, H / kRowBlock, ids, tw, lay,
                            di.status, s, ep.on ? ep.begin : 0, ep.on ? ep.end : E))
      return COLI_ERR_CUDA;
    rec.mark_through(3, 5);
  } else {
    if (!launch_route(lg, w->router_bias, T, E, k, ids, tw, di.status, s)) return COLI_ERR_CUDA;
    rec.mark(3);
    const int P = T * k;
    if (form == Form::kPrefill) {
      // many-CTA union; the prefill form computes its own tile plan afterwards
      const int chunk = union_chunk(P), NB = (P + chunk - 1) / chunk;
      const int32_t* cids = ids;
      if (!launch(union_count_kernel, dim3(NB), dim3(1024), static_cast<size_t>(E) * 4, s, cids, P, E, chunk, lay.ucnt,
                  di.status) ||
          !launch(union_scan_kernel, dim3(1), dim3(1024), 0, s, lay.ucnt, NB, E, lay.unique, lay.n_unique,
                  lay.seg_off) ||
          !launch(union_scatter_kernel, dim3(NB), dim3(kUnionThreads), static_cast<size_t>(kUnionWarps) * E * 4, s,
                  cids, P, E, chunk, static_cast<const int32_t*>(lay.ucnt), lay.perm, lay.pair_pos))
        return COLI_ERR_CUDA;
    } else if (!launch(union_kernel, dim3(1), dim3(kUnionThreads), static_cast<size_t>(kUnionWarps) * E * 4, s,
                       static_cast<const int32_t*>(ids), P, E, lay.unique, lay.n_unique, lay.seg_off, lay.perm,
                       lay.pair_pos, di.status, T, S, tokb, lay.plan, lay.tb_done, lay.rb_done, H / kRowBlock)) {
      return COLI_ERR_CUDA;
    }
    rec.mark_through(4, 5);
  }
  // 3. expert FFN and combine
  ep.ids = ids;
  if (form == Form::kPrefill)
    return run_ffn_prefill(dims, w, T, lay.unique, lay.n_unique, lay.seg_off, lay.perm, lay.pair_pos, tw, residual,
                           out, lay, di, s, rec, ep);
  InRoute ir;
  if (inroute) {
    ir.logits = lg;
    ir.bias = w->router_bias;
    ir.ids = ids;
    ir.w = tw;
  }
  if (tier) {
    // Place (and Learn): the union's experts into slots, the misses copied in
    // from host memory; the FFN then reads the slots
    if (!launch(tier_place_kernel, dim3(1), dim3(256), 0, s, static_cast<const int32_t*>(lay.unique), 0,
                static_cast<const int32_t*>(lay.n_unique), static_cast<const int32_t*>(lay.seg_off), E, tier->slots,
                tier->state, lay.sunique, di.status) ||
        !launch(tier_fill_kernel, dim3(4 * di.sms), dim3(256), 0, s, tier->cp, tier->state, E, tier->slots))
      return COLI_ERR_CUDA;
    rec.mark(5);   // the stage before the FFN ends after the copies
    return run_ffn(dims, w, T, lay.sunique, lay.n_unique, lay.seg_off, lay.perm, lay.pair_pos, tw, residual, out,
                   lay, di, s, rec, ep, ir, tier->slots);
  }
  return run_ffn(dims, w, T, lay.unique, lay.n_unique, lay.seg_off, lay.perm, lay.pair_pos, tw, residual, out, lay,
                 di, s, rec, ep, ir);
}

}  // namespace

coli_status coli_moe_layer(const coli_moe_dims* dims, const coli_moe_weights* w, const uint16_t* x, int T,
                           const float* logits_in, const uint16_t* residual, uint32_t flags, uint16_t* out,
                           float* logits_out, int32_t* topk_ids_out, float* topk_w_out, void* ws, size_t ws_bytes,
                           void* stream) {
  return layer_impl(dims, w, x, T, logits_in, residual, flags, out, logits_out, topk_ids_out, topk_w_out, ws,
                    ws_bytes, stream, EpRange());
}

coli_status coli_moe_layer_ep(const coli_moe_dims* dims, const coli_moe_weights* w, int expert_begin,
                              int expert_end, int with_shared, const uint16_t* x, int T, const float* logits_in,
                              const uint16_t* residual, uint32_t flags, float* out_partial, float* logits_out,
                              int32_t* topk_ids_out, float* topk_w_out, void* ws, size_t ws_bytes, void* stream) {
  EpRange ep;
  ep.on = true;
  ep.begin = expert_begin;
  ep.end = expert_end;
  ep.shared = with_shared ? (dims ? dims->n_shared : 0) : 0;
  ep.out_f32 = out_partial;
  return layer_impl(dims, w, x, T, logits_in, residual, flags, nullptr, logits_out, topk_ids_out, topk_w_out, ws,
                    ws_bytes, stream, ep);
}

namespace {

// out = bf16(in), four values per thread.
__global__ void __launch_bounds__(256) partial_to_bf16_kernel(const float4* __restrict__ in, uint2* __restrict__ out,
                                                             size_t n4) {
  pdl_wait();
  pdl_trigger();
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 v = in[i];
    uint2 o;
    o.x = float_to_bf16_bits(v.x) | (static_cast<uint32_t>(float_to_bf16_bits(v.y)) << 16);
    o.y = float_to_bf16_bits(v.z) | (static_cast<uint32_t>(float_to_bf16_bits(v.w)) << 16);
    out[i] = o;
  }
}

}  // namespace

coli_status coli_moe_partial_to_bf16(const float* partial, uint16_t* out, size_t n, void* stream) {
  if (n == 0) return COLI_OK;
  if (!partial || !out || n % 4 != 0 || !aligned(partial, 16) || !aligned(out, 8)) return COLI_ERR_INVALID_ARG;
  DevInfo di;
  if (dev_info(&di) != COLI_OK) return COLI_ERR_CUDA;
  const size_t n4 = n / 4;
  size_t blocks = (n4 + 255) / 256;
  if (blocks > static_cast<size_t>(4) * di.sms) blocks = static_cast<size_t>(4) * di.sms;
  return launch(partial_to_bf16_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, as_stream(stream),
                reinterpret_cast<const float4*>(partial), reinterpret_cast<uint2*>(out), n4)
             ? COLI_OK
             : COLI_ERR_CUDA;
}

coli_status coli_moe_layer_noalloc(const coli_moe_dims* dims, const coli_moe_weights* w, const uint16_t* x, int T,
                                   const float* logits_in, const uint16_t* residual, uint32_t flags, uint16_t* out,
                                   float* logits_out, int32_t* topk_ids_out, float* topk_w_out, void* stream) {
  static std::mutex mu;
  static void* scratch_ptr[kMaxDevices] = {};
  const coli_status st = check_dims(dims);
  if (st != COLI_OK) return st;
  if (T < 0) return COLI_ERR_INVALID_ARG;
  if (coli_moe_workspace_bytes(dims, T) > COLI_NOALLOC_SCRATCH_BYTES) return COLI_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return COLI_ERR_CUDA;
  void* ptr = nullptr;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (!scratch_ptr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return COLI_ERR_CUDA;
      scratch_ptr[dev] = p;
    }
    ptr = scratch_ptr[dev];
  }
  return coli_moe_layer(dims, w, x, T, logits_in, residual, flags, out, logits_out, topk_ids_out, topk_w_out, ptr,
                        COLI_NOALLOC_SCRATCH_BYTES, stream);
}

namespace {

// Checks a tier against the dims (and, with `slots`, the device slot arrays)
// and fills the kernels' view of it.
coli_status tier_args(const coli_moe_dims* d, const coli_moe_tier* t, const coli_moe_weights* slots,
                      TierArgs* out) {
  coli_status st = check_dims(d);
  if (st != COLI_OK) return st;
  if (!t || !t->state || !aligned(t->state, 256)) return COLI_ERR_INVALID_ARG;
  if (t->n_slots < 1 || t->n_slots > d->n_experts) return COLI_ERR_INVALID_ARG;
  *out = TierArgs{};
  out->slots = t->n_slots;
  out->state = t->state;
  if (!slots) return COLI_OK;
  const size_t H = d->hidden, I = d->inter, G = d->group, B = code_bits(d);
  const size_t qg = I * H * B / 8, qd = H * I * B / 8, sg = I * (H / G) * 2, sd = H * (I / G) * 2;
  const void* hs[6] = {t->gate_q, t->up_q, t->down_q, t->gate_s, t->up_s, t->down_s};
  const void* ds[6] = {slots->gate_q, slots->up_q, slots->down_q, slots->gate_s, slots->up_s, slots->down_s};
  const size_t per[6] = {qg, qg, qd, sg, sg, sd};
  for (int m = 0; m < 6; ++m) {
    if (per[m] % 16) return COLI_ERR_UNSUPPORTED;
    if (!hs[m] || !ds[m] || !aligned(hs[m], 16) || !aligned(ds[m], 16)) return COLI_ERR_INVALID_ARG;
    const void* dev = host_mapped(hs[m]);
    if (!dev) return COLI_ERR_INVALID_ARG;
    out->cp.src[m] = static_cast<const uint4*>(dev);
    out->cp.dst[m] = static_cast<uint4*>(const_cast<void*>(ds[m]));
    out->cp.per[m] = static_cast<long>(per[m] / 16);
  }
  return COLI_OK;
}

}  // namespace

size_t coli_moe_tier_state_bytes(const coli_moe_dims* dims, int32_t n_slots) {
  if (check_dims(dims) != COLI_OK || n_slots < 1 || n_slots > dims->n_experts) return 0;
  return align256(tier_state_words(dims->n_experts, n_slots) * 4);
}

coli_status coli_moe_tier_reset(const coli_moe_dims* dims, const coli_moe_tier* tier, void* stream) {
  TierArgs ta;
  coli_status st = tier_args(dims, tier, nullptr, &ta);
  if (st != COLI_OK) return st;
  DevInfo di;
  if (dev_info(&di) != COLI_OK) return COLI_ERR_CUDA;
  const int n = std::max(dims->n_experts, ta.slots);
  return launch(tier_reset_kernel, dim3((n + 255) / 256), dim3(256), 0, as_stream(stream), ta.state,
                dims->n_experts, ta.slots)
             ? COLI_OK
             : COLI_ERR_CUDA;
}

coli_status coli_moe_layer_tiered(const coli_moe_dims* dims, const coli_moe_weights* slots, const coli_moe_tier* tier,
                                  const uint16_t* x, int T, const float* logits_in, const uint16_t* residual,
                                  uint32_t flags, uint16_t* out, float* logits_out, int32_t* topk_ids_out,
                                  float* topk_w_out, void* ws, size_t ws_bytes, void* stream) {
  TierArgs ta;
  coli_status st = tier_args(dims, tier, slots, &ta);
  if (st != COLI_OK) return st;
  return layer_impl(dims, slots, x, T, logits_in, residual, flags, out, logits_out, topk_ids_out, topk_w_out, ws,
                    ws_bytes, stream, EpRange(), &ta);
}

coli_status coli_moe_tier_prefetch(const coli_moe_dims* dims, const coli_moe_weights* slots,
                                   const coli_moe_tier* tier, const int32_t* ids, int32_t n, void* stream) {
  TierArgs ta;
  coli_status st = tier_args(dims, tier, slots, &ta);
  if (st != COLI_OK) return st;
  if (n < 0 || n > ta.slots || (n > 0 && (!ids || !aligned(ids, 4)))) return COLI_ERR_INVALID_ARG;
  if (n == 0) return COLI_OK;
  DevInfo di;
  if (dev_info(&di) != COLI_OK) return COLI_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  return launch(tier_place_kernel, dim3(1), dim3(256), 0, s, ids, static_cast<int>(n),
                static_cast<const int32_t*>(nullptr), static_cast<const int32_t*>(nullptr), dims->n_experts,
                ta.slots, ta.state, static_cast<int32_t*>(nullptr), di.status) &&
                 launch(tier_fill_kernel, dim3(4 * di.sms), dim3(256), 0, s, ta.cp, ta.state, dims->n_experts,
                        ta.slots)
             ? COLI_OK
             : COLI_ERR_CUDA;
}

coli_status coli_moe_tier_lookahead(const coli_moe_dims* dims, const coli_moe_weights* next,
                                    const coli_moe_tier* next_tier, const uint16_t* x, int T, uint32_t flags,
                                    void* ws, size_t ws_bytes, void* stream) {
  TierArgs ta;
  coli_status st = tier_args(dims, next_tier, next, &ta);
  if (st != COLI_OK) return st;
  if ((st = check_weights(next, true)) != COLI_OK) return st;
  if (T < 0) return COLI_ERR_INVALID_ARG;
  if (T == 0) return COLI_OK;
  const int H = dims->hidden, E = dims->n_experts, k = dims->top_k;
  if (std::min<int64_t>(E, static_cast<int64_t>(T) * k) > ta.slots) return COLI_ERR_UNSUPPORTED;
  if (!x || !ws || !aligned(x, 16) || !aligned(ws, 256)) return COLI_ERR_INVALID_ARG;
  const Ws lay = layout(dims, T, ws);
  if (ws_bytes < lay.bytes) return COLI_ERR_WORKSPACE;
  DevInfo di;
  if (dev_info(&di) != COLI_OK) return COLI_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  const int prenorm = (flags & COLI_LAYER_PRENORM) ? 1 : 0;
  // the next layer's logits of x, as its own call would compute them
  if (T <= 8) {
    if (!launch(front_kernel, dim3(E + T), dim3(256), 0, s, x, next->router_w, T, E, H, prenorm, lay.logits, lay.xn,
                lay.xq, static_cast<uint8_t*>(nullptr), static_cast<int32_t*>(nullptr), 0, di.status,
                static_cast<int32_t*>(nullptr)))
      return COLI_ERR_CUDA;
  } else {
    if (!launch(prep_kernel, dim3(T), dim3(256), 0, s, x, H, prenorm, lay.xn, lay.xq, static_cast<uint8_t*>(nullptr),
                static_cast<int32_t*>(nullptr), 0, di.status))
      return COLI_ERR_CUDA;
    const uint16_t* xr = prenorm ? lay.xn : x;
    if (T >= kLogitsMmaMinT) {
      if (!launch(logits_mma_kernel, dim3((E + kLgBN - 1) / kLgBN, (T + kLgBM - 1) / kLgBM), dim3(256), 0, s, xr,
                  next->router_w, T, E, H, lay.logits))
        return COLI_ERR_CUDA;
    } else {
      const int tt = logits_tokens_per_block(H);
      if (!launch(logits_tile_kernel, dim3((E + 7) / 8, (T + tt - 1) / tt), dim3(256), static_cast<size_t>(tt) * H * 2,
                  s, xr, next->router_w, T, E, H, tt, lay.logits))
        return COLI_ERR_CUDA;
    }
  }
  // its top-k, then the selected experts placed (repeats are placed once)
  if (!launch_route(lay.logits, next->router_bias, T, E, k, lay.ids, lay.w, di.status, s)) return COLI_ERR_CUDA;
  return launch(tier_place_kernel, dim3(1), dim3(256), 0, s, static_cast<const int32_t*>(lay.ids), T * k,
                static_cast<const int32_t*>(nullptr), static_cast<const int32_t*>(nullptr), E, ta.slots, ta.state,
                static_cast<int32_t*>(nullptr), di.status) &&
                 launch(tier_fill_kernel, dim3(4 * di.sms), dim3(256), 0, s, ta.cp, ta.state, E, ta.slots)
             ? COLI_OK
             : COLI_ERR_CUDA;
}

coli_status coli_moe_test_wait_timeout(uint64_t limit_ns, uint64_t* elapsed_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > kWaitLimitNs) return COLI_ERR_INVALID_ARG;
  if (elapsed_ns && !aligned(elapsed_ns, 8)) return COLI_ERR_INVALID_ARG;
  DevInfo di;
  if (dev_info(&di) != COLI_OK) return COLI_ERR_CUDA;
  return launch(wait_timeout_kernel, dim3(1), dim3(32), 0, as_stream(stream), limit_ns, elapsed_ns, di.status)
             ? COLI_OK
             : COLI_ERR_CUDA;
}

coli_status coli_moe_get_status(void* stream, uint32_t* flags) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return COLI_ERR_CUDA;
  DevInfo di;
  if (dev_info(&di) != COLI_OK) return COLI_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpy(&v, di.status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return COLI_ERR_CUDA;
  const uint32_t zero = 0;
  if (cudaMemcpy(di.status, &zero, 4, cudaMemcpyHostToDevice) != cudaSuccess) return COLI_ERR_CUDA;
  if (flags) *flags = v;
  if (v == 0) return COLI_OK;
  if (v == COLI_FLAG_NONFINITE) return COLI_ERR_NONFINITE;
  return COLI_ERR_DEVICE;
}

}  // extern "C"
