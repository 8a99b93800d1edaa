/*
 * coli_moe.h -- C ABI of the B200 routed-expert MoE step
 *               (Route -> Union -> int4 SwiGLU expert FFN -> combine).
 *
 * The per-token path this library computes is the one the Colibri README
 * describes ("Come funziona", "Il percorso di ogni token": every layer of
 * every token goes Route, then Union, before the expert matmuls) and the
 * getting-started guide lists ("トークンごとの処理経路", steps 1 Route and
 * 2 Union).  The pages fix that the router picks experts per token and per
 * layer, that a batch reads each unique expert once (README, "Mai aspettare il
 * disco due volte": batch-union), that routed experts are stored int4
 * (README, "L'idea") and that placement never changes the router's decisions
 * or the weights' precision.  Placement itself (VRAM/RAM/disk tiering) is not
 * part of this library: every expert is resident in device memory (the
 * README's full expert residence, "Una gerarchia di memoria").
 *
 * Numerics this library implements (the pages give no formula):
 *   logits   l[t,e] = sum_h x[t,h] * W_r[e,h]           (fp32, x bf16)
 *   bias     l'[t,e] = l[t,e] + bias[e]                 (one fp32 add; optional)
 *   route    top-k of l' by (value desc, index asc); slot j = j-th in that order;
 *            w_j = exp(l'_j - l'_max) / sum_{i<k} exp(l'_i - l'_max)
 *   union    unique experts ascending; pairs p = t*k + j grouped by expert,
 *            stable in p
 *   expert   W = code * scale, code int4 in [-8,7] (or int8 in [-128,127]),
 *            fp16 scale per G along K;
 *            h = bf16( silu(W_gate x) * (W_up x) ),  y = W_down h   (fp32 accumulate)
 *   combine  out[t] = bf16( sum_j w[t,j] * y_{id[t,j]} + sum_s y_{E+s} + residual[t] )
 *
 * Container format (row-major, K contiguous):
 *   gate_q, up_q  uint8 [E+S][I][H/2]   down_q uint8 [E+S][H][I/2]
 *   gate_s, up_s  fp16  [E+S][I][H/G]   down_s fp16  [E+S][H][I/G]
 *   G = dims.group = 32, or 64 for the group-scaled "gs64" container the
 *   README recommends ("2. Scarica il modello"): scale c / G of a row
 *   multiplies its element c.
 *   Element c of a row is nibble (c & 1) of byte c/2 (low nibble first); the
 *   nibble n encodes code n - 16*(n >= 8).  Shared experts are ids E..E+S-1.
 *   int8 container (dims.code_bits == 8; the README requires the MTP head to
 *   be int8, "Decodifica speculativa, onestamente"): the same layout with one
 *   two's-complement byte per code, gate_q/up_q [E+S][I][H], down_q
 *   [E+S][H][I].  It runs in the split-K decode form (I a multiple of 256):
 *   batches of up to 8 tokens (the MTP head's draft batches) in one pass,
 *   larger ones in consecutive 8-token passes (each token's output is that of
 *   its batch-1 call; the weights are read once per pass); COLI_PATH_PREFILL
 *   returns COLI_ERR_UNSUPPORTED.
 *
 * Conventions for every call:
 *   - Every pointer is a DEVICE pointer owned by the caller, unless stated.
 *     The library allocates no memory at run time, keeps no per-call state
 *     and does not retain pointers after the call returns.  Its only device
 *     memory is file-scope: a status word per device and the fixed scratch
 *     array of coli_moe_layer_noalloc (COLI_NOALLOC_SCRATCH_BYTES), which
 *     exist once the library is loaded.
 *   - bf16 / fp16 tensors are passed as uint16_t bit patterns.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *     enqueue work on it: they never synchronise, never allocate, and can be
 *     captured into a CUDA graph (except coli_moe_get_status).
 *   - Argument errors are reported synchronously, before anything is
 *     launched.  Errors found on the device (non-finite logits, expert ids out
 *     of range, a pipeline wait that timed out) set bits in a per-device
 *     status word that coli_moe_get_status reads and clears; kernels never
 *     trap.
 *   - Supported shapes: group == 32 with H % 256 == 0, I % 256 == 0 or
 *     I == 128; group == 64 with H % 512 == 0, I % 512 == 0; int8 codes
 *     need I % 256 == 0 (group 32) or I % 512 == 0 (group 64); and for all
 *     1 <= k <= min(E, 32), E <= 1024, 0 <= S <= 4, T >= 0, T*k <= 2^24.
 *     Anything else returns COLI_ERR_UNSUPPORTED.
 *   - Thread safety: calls may be made concurrently from several host
 *     threads on different streams; the device status word is shared by all
 *     of them.
 */
#ifndef COLI_MOE_H
#define COLI_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  COLI_OK = 0,
  COLI_ERR_INVALID_ARG = 1,  /* NULL where a pointer is required, negative size, bad stride */
  COLI_ERR_UNSUPPORTED = 2,  /* shape outside the supported set above */
  COLI_ERR_WORKSPACE = 3,    /* ws_bytes smaller than coli_moe_workspace_bytes() */
  COLI_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, attribute, symbol) */
  COLI_ERR_NONFINITE = 5,    /* returned by coli_moe_get_status only */
  COLI_ERR_DEVICE = 6        /* returned by coli_moe_get_status: other device-side error bits */
} coli_status;

/* Device status bits (coli_moe_get_status). */
#define COLI_FLAG_NONFINITE 0x1u  /* a logit was NaN or +inf, or a selected logit was -inf */
#define COLI_FLAG_BAD_ID    0x2u  /* an expert id outside [0, E) reached the union */
#define COLI_FLAG_TIMEOUT   0x4u  /* a bounded pipeline wait expired; outputs are undefined */
#define COLI_FLAG_RANGE     0x8u  /* the prefill form met an expert input or h value of magnitude
                                   * 65536 or more, which its fp16 operands cannot hold; outputs
                                   * are undefined */

/* Layer flags (coli_moe_layer / coli_moe_expert_ffn). */
#define COLI_LAYER_PRENORM       0x1u  /* route and run the experts on n = bf16(x * rsqrt(mean(x^2) + 1e-6)) */
#define COLI_LAYER_HOST_X        0x2u  /* coli_moe_layer / _noalloc: x (and the residual, if given) are in
                                        * page-locked host memory mapped into the device's address space
                                        * (cudaHostAlloc, cudaHostRegister with cudaHostRegisterMapped);
                                        * one kernel copies the rows into the workspace before use */
#define COLI_LAYER_HOST_OUT      0x4u  /* coli_moe_layer / _noalloc: out is in such host memory; the
                                        * call's last kernel writes the bf16 rows there directly */
/* With either HOST flag, a pointer the device cannot reach (pageable host
 * memory) returns COLI_ERR_INVALID_ARG; the expert-parallel entry returns
 * COLI_ERR_UNSUPPORTED.  For small decode batches these replace two
 * cudaMemcpyAsync calls and their latency. */
#define COLI_PATH_DECODE         0x10u /* force the decode FFN form (weights streamed once, mma.sync) */
#define COLI_PATH_PREFILL        0x20u /* force the prefill FFN form (tcgen05 grouped GEMM) */
/* With neither flag the prefill form is taken when T >= 32 and T*k >= 32*min(E, T*k)
 * (at least 32 tokens per expert on average), else the decode form.  Both flags
 * together return COLI_ERR_INVALID_ARG.  The decode form runs as one kernel
 * either way: for T <= 8 (and I a multiple of 256) each gate/up tile's CTA
 * also computes that tile's K slice of the down projection (fixed-order
 * partial sums; a token's output is the same bits in any batch of up to 8);
 * otherwise gate/up tiles and then down tiles, in blocks of 16 (T <= 64) or
 * 32 tokens.  int8 codes (dims.code_bits == 8) take the first only, in 8-token
 * passes above 8 tokens. */

typedef struct {
  int32_t hidden;     /* H */
  int32_t inter;      /* I: expert intermediate size */
  int32_t n_experts;  /* E: routed experts */
  int32_t top_k;      /* k */
  int32_t n_shared;   /* S: shared experts, always active with weight 1.0 */
  int32_t group;      /* quantisation group along K: 32 or 64 */
  int32_t code_bits;  /* code container: 4 (or 0) = int4, two codes per byte; 8 = int8, one code per byte */
} coli_moe_dims;

typedef struct {
  const uint8_t *gate_q, *up_q, *down_q;     /* packed int4 codes, layout above */
  const uint16_t *gate_s, *up_s, *down_s;    /* fp16 scale bits, layout above */
  const float *router_w;                     /* fp32 [E][H]; may be NULL if logits are supplied */
  const float *router_bias;                  /* fp32 [E] or NULL */
} coli_moe_weights;

/*
 * Route: top-k selection and renormalised softmax weights per token
 * (Colibri README, "L'idea": the router picks k experts per token and per
 * layer; the renormalised softmax over the selected logits is the layer
 * statement's reading, the README gives no formula).
 *   logits   fp32 [T][E]   router logits (device)
 *   bias     fp32 [E]      additive per-expert bias, or NULL
 *   topk_ids int32 [T][k]  out: selected experts, slot order = selection order
 *   topk_w   fp32 [T][k]   out: renormalised weights (sum to 1 per token)
 * Ties go to the lowest expert index; -0.0 ties +0.0; a NaN logit ranks as
 * -inf and sets COLI_FLAG_NONFINITE.  T == 0 is a no-op.
 */
coli_status coli_moe_route(const float *logits, const float *bias, int T, int E, int k,
                           int32_t *topk_ids, float *topk_w, void *stream);

/*
 * Union: batch-union of the selected experts, without atomics (Colibri README,
 * "Mai aspettare il disco due volte": a batch reads each expert its tokens
 * selected once, however many of them selected it).
 *   topk_ids  int32 [T][k]        in
 *   unique_ids int32 [min(E,T*k)] out: experts used by the batch, ascending
 *   n_unique  int32 [1]           out: U (stays on the device)
 *   seg_off   int32 [min(E,T*k)+1] out: pairs of unique_ids[u] are
 *                                 perm[seg_off[u] .. seg_off[u+1])
 *   perm      int32 [T*k]         out: pair indices p = t*k + j, sorted by
 *                                 (expert, p)
 *   pair_pos  int32 [T*k]         out: inverse of perm (-1 for a pair whose id
 *                                 was out of range; COLI_FLAG_BAD_ID is set)
 * Entries of unique_ids/seg_off past U are left unchanged.  One CTA; T*k <= 2^24.
 */
coli_status coli_moe_union(const int32_t *topk_ids, int T, int k, int E,
                           int32_t *unique_ids, int32_t *n_unique, int32_t *seg_off,
                           int32_t *perm, int32_t *pair_pos, void *stream);

/*
 * Expert FFN + combine for an already routed and unioned batch (Colibri
 * README, "L'idea": int4 routed experts with group scales; each unique expert
 * runs once over its tokens, SwiGLU, then the routing-weighted sum back into
 * token order).
 *   x         bf16 [T][H]   expert input
 *   topk_ids, topk_w, unique_ids, n_unique, seg_off, perm, pair_pos:
 *             as produced by coli_moe_route / coli_moe_union
 *   residual  bf16 [T][H] or NULL (added once, in fp32, before rounding)
 *   out       bf16 [T][H]   out (must not alias x; may alias residual)
 *   ws        device scratch of at least coli_moe_workspace_bytes(dims, T) bytes,
 *             256-byte aligned, owned by the caller; contents on entry are ignored
 *   flags     COLI_PATH_* selects the FFN form (0 = automatic)
 */
coli_status coli_moe_expert_ffn(const coli_moe_dims *dims, const coli_moe_weights *w,
                                const uint16_t *x, int T,
                                const int32_t *topk_ids, const float *topk_w,
                                const int32_t *unique_ids, const int32_t *n_unique,
                                const int32_t *seg_off, const int32_t *perm,
                                const int32_t *pair_pos, const uint16_t *residual,
                                uint16_t *out, uint32_t flags, void *ws, size_t ws_bytes,
                                void *stream);

/*
 * One whole MoE layer: [pre-norm] -> logits -> Route -> Union -> FFN -> combine
 * (the per-token path of the Colibri README, "L'idea" and "Mai aspettare il
 * disco due volte", with every expert resident: "Una gerarchia di memoria").
 *   x          bf16 [T][H]
 *   logits_in  fp32 [T][E] or NULL: when given, replaces x . W_r^T
 *   residual   bf16 [T][H] or NULL
 *   flags      COLI_LAYER_PRENORM and/or COLI_PATH_*
 *   out        bf16 [T][H]   (must not alias x; may alias residual)
 *   logits_out fp32 [T][E] or NULL: the logits used (before the bias)
 *   topk_ids_out int32 [T][k] or NULL, topk_w_out fp32 [T][k] or NULL
 *   ws / ws_bytes as for coli_moe_expert_ffn
 */
coli_status coli_moe_layer(const coli_moe_dims *dims, const coli_moe_weights *w,
                           const uint16_t *x, int T, const float *logits_in,
                           const uint16_t *residual, uint32_t flags, uint16_t *out,
                           float *logits_out, int32_t *topk_ids_out, float *topk_w_out,
                           void *ws, size_t ws_bytes, void *stream);

/*
 * One expert-parallel rank's share of coli_moe_layer.  The pages' fastest
 * runs spread full expert residence over several GPUs (Colibri README, "Cosa
 * ottiene"); here G ranks each hold a contiguous range of the E experts, the
 * router and the union are replicated, and the ranks' partial outputs are
 * summed by an all-reduce.  The call routes every token over all E experts
 * (router_w, router_bias: the full [E][H] / [E]; or logits_in), builds the
 * union of the whole batch, and computes
 *   out_partial[t] = sum over slots j with expert_begin <= id[t][j] < expert_end
 *                    of w[t][j] * y_id(x_t)
 *                  + (with_shared ? sum_s y_{E+s}(x_t) : 0) + (residual ? residual[t] : 0)
 * in fp32, unrounded.  The sum of the ranks' partials (pass the residual on one
 * rank only), rounded once to bf16 (coli_moe_partial_to_bf16), is the layer's
 * output up to the order of that fp32 sum.
 *   w            expert tensors of this rank only: routed experts
 *                [expert_begin, expert_end) at indices 0.., then, when
 *                with_shared != 0, the S shared experts; same layouts as above
 *   out_partial  fp32 [T][H] (16-byte aligned; must not alias x)
 *   logits_out, topk_ids_out, topk_w_out, ws, ws_bytes, flags: as coli_moe_layer
 * Runs in the prefill form (any batch; the tile plan covers the rank's
 * experts only) and in the decode forms for T <= 128 (the split-K form up to 8
 * tokens, the two-phase form above; with I = 128 not for T <= 4, whose
 * two-phase kernel combines in place); decode batches above 128 tokens return
 * COLI_ERR_UNSUPPORTED; 0 <= expert_begin < expert_end <= E, else
 * COLI_ERR_INVALID_ARG.  Host-memory flags are not accepted here.
 */
coli_status coli_moe_layer_ep(const coli_moe_dims *dims, const coli_moe_weights *w, int expert_begin,
                              int expert_end, int with_shared, const uint16_t *x, int T, const float *logits_in,
                              const uint16_t *residual, uint32_t flags, float *out_partial, float *logits_out,
                              int32_t *topk_ids_out, float *topk_w_out, void *ws, size_t ws_bytes, void *stream);

/* out[i] = bf16(partial[i]) for i < n (n a multiple of 4; partial 16-byte and
 * out 8-byte aligned): the rounding step after the ranks' all-reduce. */
coli_status coli_moe_partial_to_bf16(const float *partial, uint16_t *out, size_t n, void *stream);

/*
 * coli_moe_layer without a caller-provided workspace.  The pages describe no
 * such call; it exists for callers that cannot allocate device memory when
 * they run the layer: code embedded in a host runtime that owns every device
 * allocation (a plugin or custom operator inside another inference engine),
 * real-time loops whose memory is fixed up front, or callers that simply have
 * no allocator at hand.  Instead of `ws`, it uses a scratch array of
 * COLI_NOALLOC_SCRATCH_BYTES bytes that the library itself places in device
 * memory as a file-scope variable: every GPU that loads the library holds
 * that much memory until the process exits.
 *   - Arguments and results are those of coli_moe_layer, without ws/ws_bytes.
 *   - Batches whose coli_moe_workspace_bytes(dims, T) exceeds
 *     COLI_NOALLOC_SCRATCH_BYTES are rejected with COLI_ERR_WORKSPACE before
 *     anything is launched (up to 82 tokens for H=6144, I=2048, E=256, k=8, S=1).
 *   - The first call on a device looks up the array's device address (one
 *     cudaGetSymbolAddress with that device current); make that first call
 *     before capturing a stream.  No call allocates or frees device memory.
 *   - Every call on a device uses the same array, which keeps whatever the
 *     last call left in it (the layer needs nothing in it to start at zero).
 *     Calls that can overlap on the GPU (different streams without ordering
 *     between them) race on the array and give undefined results: order them.
 */
#define COLI_NOALLOC_SCRATCH_BYTES (32u << 20)
coli_status coli_moe_layer_noalloc(const coli_moe_dims *dims, const coli_moe_weights *w,
                                   const uint16_t *x, int T, const float *logits_in,
                                   const uint16_t *residual, uint32_t flags, uint16_t *out,
                                   float *logits_out, int32_t *topk_ids_out, float *topk_w_out,
                                   void *stream);

/* Workspace bytes that serve every coli_moe_layer / coli_moe_expert_ffn call of
 * up to T_max tokens (0 for unsupported dims).  Not monotone in the form's own
 * needs: the split-K decode form's partial sums at 8 tokens can take more than
 * the two-phase form needs for larger batches, and the size returned for any
 * T_max > 8 covers them.  Host only. */
size_t coli_moe_workspace_bytes(const coli_moe_dims *dims, int T_max);

/* Where coli_moe_layer leaves the batch-union it computed (for tests and
 * diagnostics; the pages have no counterpart): byte offsets, within the `ws`
 * of a coli_moe_layer call with these dims and T, of the union step's outputs
 * as coli_moe_union defines them,
 *   off[0] unique_ids  int32 [min(E, T*k)]    off[3] perm      int32 [T*k]
 *   off[1] n_unique    int32 [1]              off[4] pair_pos  int32 [T*k]
 *   off[2] seg_off     int32 [min(E, T*k) + 1]
 * They hold that call's union once it has run, until the next call that uses
 * the same workspace.  off: host array of 5.  Host only; returns the status
 * of the dims and T checks (COLI_ERR_INVALID_ARG for T < 0 or off == NULL). */
coli_status coli_moe_union_offsets(const coli_moe_dims *dims, int T, size_t *off);

/* FFN form taken by coli_moe_layer and coli_moe_expert_ffn for these dims, T
 * and flags (the rule under COLI_PATH_* above).  Host only: launches nothing
 * and needs no device.
 *   form  host pointer; out: one of the COLI_FORM_* values below, or 0 when
 *         T == 0 (the calls are then no-ops whatever the flags)
 * Returns the status the calls give for the same dims, T and flags before they
 * look at pointers or the workspace: COLI_ERR_UNSUPPORTED for dims or batches
 * outside the supported set, COLI_ERR_INVALID_ARG for T < 0, both COLI_PATH_*
 * flags, dims == NULL or form == NULL. */
#define COLI_FORM_DECODE_SPLITK   1  /* decode form, T <= 8 and I % 256 == 0: gate/up and down in one pass */
#define COLI_FORM_DECODE_TWOPHASE 2  /* decode form, other batches: gate/up tiles, then down tiles, then combine */
#define COLI_FORM_PREFILL         3  /* prefill form: tcgen05 grouped GEMM */
coli_status coli_moe_ffn_form(const coli_moe_dims *dims, int T, uint32_t flags, int *form);

/* Synchronises `stream`, then reads and clears the calling device's status
 * word.  *flags (host pointer, may be NULL) receives the COLI_FLAG_* bits.
 * Returns COLI_OK when no bit was set, COLI_ERR_NONFINITE when only the
 * NONFINITE bit was set, COLI_ERR_DEVICE for any other bit, COLI_ERR_CUDA if
 * the synchronisation failed.  Not capturable. */
coli_status coli_moe_get_status(void *stream, uint32_t *flags);

/* Test hook of the device-side bounded waits; the pages have no counterpart.
 * Enqueues one tiny kernel whose single thread waits, with a limit of
 * limit_ns nanoseconds of %globaltimer, first on a shared-memory barrier
 * that nothing arrives on and then on a device counter that nothing
 * increments -- the same wait routines every pipeline wait of the FFN kernels
 * uses (there with a limit of 2 s).  Both waits give up, set
 * COLI_FLAG_TIMEOUT in the status word and the kernel returns: the device
 * stays usable.
 *   limit_ns    0 < limit_ns <= 2e9, else COLI_ERR_INVALID_ARG
 *   elapsed_ns  device pointer to 2 uint64 (8-byte aligned) receiving how
 *               long each wait lasted before giving up, or NULL
 * Read the result with coli_moe_get_status (COLI_ERR_DEVICE, flags
 * COLI_FLAG_TIMEOUT). */
coli_status coli_moe_test_wait_timeout(uint64_t limit_ns, uint64_t *elapsed_ns, void *stream);

/*
 * Host-RAM expert tier: Place, Overlap and Learn (Colibri README, "Una
 * gerarchia di memoria, non un requisito di memoria" and "Mai aspettare il
 * disco due volte"; getting-started guide, "トークンごとの処理経路", steps 3-5).
 * Every routed expert lives in page-locked host memory; the device holds C of
 * them at a time in slots.  A tiered layer call routes and unites the batch as
 * coli_moe_layer does, then places the union on the device: experts already in
 * a slot are hits; each miss takes the slot, not used by this batch, that
 * holds the expert routed least often so far (empty slots first, then the
 * least recently used, then the lowest index), and its three matrices are
 * copied from host memory into that slot by the library's kernels.  The FFN
 * then runs on the slots; placement changes neither the routing nor the
 * arithmetic, so the output equals coli_moe_layer's bit for bit.  Learn: the
 * tier counts the routed pairs of every expert over all calls, and the
 * eviction order keeps the most used experts resident.  Overlap: a caller
 * that predicts the next layer's experts (for example with that layer's
 * router on the current input) places them with coli_moe_tier_prefetch on
 * another stream while the current layer computes.
 *
 * coli_moe_tier (per layer):
 *   gate_q .. down_s  every routed expert's codes and scales, laid out as in
 *                     coli_moe_weights (E experts, no shared ones), in
 *                     page-locked host memory mapped into the device's address
 *                     space (cudaHostAlloc, cudaHostRegister with
 *                     cudaHostRegisterMapped); the library reads it only
 *   n_slots           C, routed experts held on the device, 1 <= C <= E
 *   state             device memory of coli_moe_tier_state_bytes(dims, C)
 *                     bytes, 256-byte aligned, owned by the caller, set up by
 *                     coli_moe_tier_reset before first use; its layout (int32
 *                     unless noted): slot_of[E] (slot of expert e, or -1),
 *                     owner[C] (expert in slot c, or -1), usage[E] (uint32,
 *                     routed pairs per expert), last[C] (uint32, the call count
 *                     at the slot's last use), calls, hits, misses, fills
 *                     (uint32 counters), then scratch
 * The weights passed with a tier (`slots`) are device arrays of C routed
 * experts followed by the S shared ones, with the router weight and bias as in
 * coli_moe_weights; their contents follow the tier (reset leaves them unused).
 */
typedef struct {
  const uint8_t *gate_q, *up_q, *down_q;
  const uint16_t *gate_s, *up_s, *down_s;
  int32_t n_slots;
  void *state;
} coli_moe_tier;

/* Device bytes of a tier's state; 0 for invalid arguments. */
size_t coli_moe_tier_state_bytes(const coli_moe_dims *dims, int32_t n_slots);

/* Empties every slot and clears the counters (enqueued on `stream`). */
coli_status coli_moe_tier_reset(const coli_moe_dims *dims, const coli_moe_tier *tier, void *stream);

/* coli_moe_layer through a tier: arguments as coli_moe_layer's, with `slots`
 * in place of the weights.  Decode form only (COLI_PATH_PREFILL, or an
 * automatic choice of the prefill form, returns COLI_ERR_UNSUPPORTED), and a
 * batch must fit the slots: min(E, T*k) <= C, else COLI_ERR_UNSUPPORTED.
 * Workspace: coli_moe_workspace_bytes(dims, T). */
coli_status coli_moe_layer_tiered(const coli_moe_dims *dims, const coli_moe_weights *slots,
                                  const coli_moe_tier *tier, const uint16_t *x, int T, const float *logits_in,
                                  const uint16_t *residual, uint32_t flags, uint16_t *out, float *logits_out,
                                  int32_t *topk_ids_out, float *topk_w_out, void *ws, size_t ws_bytes,
                                  void *stream);

/* Places experts ids[0..n) (device int32, any order, repeats allowed, n <= C)
 * as a tiered call would, without counting them as routed: the copies of the
 * misses are enqueued on `stream`.  Calls on one tier must be ordered (one
 * stream, or events); tiers of different layers are independent. */
coli_status coli_moe_tier_prefetch(const coli_moe_dims *dims, const coli_moe_weights *slots,
                                   const coli_moe_tier *tier, const int32_t *ids, int32_t n, void *stream);

/* Overlap, lookahead form (the pages' router lookahead: routing one layer
 * ahead is largely predictable): routes x with the NEXT layer's router
 * (`next`: that layer's slot arrays with its router weight and bias) and
 * places the experts it selects in that layer's tier, as coli_moe_tier_prefetch
 * would (nothing counted as routed).  Meant to run on another stream while the
 * current layer computes.  x: bf16 [T][H] device rows (COLI_LAYER_PRENORM
 * applies the next layer's pre-norm); min(E, T*k) <= C, else
 * COLI_ERR_UNSUPPORTED; ws: a workspace of coli_moe_workspace_bytes(dims, T)
 * bytes that no concurrent call uses (its routing arrays are overwritten). */
coli_status coli_moe_tier_lookahead(const coli_moe_dims *dims, const coli_moe_weights *next,
                                    const coli_moe_tier *next_tier, const uint16_t *x, int T, uint32_t flags,
                                    void *ws, size_t ws_bytes, void *stream);

/* Static description of a status code. */
const char *coli_status_str(coli_status s);

/* Library version: major*10000 + minor*100 + patch. */
int coli_moe_version(void);

/* Number of kernel launches made by the calling host thread since the last
 * reset (reset != 0 clears it).  Counting only; no device work. */
uint64_t coli_moe_launch_count(int reset);

/* Timing hook (diagnostics, host only).  While set, the next coli_moe_layer or
 * coli_moe_expert_ffn call made by this host thread records events[i]
 * (cudaEvent_t handles owned by the caller, created on the call's device) on
 * its stream at internal stage boundary i, for i < n:
 *   0 start, 1 after pre-norm/fragment copy, 2 after logits, 3 after route,
 *   4 after union, 5 after tile plan, 6 after gate/up FFN, 7 after down FFN,
 *   8 after combine.
 * Stages a call does not run record at the same point as the previous one.
 * The setting is consumed by that one call; n = 0 or events = NULL clears it. */
coli_status coli_moe_set_stage_events(void *const *events, int n);

#ifdef __cplusplus
}
#endif
#endif /* COLI_MOE_H */
