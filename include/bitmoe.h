/*
 * bitmoe.h -- C ABI of libbitmoe.so, the sm_100a (B200) hot path of MoE
 * routed-expert inference with ternary weights kept compressed in HBM.
 *
 * What the library computes (each entry point cites the passage it follows):
 *   routed-expert weights are ternary (Parallax 8B kappa article, section
 *   "Что именно доступно"), stay compressed in GPU memory and are never
 *   expanded to fp16; decode runs fused mat-vecs that read the quantized
 *   blocks directly and accumulate against int8-quantized activations; large
 *   batches run a GEMM path (Parakon Runtime README, section "How it works").
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers unless the name ends in _host.  The
 *     caller allocates and owns every buffer; the library allocates nothing,
 *     frees nothing, and keeps no state between calls other than a
 *     thread-local last-error string (moe_last_error).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream) and never synchronize, except moe_check_status.
 *   - Arguments are validated on the host before any launch: a bad argument
 *     returns a negative moe_status and launches nothing.  Problems only the
 *     device can see (an expert id out of range) are recorded in the status
 *     word at the start of the workspace and reported by moe_check_status;
 *     the kernels never trap or abort.
 *   - Device pointers must be 16-byte aligned.  Inputs are assumed finite.
 *   - The current CUDA device must be a B200 (sm_100); the library is built
 *     for sm_100a only and has no other code path.
 *
 * Storage format of a ternary matrix W [rows][k] (rows % 32 == 0,
 * k % 256 == 0).  The pages fix no byte layout; this one is chosen for the
 * decode kernels:
 *   - blocks of 256 consecutive weights of a row; scale s = fp16(absmean),
 *     weight q = sign(w) if |w| >= s/2 else 0 (see moe_quantize_weights);
 *   - 13 little-endian uint32 words per block: byte lane l (0..3) of word j
 *     (0..12) holds the five base-3 digits t = q + 1 of weights
 *     k = 20j + 4i + l, i = 0..4, as u = ceil(v * 256 / 243) with
 *     v = sum_i t_i 3^(4-i); the last word's fifth digit is a pad (t = 1);
 *   - rows are grouped in panels of 32 whose words interleave row by row:
 *     word j of block b of row r is trits[((r/32 * nb + b) * 13 + j) * 32 + r%32]
 *     with nb = k/256; the fp16 scale of block b of row r is
 *     scales[(r/32 * nb + b) * 32 + r%32].
 * That is 52 bytes of digits plus a 2-byte scale per 256 weights (1.6875
 * bits per weight).
 *
 * Storage format of a 1-bit sign-code matrix (MOE_FORMAT_SIGN; the 1-bit
 * tier of the pxq_llama README, "What's PXQ?": sign codes times scales).
 * The same blocks, fp16 absmean scales and 32-row panels; q = -1 where
 * w < 0, else +1; 8 uint32 words per block, word j holding weights
 * 32j .. 32j+31 of the block, weight 32j + 4i + l in bit 8l + i (i = 0..7,
 * l = 0..3), a set bit meaning +1; word j of block b of row r is
 * codes[((r/32 * nb + b) * 8 + j) * 32 + r%32].  34 bytes per 256 weights
 * (1.0625 bits per weight).
 *
 * Two-level scales (MOE_FORMAT_E16; pxq_llama README, "What's PXQ?": a
 * per-row fp16 anchor plus a 4-bit sub-scale per 16-element block): the
 * ternary digits above, with per row an fp16 anchor A (in `scales`, one per
 * row) and per 16-weight block h a 4-bit code c_h (in `codes`: word u of
 * block b of row r is codes[((r/32 * nb + b) * 2 + u) * 32 + r%32], block
 * 8u + v in bits 4v..4v+3), the block's scale being A * (c_h + 1) / 16.
 * Quantization (moe_quantize_weights_e16): A = fp16(max over the row's
 * 16-blocks of mean|w|), c_h = clamp(rint(16 * mean_h / A) - 1, 0, 15),
 * q = sign(w) where |w| >= s_h / 2, else 0.  60 bytes per 256 weights plus
 * 2 bytes per row.
 */
#ifndef BITMOE_H
#define BITMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* moe_stream_t; /* a cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,       /* null pointer, non-positive size, k > E ... */
  MOE_ERR_UNSUPPORTED_SHAPE = -2, /* outside the documented shape limits        */
  MOE_ERR_ALIGNMENT = -3,         /* a device pointer not 16-byte aligned       */
  MOE_ERR_WORKSPACE = -4,         /* workspace smaller than moe_workspace_bytes */
  MOE_ERR_CUDA = -5,              /* a CUDA runtime error (see moe_last_error)  */
  MOE_ERR_TIMEOUT = -6,           /* a bounded device-side wait ran out         */
  MOE_ERR_BAD_INDEX = -7,         /* an expert id outside [0, n_experts)        */
  MOE_ERR_DEVICE = -8,            /* the current device is not sm_100           */
  MOE_ERR_BOUNDS = -9             /* bounds-checked build only (MOE_CHECKED): a
                                     kernel computed an index outside its buffer
                                     and skipped the access                     */
} moe_status;

/* Weight formats. */
typedef enum { MOE_FORMAT_TERNARY = 0, MOE_FORMAT_SIGN = 1, MOE_FORMAT_E16 = 2 } moe_format;

/* One packed matrix in one of the storage formats above. */
typedef struct {
  int32_t rows;          /* multiple of 32                          */
  int32_t k;             /* multiple of 256                         */
  const uint32_t* trits; /* the packed words, device: moe_trit_words(rows, k)
                            base-3 words, or moe_sign_words(rows, k) sign
                            words for MOE_FORMAT_SIGN                */
  const uint16_t* scales;/* moe_scale_count(rows, k) fp16, device, or
                            one fp16 anchor per row for MOE_FORMAT_E16 */
  int32_t format;        /* a moe_format                             */
  const uint32_t* codes; /* MOE_FORMAT_E16: moe_e16_code_words(rows, k)
                            sub-scale words, device; else unused      */
} moe_tmat;

/* One MoE layer.  Expert e owns rows [e*ffn, (e+1)*ffn) of gate and up
 * (k = hidden) and rows [e*hidden, (e+1)*hidden) of down (k = ffn).  The
 * three matrices share one format.  Limits: hidden and ffn multiples of 256,
 * hidden <= 16384, ffn <= 8192, 1 <= top_k <= min(n_experts, 32),
 * n_experts <= 1024.  All three formats run the decode path (up to 64
 * tokens) and the prefill GEMM (moe_expert_ffn_prefill, moe_forward of more
 * than 64 tokens); the one-token fused step takes all three formats where
 * its shared-memory plan fits one CTA (hidden <= 4096 and at most one
 * 32-row panel of hidden per SM, ffn <= 2048, top_k <= 8, n_experts <= 256
 * and at most two per SM); other one-token shapes take the decode chains. */
typedef struct {
  int32_t hidden, ffn, n_experts, top_k;
  moe_tmat gate, up, down;
} moe_layer;

/* ---- sizes ------------------------------------------------------------ */
size_t moe_trit_words(int64_t rows, int64_t k);  /* rows*(k/256)*13 */
size_t moe_sign_words(int64_t rows, int64_t k);  /* rows*(k/256)*8  */
size_t moe_e16_code_words(int64_t rows, int64_t k); /* rows*(k/256)*2 */
size_t moe_scale_count(int64_t rows, int64_t k); /* rows*(k/256)    */
/* Bytes of workspace a decode (prefill = 0) or prefill (prefill = 1) call
 * of `ntok` tokens, or moe_forward, needs.  0 on invalid arguments.        */
size_t moe_workspace_bytes(const moe_layer* layer, int32_t ntok, int32_t prefill);
/* Where a workspace of this layer (for `ntok` tokens, decode or prefill
 * layout) holds the int8 codes [ntok][hidden] and fp32 scales
 * [ntok][hidden/32] of x (S1, pxq_llama README, "PXQ vs MXFP4": one scale
 * per 32-value block): byte offsets from the workspace's start.  Every
 * moe_forward call writes them there (the same values moe_quant_act_q8
 * gives), so a caller can hand them on, e.g. to moe_shared_ffn_add, without
 * quantizing x again.  MOE_ERR_INVALID_ARG on a bad layer or ntok <= 0.    */
int moe_workspace_act(const moe_layer* layer, int32_t ntok, int32_t prefill, size_t* xq_offset,
                      size_t* xd_offset);
/* Zero a workspace (status word and counters).  Every workspace must be
 * initialised once before its first use; calls leave it reusable.         */
int moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream);

/* ---- S0: weight quantization (offline; Parallax 8B kappa article,
 *      "Что именно доступно": ternary routed-expert weights) ------------
 * w [rows][k] fp32 row-major -> trits, scales in the storage format.  Per
 * 256-block: s = fp16 round-to-nearest-even of (sum |w| in fp64, ascending
 * k) / 256; q = sign(w) where |w| >= 0.5*s (in fp32), else 0.  The output
 * bytes do not depend on the launch configuration.                        */
int moe_quantize_weights(const float* w, int64_t rows, int64_t k, uint32_t* trits,
                         uint16_t* scales, moe_stream_t stream);
/* The same to 1-bit sign codes (MOE_FORMAT_SIGN): the same scales; q = -1
 * where w < 0, else +1 (see the storage format above).                    */
int moe_quantize_weights_sign(const float* w, int64_t rows, int64_t k, uint32_t* codes,
                              uint16_t* scales, moe_stream_t stream);
/* The same to ternary digits with two-level scales (MOE_FORMAT_E16): trits
 * as moe_quantize_weights' (digits of the E16 quantization), codes
 * [moe_e16_code_words(rows, k)], anchors [rows] fp16.                     */
int moe_quantize_weights_e16(const float* w, int64_t rows, int64_t k, uint32_t* trits,
                             uint32_t* codes, uint16_t* anchors, moe_stream_t stream);

/* ---- S1: activation quantization (Parakon Runtime README, "How it works":
 *      int8-quantized activations; pxq_llama README, "PXQ vs MXFP4": one
 *      scale per 32-value block) ------------------------------------------
 * x [ntok][k] fp32 -> xq [ntok][k] int8, xd [ntok][k/32] fp32 with, per 32
 * values, d = amax/127 and q = clamp(rint(x/d), -127, 127) (IEEE division,
 * ties to even; a block whose d is 0 gets q = 0).  k % 32 == 0,
 * k <= 65536, ntok <= 2^24.                                               */
int moe_quant_act_q8(const float* x, int32_t ntok, int32_t k, int8_t* xq, float* xd,
                     moe_stream_t stream);

/* ---- S2: router (llama-modchip page, "Key highlights": every top-k expert
 *      is evaluated, none dropped) ---------------------------------------
 * logits = w_router [E][hidden] . x_t in fp32 in a fixed order (32 partial
 * sums over k = l mod 32 ascending with fused multiply-adds, then pairwise
 * rounds at distances 16, 8, 4, 2, 1); idx [ntok][top_k] = experts by
 * descending logit, ties to the lower id; wts [ntok][top_k] = softmax over
 * the selected logits (the full softmax renormalised over the top-k).
 * ntok <= 65536, hidden % 256 == 0, hidden <= 16384, n_experts <= 1024,
 * top_k <= min(n_experts, 32).                                            */
int moe_route_topk(const float* x, const float* w_router, int32_t ntok, int32_t hidden,
                   int32_t n_experts, int32_t top_k, int32_t* idx, float* wts, void* ws,
                   size_t ws_bytes, moe_stream_t stream);
/* Workspace bytes moe_route_topk needs (it keeps the [ntok][E] logits there). */
size_t moe_route_workspace_bytes(int32_t ntok, int32_t n_experts);

/* ---- S3-S5: expert FFN, decode (Parakon Runtime README, "How it works":
 *      fused mat-vecs over the compressed blocks against int8 activations;
 *      pxq_llama README, "Updates -- 2026-07-28": gate/up with the SiLU
 *      unary) --------------------------------------------------------------
 * For each token t and slot j (e = idx[t][j]):
 *   g = Wg_e . x^_t, u = Wu_e . x^_t; a = g / (1 + exp(-g)) * u (fp32);
 *   (aq, ad) = q8(a) in 32-blocks; y_t = sum_j wts[t][j] * (Wd_e . a^)
 * summed over the slots in order.  y [ntok][hidden] fp32 is overwritten.
 * 1 <= ntok <= 64.  An id outside [0, E) sets MOE_ERR_BAD_INDEX in the
 * workspace status and its slot contributes nothing.                      */
int moe_expert_ffn_decode(const moe_layer* layer, int32_t ntok, const int8_t* xq,
                          const float* xd, const int32_t* idx, const float* wts, float* y,
                          void* ws, size_t ws_bytes, moe_stream_t stream);

/* ---- decode without a caller workspace ---------------------------------------
 * No counterpart on the pages this library follows: an addition for callers
 * that cannot allocate device memory at call time (a plug-in whose host
 * application owns every device allocation, a serving loop that must never
 * enter the CUDA allocator, code held to a device-memory budget fixed at
 * start-up).  Same computation and arguments as moe_expert_ffn_decode, minus
 * the workspace: the scratch is a 4 MiB array inside this library, reserved
 * on every GPU that loads the library and held until the process exits.
 *   - A call that needs more scratch than that
 *     (moe_workspace_bytes(layer, ntok, 0) > 4 MiB) returns
 *     MOE_ERR_WORKSPACE and launches nothing.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - Every call clears and reuses the same array, so two calls whose work
 *     can overlap on the GPU (other streams, other host threads) race; keep
 *     them ordered on one stream.
 *   - Arguments are checked before the array is touched: a refused call
 *     (NULL or misaligned pointer, bad sizes) clears nothing.
 *   - No device-side status can be observed through this entry point: each
 *     call clears the array's status word, and there is no workspace to pass
 *     to moe_check_status.  Expert ids outside [0, E) contribute nothing and
 *     are not reported.
 *   - It allocates and frees nothing.                                      */
int moe_expert_ffn_decode_static(const moe_layer* layer, int32_t ntok, const int8_t* xq,
                                 const float* xd, const int32_t* idx, const float* wts, float* y,
                                 moe_stream_t stream);

/* ---- S7: expert FFN, prefill (Parakon Runtime README, "How it works":
 *      large batches take a GEMM path over the quantized tiles) -----------
 * Same result as moe_expert_ffn_decode for any ntok >= 1 (up to rounding
 * order), computed by grouping the (token, slot) pairs by expert and running
 * an int8 tensor-core grouped GEMM (exact int32 block sums; ternary, sign
 * codes and two-level scales).  ntok <= 65536.                             */
int moe_expert_ffn_prefill(const moe_layer* layer, int32_t ntok, const int8_t* xq,
                           const float* xd, const int32_t* idx, const float* wts, float* y,
                           void* ws, size_t ws_bytes, moe_stream_t stream);

/* ---- the whole step ------------------------------------------------------
 * S1 + S2 + (S3-S5 or S7): y [ntok][hidden] = MoE(x [ntok][hidden]).  Uses
 * the decode path for ntok <= 64 and the prefill path above: one token runs
 * as one cooperative kernel (the one-token step) where the layer's shape
 * allows, 2..64 tokens as three kernels (routing with the activation
 * quantization and the grouping in one launch, then the grouped gate/up and
 * down mat-vecs).  x and y are device pointers; the quantized x, the routing
 * and the intermediates live in the workspace.                             */
int moe_forward(const moe_layer* layer, const float* w_router, int32_t ntok, const float* x,
                float* y, void* ws, size_t ws_bytes, moe_stream_t stream);
/* The same with x and y in HOST memory (pinned for asynchronous copies):
 * copies x in, runs moe_forward, copies y out, all on `stream`.  Up to 64 KB
 * of page-locked x is moved in by a small kernel that addresses it over the
 * bus, and the step's kernels store y straight into page-locked y of that
 * size; larger or pageable buffers go by DMA copies.  The host buffers must
 * stay valid until the stream reaches the end of the call.                */
int moe_forward_host(const moe_layer* layer, const float* w_router, int32_t ntok,
                     const float* x_host, float* y_host, void* ws, size_t ws_bytes,
                     moe_stream_t stream);

/* ---- shared expert (llama-modchip page, "The interesting bit": shared
 *      experts stay at higher precision beside the low-bit routed experts) --
 * An always-active FFN in 8-bit blocks of 32 weights: per block
 * d = fp16_RNE(amax/127) (the division in fp64), q = clamp(rint(w/d), -127,
 * 127) with an IEEE fp32 division by the fp16 value (a block whose d is 0 is
 * all zeros); codes row-major int8 [rows][k], scales fp16 [rows][k/32].    */
typedef struct {
  int32_t hidden, ffn;       /* multiples of 256 and of 32                 */
  const int8_t* gate_q;  const uint16_t* gate_d;   /* [ffn][hidden]       */
  const int8_t* up_q;    const uint16_t* up_d;     /* [ffn][hidden]       */
  const int8_t* down_q;  const uint16_t* down_d;   /* [hidden][ffn]       */
} moe_shared;
/* w [rows][k] fp32 -> q, d in the 8-bit block format (k % 32 == 0).        */
int moe_quantize_weights_q8(const float* w, int64_t rows, int64_t k, int8_t* q, uint16_t* d,
                            moe_stream_t stream);
/* Workspace bytes of moe_shared_ffn_add for `ntok` tokens (0 on bad args). */
size_t moe_shared_workspace_bytes(const moe_shared* shared, int32_t ntok);
/* y [ntok][hidden] += Wd (q8(silu(Wg x^) * Wu x^))^ for the int8 activations
 * xq [ntok][hidden], xd [ntok][hidden/32] (moe_quant_act_q8's output): the
 * shared expert's output added to the routed experts' sum (call it after
 * moe_expert_ffn_decode / moe_forward on the same stream).  ws is a separate
 * scratch of moe_shared_workspace_bytes bytes.                             */
int moe_shared_ffn_add(const moe_shared* shared, int32_t ntok, const int8_t* xq, const float* xd,
                       float* y, void* ws, size_t ws_bytes, moe_stream_t stream);
/* y [ntok][hidden] = the routed experts' sum (moe_forward) plus the shared
 * expert's FFN, bit for bit what moe_forward followed by moe_shared_ffn_add
 * on the int8 x that moe_forward leaves in ws (moe_workspace_act) gives.
 * One token of a layer whose one-token step applies (moe_forward launches
 * k_step1) with a shared ffn of at most 64 blocks of 32 rows runs as that one
 * launch: the shared expert's 32-row gate/up blocks are units after the
 * routed ones (their weights prefetched into L2 at the start), published with
 * the step's tagged words, and each CTA with a 32-row panel of hidden adds
 * the panel's rows of the shared down projection to y after the routed
 * combine.  Any other call runs moe_forward, then moe_shared_ffn_add's
 * kernels.  ws: moe_workspace_bytes(layer, ntok) bytes; shared_ws:
 * moe_shared_workspace_bytes(shared, ntok) bytes; shared->hidden must equal
 * layer->hidden (MOE_ERR_INVALID_ARG otherwise).  Errors as moe_forward and
 * moe_shared_ffn_add.  (llama-modchip page, "The interesting bit": the
 * shared expert beside the routed ones.)                                   */
int moe_forward_shared(const moe_layer* layer, const moe_shared* shared, const float* w_router,
                       int32_t ntok, const float* x, float* y, void* ws, size_t ws_bytes,
                       void* shared_ws, size_t shared_ws_bytes, moe_stream_t stream);

/* ---- status ------------------------------------------------------------- */
/* Synchronizes `stream`, returns the status recorded in the workspace by
 * the device (MOE_OK or a negative moe_status) and clears it.             */
int moe_check_status(void* ws, moe_stream_t stream);
/* Message of the last failing call on this thread ("" if none). */
const char* moe_last_error(void);

/* ---- tracing --------------------------------------------------------------
 * Kernel ids reported by the tracing calls below. */
typedef enum {
  MOE_K_QUANTIZE_WEIGHTS = 0, MOE_K_QUANT_ACT = 1, MOE_K_ROUTER_LOGITS = 2, MOE_K_TOPK = 3,
  MOE_K_GROUP = 4, MOE_K_GATEUP = 5, MOE_K_DOWN = 6, MOE_K_DEBUG_MATVEC = 7,
  MOE_K_PREFILL_GATEUP = 8, MOE_K_PREFILL_DOWN = 9, MOE_K_ROUTE = 10, MOE_K_COMBINE = 11,
  MOE_K_STEP1 = 12, MOE_K_PREFILL_GATHER = 13, MOE_K_COPY = 14, MOE_K_ROUTER_QUANT = 15,
  MOE_K_TOPK_GROUP = 16, MOE_K_SHARED = 17, MOE_K_TC_GATEUP = 18, MOE_K_TC_DOWN = 19,
  MOE_K_ROUTE_GROUP = 20, MOE_K_COUNT = 21
} moe_kernel_id;
/* Number of kernels this thread has launched through the library so far. */
int64_t moe_launch_count(void);
/* Start tracing on this thread: after each kernel it launches, the library
 * records events[n] (caller-created cudaEvent_t handles, timing enabled) on
 * the kernel's stream and notes the kernel id, until `capacity` events are
 * used.  moe_trace_end stops tracing, copies the ids of the recorded events
 * into kernel_ids and returns how many were recorded.                     */
int moe_trace_begin(void* const* events, int32_t capacity);
int moe_trace_end(int32_t* kernel_ids, int32_t capacity);
/* Name of a kernel id ("" if out of range). */
const char* moe_kernel_name(int32_t id);

/* ---- test hook ------------------------------------------------------------
 * The decode kernels' mat-vec on one matrix: for tokens t < ntok and rows r
 * of m, out[t][r] = sum_b s[r][b] * sum_{j in b} xd[t][j] * isum[t][r][j]
 * (fp32), and, if isum != NULL, the exact int32 block sums
 * isum[t][r][j] = sum_{k in block j} q[r][k] * xq[t][k].  ntok <= 64.    */
int moe_debug_matvec(const moe_tmat* m, int32_t ntok, const int8_t* xq, const float* xd,
                     float* out, int32_t* isum, moe_stream_t stream);

/* The exact int32 block sums of the tensor-core paths (pxq_llama README,
 * "PXQ vs MXFP4": one fixup per 32-value activation block; Parakon Runtime
 * README, "How it works": int8 x quantized-block products).  Runs the expert
 * FFN of moe_expert_ffn_decode (prefill == 0: the grouped tensor-core
 * mat-vecs, any ntok <= 64, ternary layers with hidden and ffn <= 4096) or of
 * moe_expert_ffn_prefill (prefill != 0: the grouped tensor-core GEMM, any of
 * the three formats) with the same arguments, and also writes, for every
 * (token, slot) pair p = t * top_k + j, row and 32-value block s, the exact
 * sum(q * a) (two-level scales: sum over the block's two 16-weight halves h
 * of (c_h + 1) * sum_{k in h} q * a):
 *   isum_gu [p][2][ffn][hidden/32]   gate (index 0) and up (index 1) rows
 *                                    against the pair's token's codes xq;
 *   isum_dn [p][hidden][ffn/32]      down rows against the pair's int8
 *                                    SwiGLU codes;
 *   aq      [p][ffn] (may be NULL)   those SwiGLU codes.
 * Device arrays, 16-byte aligned; entries of pairs whose expert id is out of
 * range are not written.  A layer the path does not take:
 * MOE_ERR_UNSUPPORTED_SHAPE.                                                */
/* Test knob of the bounded device waits (no page has a counterpart: every
 * device wait of this library is bounded, and this lets a test make one run
 * out on purpose and read the reported status).  Writes `mode` and `polls` into the
 * workspace header (synchronizing `stream`); calls on that workspace then:
 *   mode 0: run normally (a fresh workspace holds 0);
 *   mode 1: the one-token step polls its router logits for a tag that no CTA
 *           publishes, gives up after `polls` rounds, records MOE_ERR_TIMEOUT
 *           and leaves before any weight copy is issued;
 *   mode 2: the gather warp of the tensor-core mat-vecs withholds its first
 *           arrival, so the MMA and fixup waits run out after `polls` checks
 *           (each a suspended wait of at most ~20 us), record
 *           MOE_ERR_TIMEOUT, drain the copies in flight and free tensor memory.
 * polls == 0 keeps the kernels' default budgets.  Outputs of a call that
 * timed out are undefined; the context stays usable.                       */
int moe_debug_wait_knob(void* ws, size_t ws_bytes, int32_t mode, int32_t polls, moe_stream_t stream);

int moe_debug_ffn_blocksums(const moe_layer* layer, int32_t ntok, const int8_t* xq, const float* xd,
                            const int32_t* idx, const float* wts, float* y, void* ws, size_t ws_bytes,
                            int32_t prefill, int32_t* isum_gu, int32_t* isum_dn, int8_t* aq,
                            moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* BITMOE_H */
