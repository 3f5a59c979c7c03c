// api.cu -- the extern "C" entry points of libbitmoe: argument validation,
// workspace layout, and the launch sequence of each call.
#include <atomic>
#include <cstring>

#include <algorithm>

#include "bitmoe.h"
#include "common.cuh"
#include "decode.cuh"
#include "decode2.cuh"
#include "prefill.cuh"
#include "tcmv.cuh"
#include "shared.cuh"
#include "quant.cuh"
#include "router.cuh"

namespace bitmoe {

static thread_local char g_last_error[512] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
}

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

static thread_local int64_t g_launches = 0;
static thread_local cudaEvent_t* g_trace_events = nullptr;
static thread_local int g_trace_cap = 0;
static thread_local int g_trace_n = 0;
static thread_local int g_trace_ids[4096];

void note_launch(int kernel_id, cudaStream_t stream) {
  ++g_launches;
  if (g_trace_events && g_trace_n < g_trace_cap && g_trace_n < 4096) {
    cudaEventRecord(g_trace_events[g_trace_n], stream);
    g_trace_ids[g_trace_n++] = kernel_id;
  }
}

int check_launch(const char* what) {
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(err));
  return MOE_OK;
}

int check_device() {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(err));
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return fail(MOE_ERR_DEVICE, "device %d is sm_%d%d; libbitmoe runs on sm_100 (B200) only", dev,
                major, minor);
  return MOE_OK;
}

// ---------------------------------------------------------------- workspace
struct WsLayout {
  size_t logits = 0, xq = 0, xd = 0, idx = 0, wts = 0, aq = 0, ad = 0, ye = 0, cnt = 0;
  size_t units = 0;       // tagged gate/up unit outputs of the one-token step
  size_t sunits = 0;      // the same for a shared expert's blocks
  size_t xs = 0, ys = 0;  // device copies of x and y for the host-buffer entry point
  size_t bgu = 0, bdn = 0;  // prefill only
  GroupWs grp;
  size_t total = 0;
};

static WsLayout ws_layout(int H, int F, int E, int K, int T, bool prefill) {
  WsLayout L;
  size_t off = kWsHeaderBytes;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  // fp32 [T][E], or for the one-token step E tagged logits one 128-byte line apart
  L.logits = take(std::max(sizeof(float) * T * static_cast<size_t>(E), static_cast<size_t>(128) * E));
  L.xq = take(static_cast<size_t>(T) * H);
  L.xd = take(sizeof(float) * T * static_cast<size_t>(H / kQBlock));
  L.idx = take(sizeof(int32_t) * T * static_cast<size_t>(K));
  L.wts = take(sizeof(float) * T * static_cast<size_t>(K));
  L.aq = take(static_cast<size_t>(T) * K * F);
  L.ad = take(sizeof(float) * T * static_cast<size_t>(K) * (F / kQBlock));
  L.ye = take(sizeof(float) * T * static_cast<size_t>(K) * H);
  L.cnt = take(sizeof(int32_t) * T * static_cast<size_t>(H / kPanel));
  L.units = take(sizeof(unsigned long long) * K * static_cast<size_t>(F / kPanel) * (kPanel / 4 + 2));
  L.sunits = take(sizeof(unsigned long long) * kMaxSharedUnits * (kPanel / 4 + 2));  // a shared expert's blocks
  L.xs = take(sizeof(float) * T * static_cast<size_t>(H));
  L.ys = take(sizeof(float) * T * static_cast<size_t>(H));
  off = group_ws_layout(E, T * K, off, &L.grp);
  if (prefill) {
    // groups of at most G pairs: at most T*K/G full ones plus one partial per expert
    const size_t groups = static_cast<size_t>(T) * K / prefill_group_pairs() + E + 1;
    L.bgu = take(groups * (H / kBlock) * prefill_block_bytes());
    L.bdn = take(groups * (F / kBlock) * prefill_block_bytes());
  }
  L.total = off;
  return L;
}

static int check_layer(const moe_layer* L) {
  if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
  const int H = L->hidden, F = L->ffn, E = L->n_experts, K = L->top_k;
  if (H <= 0 || F <= 0 || E <= 0 || K <= 0)
    return fail(MOE_ERR_INVALID_ARG, "layer sizes must be positive (hidden %d ffn %d E %d k %d)", H, F,
                E, K);
  if (K > E) return fail(MOE_ERR_INVALID_ARG, "top_k %d > n_experts %d", K, E);
  if (H % kBlock || F % kBlock)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "hidden %d and ffn %d must be multiples of 256", H, F);
  if (H > kMaxHidden || F > kMaxFfn || E > kMaxExperts || K > kMaxTopK)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                "limits: hidden <= %d, ffn <= %d, n_experts <= %d, top_k <= %d", kMaxHidden, kMaxFfn,
                kMaxExperts, kMaxTopK);
  const moe_tmat* m[3] = {&L->gate, &L->up, &L->down};
  const char* names[3] = {"gate", "up", "down"};
  if (L->gate.format != MOE_FORMAT_TERNARY && L->gate.format != MOE_FORMAT_SIGN && L->gate.format != MOE_FORMAT_E16)
    return fail(MOE_ERR_INVALID_ARG, "unknown weight format %d", L->gate.format);
  if (L->up.format != L->gate.format || L->down.format != L->gate.format)
    return fail(MOE_ERR_INVALID_ARG, "gate, up and down must share one weight format");
  for (int i = 0; i < 3; ++i) {
    const int rows = i < 2 ? E * F : E * H, k = i < 2 ? H : F;
    if (m[i]->rows != rows || m[i]->k != k)
      return fail(MOE_ERR_INVALID_ARG, "%s is [%d][%d], expected [%d][%d]", names[i], m[i]->rows,
                  m[i]->k, rows, k);
    if (!m[i]->trits || !m[i]->scales) return fail(MOE_ERR_INVALID_ARG, "%s has a NULL pointer", names[i]);
    if (!aligned16(m[i]->trits) || !aligned16(m[i]->scales))
      return fail(MOE_ERR_ALIGNMENT, "%s pointers must be 16-byte aligned", names[i]);
    if (m[i]->format == MOE_FORMAT_E16) {
      if (!m[i]->codes) return fail(MOE_ERR_INVALID_ARG, "%s has no sub-scale codes", names[i]);
      if (!aligned16(m[i]->codes)) return fail(MOE_ERR_ALIGNMENT, "%s codes must be 16-byte aligned", names[i]);
    }
  }
  return MOE_OK;
}

template <typename... Ps>
static int check_ptrs(const char* what, Ps... ps) {
  const void* arr[] = {static_cast<const void*>(ps)...};
  for (const void* p : arr) {
    if (!p) return fail(MOE_ERR_INVALID_ARG, "%s: NULL pointer argument", what);
    if (!aligned16(p)) return fail(MOE_ERR_ALIGNMENT, "%s: pointers must be 16-byte aligned", what);
  }
  return MOE_OK;
}

static DecodeParams make_params(const moe_layer* L, int ntok, const int8_t* xq, const float* xd,
                                const int32_t* idx, const float* wts, float* y, void* ws,
                                const WsLayout& W) {
  DecodeParams P;
  P.hidden = L->hidden; P.ffn = L->ffn; P.n_experts = L->n_experts; P.top_k = L->top_k;
  P.ntok = ntok;
  P.gate_trits = L->gate.trits; P.gate_scales = L->gate.scales;
  P.up_trits = L->up.trits;     P.up_scales = L->up.scales;
  P.down_trits = L->down.trits; P.down_scales = L->down.scales;
  P.xq = xq; P.xd = xd; P.idx = idx; P.wts = wts; P.y = y;
  unsigned char* base = static_cast<unsigned char*>(ws);
  P.aq = reinterpret_cast<int8_t*>(base + W.aq);
  P.ad = reinterpret_cast<float*>(base + W.ad);
  P.ye = reinterpret_cast<float*>(base + W.ye);
  P.cnt = reinterpret_cast<int32_t*>(base + W.cnt);
  P.status = &reinterpret_cast<WsHeader*>(ws)->status;
  P.direct = ntok == 1;
  P.format = L->gate.format;
  P.gate_codes = L->gate.codes;
  P.up_codes = L->up.codes;
  P.down_codes = L->down.codes;
  P.items = reinterpret_cast<const Item*>(base + W.grp.items);
  P.n_items = reinterpret_cast<const int32_t*>(base + W.grp.n_items);
  P.pairs = reinterpret_cast<const int32_t*>(base + W.grp.pairs);
  P.group_scratch = reinterpret_cast<int32_t*>(base + W.grp.scratch);
  P.group_chunk = kChunk;
  const bool pf = W.bgu != 0;
  P.bgu = pf ? base + W.bgu : nullptr;
  P.bdn = pf ? base + W.bdn : nullptr;
  return P;
}

static int sm_count() {
  constexpr int kMaxDev = 64;
  static std::atomic<int> cache[kMaxDev];  // per device, written once (any thread)
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < kMaxDev) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c) return c;
  }
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (n <= 0) n = 148;
  if (dev >= 0 && dev < kMaxDev) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

static Decode2Params make_d2(const DecodeParams& P, void* ws, const WsLayout& W) {
  Decode2Params D;
  D.P = P;
  unsigned char* base = static_cast<unsigned char*>(ws);
  D.route_cnt = reinterpret_cast<uint32_t*>(&reinterpret_cast<WsHeader*>(ws)->pad[0]);
  D.logits = reinterpret_cast<float*>(base + W.logits);
  D.x = nullptr;
  D.wr = nullptr;
  D.route_warps = 0;
  D.route_tc = 0;
  D.n_sm = sm_count();
  return D;
}

// Decode from quantized activations and routing.  One token: the persistent
// cp.async mat-vec kernels over the slots directly.  More tokens: grouped by
// expert, then the grouped mat-vec kernels that decode each weight once for
// all the tokens of a group.
static int launch_decode(const DecodeParams& P, void* ws, const WsLayout& W, cudaStream_t stream) {
  if (!P.direct) {
    int rc = launch_group(P, stream);
    if (rc) return rc;
    return launch_ffn(P, stream);
  }
  // sign codes and two-level scales: the grouped kernels in direct mode
  // (item i = slot i)
  if (P.format != MOE_FORMAT_TERNARY) return launch_ffn(P, stream);
  Decode2Params D = make_d2(P, ws, W);
  return launch_decode2(D, false, stream);
}

// ---------------------------------------------------------------- small host copies
constexpr size_t kSmallHostCopy = 64 * 1024;

// The device address of page-locked host memory, or null if the GPU cannot
// address it (pageable memory).
static void* host_device_view(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (a.type != cudaMemoryTypeHost || a.devicePointer == nullptr) return nullptr;
  return a.devicePointer;
}

// dst[i] = src[i] for `bytes` (a multiple of 16, both 16-byte aligned).
__global__ void __launch_bounds__(512) k_copy16(int4* __restrict__ dst, const int4* __restrict__ src, size_t n16) {
  pdl_enter();
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    dst[i] = src[i];
}

static int launch_copy16(void* dst, const void* src, size_t bytes, cudaStream_t s) {
  const size_t n16 = bytes / 16;
  const unsigned grid = static_cast<unsigned>((n16 + 511) / 512 < 8 ? (n16 + 511) / 512 : 8);
  launch_k(k_copy16, dim3(grid), dim3(512), 0, s, static_cast<int4*>(dst), static_cast<const int4*>(src), n16);
  note_launch(MOE_K_COPY, s);
  return check_launch("forward_host: copy");
}

// One token of a ternary layer: the routing kernel and the tensor-core
// mat-vecs, or the fused one-token step (chosen by layer size).
#ifndef MOE_ONE_TOKEN_TC_MIN_HIDDEN
#define MOE_ONE_TOKEN_TC_MIN_HIDDEN 1000000
#endif
static bool one_token_on_tensor_cores(const DecodeParams& P) {
  return tc_ffn_supported(P) && P.hidden >= MOE_ONE_TOKEN_TC_MIN_HIDDEN;
}

// The checks of moe_expert_ffn_decode that do not involve a workspace (layer,
// pointers, token count, device), for entry points that bring their own
// scratch and must validate a call before touching it.
int check_decode_call(const char* what, const moe_layer* L, int32_t ntok, const int8_t* xq, const float* xd,
                      const int32_t* idx, const float* wts, float* y) {
  int rc = check_layer(L);
  if (rc) return rc;
  if ((rc = check_ptrs(what, xq, xd, idx, wts, y))) return rc;
  if (ntok <= 0) return fail(MOE_ERR_INVALID_ARG, "%s: ntok must be > 0", what);
  if (ntok > kMaxDecodeTokens)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "%s: decode takes at most %d tokens", what, kMaxDecodeTokens);
  return check_device();
}

}  // namespace bitmoe

using namespace bitmoe;

extern "C" {

size_t moe_e16_code_words(int64_t rows, int64_t k) {
  if (rows <= 0 || k <= 0) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(k / kBlock) * kE16Words;
}

size_t moe_sign_words(int64_t rows, int64_t k) {
  if (rows <= 0 || k <= 0) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(k / kBlock) * kSignWords;
}

size_t moe_trit_words(int64_t rows, int64_t k) {
  if (rows <= 0 || k <= 0) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(k / kBlock) * kBlockWords;
}

size_t moe_scale_count(int64_t rows, int64_t k) {
  if (rows <= 0 || k <= 0) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(k / kBlock);
}

size_t moe_workspace_bytes(const moe_layer* L, int32_t ntok, int32_t prefill) {
  if (check_layer(L) != MOE_OK || ntok <= 0) return 0;
  return ws_layout(L->hidden, L->ffn, L->n_experts, L->top_k, ntok, prefill != 0).total;
}

int moe_workspace_act(const moe_layer* L, int32_t ntok, int32_t prefill, size_t* xq_offset, size_t* xd_offset) {
  int rc = check_layer(L);
  if (rc) return rc;
  if (ntok <= 0 || !xq_offset || !xd_offset) return fail(MOE_ERR_INVALID_ARG, "workspace_act: ntok > 0, offsets");
  const WsLayout W = ws_layout(L->hidden, L->ffn, L->n_experts, L->top_k, ntok, prefill != 0);
  *xq_offset = W.xq;
  *xd_offset = W.xd;
  return MOE_OK;
}

size_t moe_route_workspace_bytes(int32_t ntok, int32_t n_experts) {
  if (ntok <= 0 || n_experts <= 0) return 0;
  return kWsHeaderBytes + align_up(sizeof(float) * static_cast<size_t>(ntok) * n_experts, 256);
}

int moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!ws || ws_bytes < kWsHeaderBytes) return fail(MOE_ERR_INVALID_ARG, "workspace too small or NULL");
  if (!aligned16(ws)) return fail(MOE_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  int rc = check_device();
  if (rc) return rc;
  cudaError_t err = cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(err));
  return MOE_OK;
}

int moe_quantize_weights(const float* w, int64_t rows, int64_t k, uint32_t* trits, uint16_t* scales,
                         moe_stream_t stream) {
  int rc = check_ptrs("quantize_weights", w, trits, scales);
  if (rc) return rc;
  if (rows <= 0 || k <= 0) return fail(MOE_ERR_INVALID_ARG, "quantize_weights: rows, k must be > 0");
  if (rows % kPanel || k % kBlock)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "quantize_weights: rows %% 32 and k %% 256 must be 0");
  if ((rc = check_device())) return rc;
  return launch_quantize_weights(w, rows, k, trits, scales, static_cast<cudaStream_t>(stream));
}

int moe_quantize_weights_sign(const float* w, int64_t rows, int64_t k, uint32_t* codes, uint16_t* scales,
                              moe_stream_t stream) {
  int rc = check_ptrs("quantize_weights_sign", w, codes, scales);
  if (rc) return rc;
  if (rows <= 0 || k <= 0) return fail(MOE_ERR_INVALID_ARG, "quantize_weights_sign: rows, k must be > 0");
  if (rows % kPanel || k % kBlock)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "quantize_weights_sign: rows %% 32 and k %% 256 must be 0");
  if ((rc = check_device())) return rc;
  return launch_quantize_weights(w, rows, k, codes, scales, static_cast<cudaStream_t>(stream), true);
}

int moe_quantize_weights_e16(const float* w, int64_t rows, int64_t k, uint32_t* trits, uint32_t* codes,
                             uint16_t* anchors, moe_stream_t stream) {
  int rc = check_ptrs("quantize_weights_e16", w, trits, codes, anchors);
  if (rc) return rc;
  if (rows <= 0 || k <= 0) return fail(MOE_ERR_INVALID_ARG, "quantize_weights_e16: rows, k must be > 0");
  if (rows % kPanel || k % kBlock)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "quantize_weights_e16: rows %% 32 and k %% 256 must be 0");
  if ((rc = check_device())) return rc;
  return launch_quantize_weights_e16(w, rows, k, trits, codes, anchors, static_cast<cudaStream_t>(stream));
}

int moe_quant_act_q8(const float* x, int32_t ntok, int32_t k, int8_t* xq, float* xd,
                     moe_stream_t stream) {
  int rc = check_ptrs("quant_act_q8", x, xq, xd);
  if (rc) return rc;
  if (ntok <= 0 || k <= 0) return fail(MOE_ERR_INVALID_ARG, "quant_act_q8: ntok, k must be > 0");
  if (k % kQBlock || k > 65536 || ntok > (1 << 24))
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "quant_act_q8: k %% 32 == 0, k <= 65536, ntok <= 2^24");
  if ((rc = check_device())) return rc;
  return launch_quant_act_q8(x, ntok, k, xq, xd, static_cast<cudaStream_t>(stream));
}

int moe_route_topk(const float* x, const float* w_router, int32_t ntok, int32_t hidden,
                   int32_t n_experts, int32_t top_k, int32_t* idx, float* wts, void* ws,
                   size_t ws_bytes, moe_stream_t stream) {
  int rc = check_ptrs("route_topk", x, w_router, idx, wts, ws);
  if (rc) return rc;
  if (ntok <= 0 || hidden <= 0 || n_experts <= 0 || top_k <= 0 || top_k > n_experts)
    return fail(MOE_ERR_INVALID_ARG, "route_topk: need positive sizes and top_k <= n_experts");
  if (hidden % kBlock || hidden > kMaxHidden || n_experts > kMaxExperts || top_k > kMaxTopK ||
      ntok > 65536)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "route_topk: shape outside the documented limits");
  if (ws_bytes < moe_route_workspace_bytes(ntok, n_experts))
    return fail(MOE_ERR_WORKSPACE, "route_topk: workspace %zu < %zu bytes", ws_bytes,
                moe_route_workspace_bytes(ntok, n_experts));
  if ((rc = check_device())) return rc;
  float* logits = reinterpret_cast<float*>(static_cast<unsigned char*>(ws) + kWsHeaderBytes);
  return launch_route_topk(x, w_router, ntok, hidden, n_experts, top_k, idx, wts, logits,
                           static_cast<cudaStream_t>(stream));
}

static int ffn_common(const char* what, const moe_layer* L, int32_t ntok, const int8_t* xq,
                      const float* xd, const int32_t* idx, const float* wts, float* y, void* ws,
                      size_t ws_bytes, bool prefill, WsLayout* W) {
  int rc = check_layer(L);
  if (rc) return rc;
  if ((rc = check_ptrs(what, xq, xd, idx, wts, y, ws))) return rc;
  if (ntok <= 0) return fail(MOE_ERR_INVALID_ARG, "%s: ntok must be > 0", what);
  if (!prefill && ntok > kMaxDecodeTokens)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "%s: decode takes at most %d tokens", what, kMaxDecodeTokens);
  if (prefill && ntok > 65536) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "%s: ntok <= 65536", what);
  *W = ws_layout(L->hidden, L->ffn, L->n_experts, L->top_k, ntok, prefill);
  if (ws_bytes < W->total)
    return fail(MOE_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", what, ws_bytes, W->total);
  return check_device();
}

int moe_expert_ffn_decode(const moe_layer* L, int32_t ntok, const int8_t* xq, const float* xd,
                          const int32_t* idx, const float* wts, float* y, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
  WsLayout W;
  int rc = ffn_common("expert_ffn_decode", L, ntok, xq, xd, idx, wts, y, ws, ws_bytes, false, &W);
  if (rc) return rc;
  DecodeParams P = make_params(L, ntok, xq, xd, idx, wts, y, ws, W);
  return launch_decode(P, ws, W, static_cast<cudaStream_t>(stream));
}

int moe_expert_ffn_prefill(const moe_layer* L, int32_t ntok, const int8_t* xq, const float* xd,
                           const int32_t* idx, const float* wts, float* y, void* ws, size_t ws_bytes,
                           moe_stream_t stream) {
  WsLayout W;
  int rc = ffn_common("expert_ffn_prefill", L, ntok, xq, xd, idx, wts, y, ws, ws_bytes, true, &W);
  if (rc) return rc;
  DecodeParams P = make_params(L, ntok, xq, xd, idx, wts, y, ws, W);
  return launch_prefill(P, static_cast<cudaStream_t>(stream));
}

static int check_shared(const char* what, const moe_shared* S);

// moe_forward, and with `shared` (one token, a shared expert the one-token
// step takes) the shared expert in the same launch; *fused tells which.
static int forward_impl(const moe_layer* L, const float* w_router, int32_t ntok, const float* x, float* y,
                        void* ws, size_t ws_bytes, moe_stream_t stream, const SharedParams* shared, bool* fused) {
  if (fused) *fused = false;
  int rc = check_layer(L);
  if (rc) return rc;
  if ((rc = check_ptrs("forward", w_router, x, y, ws))) return rc;
  if (ntok <= 0 || ntok > 65536) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "forward: 1 <= ntok <= 65536");
  const bool prefill = ntok > kMaxDecodeTokens;
  // layers whose one token does not take the fused one-token step: sign
  // codes and two-level scales of shapes the step does not fit (ternary
  // layers of such shapes take the first-version one-token chain below)
  bool chain1 = false;
  WsLayout W = ws_layout(L->hidden, L->ffn, L->n_experts, L->top_k, ntok, prefill);
  if (ws_bytes < W.total) return fail(MOE_ERR_WORKSPACE, "forward: workspace %zu < %zu bytes", ws_bytes, W.total);
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char* base = static_cast<unsigned char*>(ws);
  int8_t* xq = reinterpret_cast<int8_t*>(base + W.xq);
  float* xd = reinterpret_cast<float*>(base + W.xd);
  int32_t* idx = reinterpret_cast<int32_t*>(base + W.idx);
  float* wts = reinterpret_cast<float*>(base + W.wts);
  float* logits = reinterpret_cast<float*>(base + W.logits);
  DecodeParams P = make_params(L, ntok, xq, xd, idx, wts, y, ws, W);
  if (ntok == 1 && L->gate.format != MOE_FORMAT_TERNARY) {
    size_t smem_s = 0;
    chain1 = !step1_supported(P, sm_count(), &smem_s);
  }
  if ((ntok > 1 || chain1) && !prefill && route_group_ok(P, sm_count())) {
    // few tokens (and one token the fused step does not take): router logits, activation
    // quantization, top-k and grouping in one launch, then the grouped
    // mat-vecs
    WsHeader* hd = reinterpret_cast<WsHeader*>(ws);
    if ((rc = launch_route_group(P, x, w_router, logits, wts, reinterpret_cast<uint32_t*>(&hd->pad[1]), sm_count(), s)))
      return rc;
    return launch_ffn(P, s);
  }
  if ((ntok > 1 || chain1) && !prefill && router_quant_small_ok(ntok, L->hidden)) {
    // the same in two launches where no one-wave shape exists: router
    // logits with the activation quantization, then the top-k with the
    // grouping
    if ((rc = launch_router_quant_small(x, w_router, ntok, L->hidden, L->n_experts, logits, xq, xd, s)))
      return rc;
    if ((rc = launch_topk_group(P, logits, wts, s))) return rc;
    return launch_ffn(P, s);
  }
  if (ntok > 1 || chain1) {
    if ((rc = launch_quant_act_q8(x, ntok, L->hidden, xq, xd, s))) return rc;
    if ((rc = launch_route_topk(x, w_router, ntok, L->hidden, L->n_experts, L->top_k, idx, wts, logits, s)))
      return rc;
    return prefill ? launch_prefill(P, s) : launch_decode(P, ws, W, s);
  }
  // one token: the whole step in one cooperative kernel where the shape
  // allows it; otherwise act quant, router and top-k in one kernel, then the
  // gate/up and down kernels, chained with programmatic dependent launch
  Decode2Params D = make_d2(P, ws, W);
  D.x = x;
  D.wr = w_router;
  if (one_token_on_tensor_cores(P)) {
    // the routing kernel, then the tensor-core mat-vecs over the top_k slots
    if ((rc = launch_route_only(D, s))) return rc;
    return launch_ffn_tc(P, s);
  }
  size_t smem1 = 0;
  if (step1_supported(P, D.n_sm, &smem1)) {
    WsHeader* hd = reinterpret_cast<WsHeader*>(ws);
    if (shared && fused) *fused = true;
    return launch_step1(D, reinterpret_cast<unsigned long long*>(&hd->pad[3]),
                        reinterpret_cast<unsigned long long*>(static_cast<unsigned char*>(ws) + W.units), s,
                        fused ? shared : nullptr,
                        reinterpret_cast<unsigned long long*>(static_cast<unsigned char*>(ws) + W.sunits));
  }
  return launch_decode2(D, true, s);
}

int moe_forward(const moe_layer* L, const float* w_router, int32_t ntok, const float* x, float* y,
                void* ws, size_t ws_bytes, moe_stream_t stream) {
  return forward_impl(L, w_router, ntok, x, y, ws, ws_bytes, stream, nullptr, nullptr);
}

int moe_forward_shared(const moe_layer* L, const moe_shared* S, const float* w_router, int32_t ntok,
                       const float* x, float* y, void* ws, size_t ws_bytes, void* shared_ws,
                       size_t sws_bytes, moe_stream_t stream) {
  int rc = check_layer(L);
  if (rc) return rc;
  if ((rc = check_shared("forward_shared", S))) return rc;
  if ((rc = check_ptrs("forward_shared", w_router, x, y, ws, shared_ws))) return rc;
  if (S->hidden != L->hidden)
    return fail(MOE_ERR_INVALID_ARG, "forward_shared: shared expert hidden %d != layer hidden %d", S->hidden, L->hidden);
  if (ntok <= 0 || ntok > 65536) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "forward_shared: 1 <= ntok <= 65536");
  const size_t sneed = shared_ws_bytes(S->hidden, S->ffn, ntok);
  if (sws_bytes < sneed)
    return fail(MOE_ERR_WORKSPACE, "forward_shared: shared workspace %zu < %zu bytes", sws_bytes, sneed);
  const SharedParams SP{S->hidden, S->ffn, S->gate_q, S->gate_d, S->up_q, S->up_d, S->down_q, S->down_d};
  const bool fusable = ntok == 1 && S->ffn / kQBlock <= kMaxSharedUnits;
  bool fused = false;
  if ((rc = forward_impl(L, w_router, ntok, x, y, ws, ws_bytes, stream, fusable ? &SP : nullptr, &fused))) return rc;
  if (fused) return MOE_OK;
  // the shared expert's own kernels on the int8 x the step left in ws
  const WsLayout W = ws_layout(L->hidden, L->ffn, L->n_experts, L->top_k, ntok, ntok > kMaxDecodeTokens);
  const unsigned char* base = static_cast<const unsigned char*>(ws);
  return launch_shared_ffn_add(SP, ntok, reinterpret_cast<const int8_t*>(base + W.xq),
                               reinterpret_cast<const float*>(base + W.xd), y, shared_ws,
                               static_cast<cudaStream_t>(stream));
}

int moe_forward_host(const moe_layer* L, const float* w_router, int32_t ntok, const float* x_host,
                     float* y_host, void* ws, size_t ws_bytes, moe_stream_t stream) {
  int rc = check_layer(L);
  if (rc) return rc;
  if (!x_host || !y_host) return fail(MOE_ERR_INVALID_ARG, "forward_host: NULL host buffer");
  if ((rc = check_ptrs("forward_host", w_router, ws))) return rc;
  if (ntok <= 0 || ntok > 65536) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "forward_host: 1 <= ntok <= 65536");
  const bool prefill = ntok > kMaxDecodeTokens;
  WsLayout W = ws_layout(L->hidden, L->ffn, L->n_experts, L->top_k, ntok, prefill);
  if (ws_bytes < W.total)
    return fail(MOE_ERR_WORKSPACE, "forward_host: workspace %zu < %zu bytes", ws_bytes, W.total);
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char* base = static_cast<unsigned char*>(ws);
  float* xs = reinterpret_cast<float*>(base + W.xs);
  float* ys = reinterpret_cast<float*>(base + W.ys);
  const size_t bytes = sizeof(float) * static_cast<size_t>(ntok) * L->hidden;
  // A few kilobytes of page-locked memory the GPU can address: one CTA
  // copies x in with loads over the bus (about a microsecond, and chained to
  // the step by programmatic dependent launch) instead of a DMA copy, whose
  // setup costs several microseconds, and the step's kernels store y straight
  // into the host buffer.  Larger or pageable buffers: DMA copies.
  const void* xd = host_device_view(x_host);
  void* yd = host_device_view(y_host);
  const bool small = bytes <= kSmallHostCopy && xd && yd && aligned16(xd) && aligned16(yd);
  cudaError_t err = cudaSuccess;
  if (small) {
    if ((rc = launch_copy16(xs, xd, bytes, s))) return rc;
  } else {
    err = cudaMemcpyAsync(xs, x_host, bytes, cudaMemcpyHostToDevice, s);
    if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "forward_host: copy in: %s", cudaGetErrorString(err));
  }
  if (small) return moe_forward(L, w_router, ntok, xs, static_cast<float*>(yd), ws, ws_bytes, stream);
  if ((rc = moe_forward(L, w_router, ntok, xs, ys, ws, ws_bytes, stream))) return rc;
  err = cudaMemcpyAsync(y_host, ys, bytes, cudaMemcpyDeviceToHost, s);
  if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "forward_host: copy out: %s", cudaGetErrorString(err));
  return MOE_OK;
}

static int check_shared(const char* what, const moe_shared* S) {
  if (!S) return fail(MOE_ERR_INVALID_ARG, "%s: NULL shared expert", what);
  if (S->hidden <= 0 || S->ffn <= 0) return fail(MOE_ERR_INVALID_ARG, "%s: sizes must be positive", what);
  if (S->hidden % kBlock || S->ffn % kQBlock || S->hidden > kMaxHidden || S->ffn > kMaxFfn)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "%s: hidden %% 256, ffn %% 32, hidden <= %d, ffn <= %d", what, kMaxHidden,
                kMaxFfn);
  return check_ptrs(what, S->gate_q, S->gate_d, S->up_q, S->up_d, S->down_q, S->down_d);
}

int moe_quantize_weights_q8(const float* w, int64_t rows, int64_t k, int8_t* q, uint16_t* d, moe_stream_t stream) {
  int rc = check_ptrs("quantize_weights_q8", w, q, d);
  if (rc) return rc;
  if (rows <= 0 || k <= 0) return fail(MOE_ERR_INVALID_ARG, "quantize_weights_q8: rows, k must be > 0");
  if (k % kQBlock) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "quantize_weights_q8: k %% 32 must be 0");
  if ((rc = check_device())) return rc;
  return launch_quantize_weights_q8(w, rows, k, q, d, static_cast<cudaStream_t>(stream));
}

size_t moe_shared_workspace_bytes(const moe_shared* S, int32_t ntok) {
  if (!S || S->hidden <= 0 || S->ffn <= 0 || S->ffn % kQBlock || ntok <= 0 || ntok > 65536) return 0;
  return shared_ws_bytes(S->hidden, S->ffn, ntok);
}

int moe_shared_ffn_add(const moe_shared* S, int32_t ntok, const int8_t* xq, const float* xd, float* y, void* ws,
                       size_t ws_bytes, moe_stream_t stream) {
  int rc = check_shared("shared_ffn_add", S);
  if (rc) return rc;
  if ((rc = check_ptrs("shared_ffn_add", xq, xd, y, ws))) return rc;
  if (ntok <= 0 || ntok > 65536) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "shared_ffn_add: 1 <= ntok <= 65536");
  const size_t need = shared_ws_bytes(S->hidden, S->ffn, ntok);
  if (ws_bytes < need) return fail(MOE_ERR_WORKSPACE, "shared_ffn_add: workspace %zu < %zu bytes", ws_bytes, need);
  if ((rc = check_device())) return rc;
  SharedParams P{S->hidden, S->ffn, S->gate_q, S->gate_d, S->up_q, S->up_d, S->down_q, S->down_d};
  return launch_shared_ffn_add(P, ntok, xq, xd, y, ws, static_cast<cudaStream_t>(stream));
}

int moe_check_status(void* ws, moe_stream_t stream) {
  if (!ws) return fail(MOE_ERR_INVALID_ARG, "check_status: NULL workspace");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t status = 0;
  cudaError_t err = cudaMemcpyAsync(&status, ws, sizeof(status), cudaMemcpyDeviceToHost, s);
  if (err == cudaSuccess) err = cudaStreamSynchronize(s);
  if (err == cudaSuccess) err = cudaMemsetAsync(ws, 0, sizeof(int32_t), s);
  if (err == cudaSuccess) err = cudaStreamSynchronize(s);
  if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "check_status: %s", cudaGetErrorString(err));
  if (status) set_error("device reported status %d", status);
  return status;
}

const char* moe_last_error(void) { return g_last_error; }

int64_t moe_launch_count(void) { return g_launches; }

int moe_trace_begin(void* const* events, int32_t capacity) {
  if (!events || capacity <= 0) return fail(MOE_ERR_INVALID_ARG, "trace_begin: no events");
  g_trace_events = reinterpret_cast<cudaEvent_t*>(const_cast<void**>(events));
  g_trace_cap = capacity;
  g_trace_n = 0;
  return MOE_OK;
}

int moe_trace_end(int32_t* kernel_ids, int32_t capacity) {
  const int n = g_trace_n;
  if (kernel_ids)
    for (int i = 0; i < n && i < capacity; ++i) kernel_ids[i] = g_trace_ids[i];
  g_trace_events = nullptr;
  g_trace_cap = 0;
  g_trace_n = 0;
  return n;
}

const char* moe_kernel_name(int32_t id) {
  static const char* names[MOE_K_COUNT] = {
      "quantize_weights", "quant_act_q8", "router_logits", "topk_softmax", "group",
      "gateup", "down", "debug_matvec", "prefill_gateup", "prefill_down", "route", "combine", "step1", "prefill_gather", "copy",
      "router_quant", "topk_group", "shared", "tc_gateup", "tc_down", "route_group"};
  return (id >= 0 && id < MOE_K_COUNT) ? names[id] : "";
}

int moe_debug_matvec(const moe_tmat* m, int32_t ntok, const int8_t* xq, const float* xd, float* out,
                     int32_t* isum, moe_stream_t stream) {
  if (!m) return fail(MOE_ERR_INVALID_ARG, "debug_matvec: NULL matrix");
  int rc = check_ptrs("debug_matvec", m->trits, m->scales, xq, xd, out);
  if (rc) return rc;
  if (isum && !aligned16(isum)) return fail(MOE_ERR_ALIGNMENT, "debug_matvec: isum not aligned");
  if (ntok <= 0 || ntok > kMaxDecodeTokens || m->rows <= 0 || m->k <= 0)
    return fail(MOE_ERR_INVALID_ARG, "debug_matvec: bad sizes");
  if (m->rows % kPanel || m->k % kBlock || m->k > kMaxHidden)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "debug_matvec: rows %% 32, k %% 256, k <= %d", kMaxHidden);
  if (m->format != MOE_FORMAT_TERNARY && m->format != MOE_FORMAT_SIGN && m->format != MOE_FORMAT_E16)
    return fail(MOE_ERR_INVALID_ARG, "debug_matvec: unknown weight format %d", m->format);
  if (m->format == MOE_FORMAT_E16 && (!m->codes || !aligned16(m->codes)))
    return fail(MOE_ERR_INVALID_ARG, "debug_matvec: E16 codes missing or not 16-byte aligned");
  if ((rc = check_device())) return rc;
  return launch_debug_matvec(m, ntok, xq, xd, out, isum, static_cast<cudaStream_t>(stream));
}

int moe_debug_ffn_blocksums(const moe_layer* L, int32_t ntok, const int8_t* xq, const float* xd,
                            const int32_t* idx, const float* wts, float* y, void* ws, size_t ws_bytes,
                            int32_t prefill, int32_t* isum_gu, int32_t* isum_dn, int8_t* aq,
                            moe_stream_t stream) {
  WsLayout W;
  int rc = ffn_common("debug_ffn_blocksums", L, ntok, xq, xd, idx, wts, y, ws, ws_bytes, prefill != 0, &W);
  if (rc) return rc;
  if (!isum_gu || !isum_dn || !aligned16(isum_gu) || !aligned16(isum_dn))
    return fail(MOE_ERR_INVALID_ARG, "debug_ffn_blocksums: isum_gu and isum_dn must be 16-byte aligned device arrays");
  DecodeParams P = make_params(L, ntok, xq, xd, idx, wts, y, ws, W);
  P.dbg_isum_gu = isum_gu;
  P.dbg_isum_dn = isum_dn;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (prefill) {
    if (!prefill_tc_supported(P))
      return fail(MOE_ERR_UNSUPPORTED_SHAPE, "debug_ffn_blocksums: the prefill GEMM does not take this layer");
    rc = launch_prefill(P, s);
  } else {
    if (!tc_ffn_supported(P))
      return fail(MOE_ERR_UNSUPPORTED_SHAPE, "debug_ffn_blocksums: the tensor-core decode does not take this layer");
    if (!P.direct && (rc = launch_group(P, s))) return rc;
    if (!rc) rc = launch_ffn_tc(P, s);
  }
  if (rc || !aq) return rc;
  const size_t bytes = static_cast<size_t>(ntok) * L->top_k * L->ffn;
  cudaError_t err = cudaMemcpyAsync(aq, P.aq, bytes, cudaMemcpyDeviceToDevice, s);
  if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "debug_ffn_blocksums: copy of aq: %s", cudaGetErrorString(err));
  return MOE_OK;
}

int moe_debug_wait_knob(void* ws, size_t ws_bytes, int32_t mode, int32_t polls, moe_stream_t stream) {
  if (!ws || ws_bytes < kWsHeaderBytes) return fail(MOE_ERR_INVALID_ARG, "debug_wait_knob: no workspace");
  if (mode < 0 || mode > kKnobTcGather || polls < 0)
    return fail(MOE_ERR_INVALID_ARG, "debug_wait_knob: mode %d, polls %d", mode, polls);
  int rc = check_device();
  if (rc) return rc;
  const int32_t v[2] = {mode, polls};
  cudaError_t err = cudaMemcpyAsync(static_cast<int32_t*>(ws) + kWsKnobMode, v, sizeof(v), cudaMemcpyHostToDevice,
                                    static_cast<cudaStream_t>(stream));
  if (err == cudaSuccess) err = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "debug_wait_knob: %s", cudaGetErrorString(err));
  return MOE_OK;
}

}  // extern "C"
