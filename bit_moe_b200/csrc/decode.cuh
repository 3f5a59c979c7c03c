// decode.cuh -- parameters and launchers of the expert-FFN mat-vec kernels.
#pragma once

#include "common.cuh"

namespace bitmoe {

constexpr int kGateUpWarps = 8;  // warps of a gate/up CTA; they split the hidden blocks
constexpr int kDownWarps = 4;    // warps (= 32-row panels) of a down CTA
constexpr int kChunk = 8;        // most (token, slot) pairs sharing one weight decode

// A work item: up to kChunk (token, slot) pairs routed to one expert.
struct Item {
  int expert;  // -1: pairs whose expert id was out of range
  int start;   // first entry in the pair list
  int count;   // 1..kChunk
  int pad;
};

struct DecodeParams {
  int hidden, ffn, n_experts, top_k, ntok;
  const uint32_t* gate_trits; const uint16_t* gate_scales;
  const uint32_t* up_trits;   const uint16_t* up_scales;
  const uint32_t* down_trits; const uint16_t* down_scales;
  const int8_t* xq; const float* xd;     // [ntok][hidden], [ntok][hidden/32]
  const int32_t* idx; const float* wts;  // [ntok][top_k]
  int8_t* aq; float* ad;                 // [ntok*top_k][ffn], [ntok*top_k][ffn/32]
  float* ye;                             // [ntok*top_k][hidden] per-pair down outputs
  int32_t* cnt;                          // [ntok][hidden/32] arrival counters (kept at 0)
  float* y;                              // [ntok][hidden]
  int32_t* status;
  // grouped mode (ntok > 1): items and the pair list, built on the device
  int direct;                            // 1: item i is pair i (ntok == 1)
  int format;                            // MOE_FORMAT_TERNARY, _SIGN or _E16
  const uint32_t* gate_codes;            // MOE_FORMAT_E16: 4-bit sub-scale words (the
  const uint32_t* up_codes;              // *_scales pointers then hold per-row anchors)
  const uint32_t* down_codes;
  const Item* items;                     // [ntok*top_k + n_experts]
  const int32_t* n_items;
  const int32_t* pairs;                  // [ntok*top_k] pair ids grouped by expert
  int32_t* group_scratch;                // [2*(n_experts+1)] counters for the grouping
  int group_chunk;                       // most pairs per item (kChunk for decode)
  // prefill only: the activation blocks of every 64-pair group, laid out as
  // the tensor-core kernel's shared-memory stages, for gate/up and for down
  unsigned char* bgu;                        // [groups][hidden/256] blocks
  unsigned char* bdn;                        // [groups][ffn/256] blocks
  // test hook of the tensor-core mat-vecs (null otherwise): the exact block
  // sums sum(q * a) of every pair, row and 32-block, gate/up as
  // [pairs][2][ffn][hidden/32] and down as [pairs][hidden][ffn/32]
  int32_t* dbg_isum_gu = nullptr;
  int32_t* dbg_isum_dn = nullptr;
};

// Fetch work item `it`; returns false when there is none.
__device__ __forceinline__ bool fetch_item(const DecodeParams& P, int it, Item& item) {
  if (P.direct) {
    if (it >= P.ntok * P.top_k) return false;
    const int e = P.idx[it];
    item.expert = (e >= 0 && e < P.n_experts) ? e : -1;
    item.start = it;
    item.count = 1;
    return true;
  }
  if (it >= *P.n_items) return false;
  item = P.items[it];
  return true;
}

__device__ __forceinline__ int item_pair(const DecodeParams& P, const Item& item, int n) {
  if (!P.direct && !MOE_IN(item.start + n, P.ntok * P.top_k, P.status)) return 0;
  return P.direct ? item.start + n : P.pairs[item.start + n];
}

// Bounds-checked build: a (token, slot) pair id inside [0, ntok * top_k).
__device__ __forceinline__ bool pair_ok(const DecodeParams& P, int pair) {
  return MOE_IN(pair, P.ntok * P.top_k, P.status);
}

// The CTA that completes the last of token t's top_k slots for 32-row panel
// `panel` of hidden (counted in P.cnt, reset by that CTA) combines
// y[t] = sum_j wts[t][j] * ye[t][j] over the slots in order; called by a
// whole warp (lane = row of the panel) after its ye values are visible.
__device__ __forceinline__ void arrive_and_combine(const DecodeParams& P, int pair, int panel,
                                                   int lane) {
  const int K = P.top_k, H = P.hidden;
  const int t = pair / K;
  if (!MOE_IN(t, P.ntok, P.status) || !MOE_IN(panel, H / kPanel, P.status)) return;
  int32_t* c = P.cnt + static_cast<size_t>(t) * (H / kPanel) + panel;
  int old = 0;
  if (lane == 0) old = atomicAdd(c, 1);
  old = __shfl_sync(0xffffffffu, old, 0);
  if (old == K - 1) {
    __threadfence();
    float y = 0.f;
    const float* ye = P.ye + static_cast<size_t>(t) * K * H + panel * kPanel + lane;
    for (int j = 0; j < K; ++j)
      y = __fmaf_rn(__ldcg(P.wts + static_cast<size_t>(t) * K + j), __ldcg(ye + static_cast<size_t>(j) * H), y);
    P.y[static_cast<size_t>(t) * H + panel * kPanel + lane] = y;
    if (lane == 0) atomicExch(c, 0);
  }
}

// Bytes of workspace the grouped mode needs after `off`; writes the offsets.
struct GroupWs {
  size_t items = 0, n_items = 0, pairs = 0, scratch = 0;
};
size_t group_ws_layout(int E, int npairs, size_t off, GroupWs* G);

// Argument checks of a decode call that do not involve its workspace.
int check_decode_call(const char* what, const moe_layer* L, int32_t ntok, const int8_t* xq, const float* xd,
                      const int32_t* idx, const float* wts, float* y);

int launch_group(const DecodeParams& P, cudaStream_t stream);
// Top-k softmax of P.ntok <= 64 tokens' logits ([ntok][E] fp32) into P.idx
// and wts, then the grouping of launch_group, in one single-CTA kernel.
int launch_topk_group(const DecodeParams& P, const float* logits, float* wts, cudaStream_t stream);
// Router logits, activation quantization, top-k and grouping of up to 64
// tokens in one launch (k_route_group); route_group_ok tells whether a
// one-wave shape exists.  ticket: a workspace counter that is zero between
// launches.
bool route_group_ok(const DecodeParams& P, int n_sm);
int launch_route_group(const DecodeParams& P, const float* x, const float* wr, float* logits, float* wts,
                       uint32_t* ticket, int n_sm, cudaStream_t stream);
int launch_ffn(const DecodeParams& P, cudaStream_t stream);
int launch_debug_matvec(const moe_tmat* m, int ntok, const int8_t* xq, const float* xd, float* out,
                        int32_t* isum, cudaStream_t stream);

}  // namespace bitmoe
