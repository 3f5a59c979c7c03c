// decode2.cuh -- the decode step as three chained kernels (sm_100a):
//   k_route        activation q8 + router logits + top-k softmax, fused; with
//                  more than one token the last CTA also groups the (token,
//                  slot) pairs by expert
//   k_gateup_tma   gate+up mat-vecs, SwiGLU and int8 requant of a
//   k_down_tma     down mat-vec and the weighted top-k combine
// launched back to back with programmatic dependent launch.  The mat-vec
// kernels are persistent (one or two CTAs per SM); each warp streams the
// 256-weight blocks of 32-row panels it decodes into its own shared-memory
// ring with cp.async, decodes the base-3 digits in registers and accumulates
// with dp4a.
#pragma once

#include "common.cuh"
#include "decode.cuh"

namespace bitmoe {

constexpr int kConsumerWarps = 8;  // warps of a mat-vec CTA
constexpr int kMatBytes = kBlockWords * kPanel * 4 + kPanel * 2;  // 1728: one block of a panel
constexpr int kActBytes = kBlock + kSubPerBlock * 4;              // 288: codes + scales of one block

struct Decode2Params {
  DecodeParams P;           // shapes, weights, FFN inputs/outputs, status, grouping tables
  uint32_t* route_cnt;      // last-arriver counter of k_route (kept at 0)
  float* logits;            // [ntok][E]
  const float* x;           // [ntok][hidden] fp32 input of k_route
  const float* wr;          // [E][hidden] router
  int route_warps;          // experts per k_route CTA
  int route_tc;             // tokens per k_route CTA
  int n_sm;                 // persistent grid size of the mat-vec kernels
};

int launch_decode2(Decode2Params& D, bool with_route, cudaStream_t stream);
// k_route alone (activation q8, router logits, top-k softmax into P.idx,
// P.wts; grouping with more than one token), for the tensor-core mat-vecs.
int launch_route_only(Decode2Params& D, cudaStream_t stream);

// The whole one-token step in one cooperative kernel (step1.cu).
bool step1_supported(const DecodeParams& P, int n_sm, size_t* smem);
// `ticket`: a 64-bit counter that only grows; `units`: top_k * (ffn / 32) * 10
// 8-byte words for the tagged gate/up unit outputs; the logits area of D must
// hold 128 bytes per expert (tagged logits).  With `shared` (hidden equal to
// the layer's, ffn a multiple of 32 of at most kMaxSharedUnits blocks) the
// same launch adds the shared expert's FFN to y; `sunits` then holds
// (ffn / 32) * 10 words for its tagged block outputs.
struct SharedParams;
int launch_step1(const Decode2Params& D, unsigned long long* ticket, unsigned long long* units,
                 cudaStream_t stream, const SharedParams* shared = nullptr, unsigned long long* sunits = nullptr);

}  // namespace bitmoe
