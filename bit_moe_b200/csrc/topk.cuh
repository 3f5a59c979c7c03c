// topk.cuh -- top-k of one token's expert logits and the renormalised softmax
// over the selected, by one warp in registers (sm_100a).
//
// llama-modchip page, "Key highlights": every one of the token's top-k experts
// is evaluated.  The selection is an integer result: k rounds, each taking the
// largest remaining logit and, among equal logits, the lowest expert id.  The
// weights are w_r = exp(l_r - l_0) / sum_s exp(l_s - l_0), the sum taken in
// rank order s = 0, 1, ..., k-1.
#pragma once

#include "common.cuh"

namespace bitmoe {

// key[i]: f32_key of the logit of expert lane + 32*i, for the i set in `need`
// (the others are never chosen).  On return lane r < k holds the expert of
// rank r in my_e and its weight in my_w.
template <int kPer>
__device__ __forceinline__ void warp_topk_softmax(const uint32_t (&key)[kPer], uint32_t need, int k,
                                                  int lane, int& my_e, float& my_w) {
  constexpr int kNone = 0x7fffffff;
  uint32_t avail = need;
  uint32_t my_k = 0u, k0 = 0u;
  my_e = 0;
#pragma unroll 1
  for (int r = 0; r < k; ++r) {
    // the lane's best remaining entry (its entries are in ascending id order,
    // so it keeps the first of equal keys), then the largest key over the
    // warp and the lowest id holding it
    uint32_t bk = 0u;
    int bi = kNone;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (((avail >> i) & 1u) && (bi == kNone || key[i] > bk)) { bk = key[i]; bi = lane + 32 * i; }
    const uint32_t wk = __reduce_max_sync(0xffffffffu, bi == kNone ? 0u : bk);
    const int wi = static_cast<int>(
        __reduce_min_sync(0xffffffffu, (bi != kNone && bk == wk) ? static_cast<uint32_t>(bi) : 0xffffffffu));
    if ((wi & 31) == lane && wi >= 0) avail &= ~(1u << (wi >> 5));
    if (lane == r) { my_e = wi; my_k = wk; }
    if (r == 0) k0 = wk;
  }
  // the logits come back from their keys (-0 as +0, which gives the same
  // differences' exponentials)
  const float l0 = f32_unkey(k0);
  const float ex = lane < k ? expf(__fsub_rn(f32_unkey(my_k), l0)) : 0.f;
  float den = 0.f;
#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r) {
    const float er = __shfl_sync(0xffffffffu, ex, r);
    if (r < k) den = __fadd_rn(den, er);
  }
  my_w = lane < k ? __fdiv_rn(ex, den) : 0.f;
}

}  // namespace bitmoe
