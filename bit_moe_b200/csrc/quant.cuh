// quant.cuh -- launchers of the weight and activation quantization kernels.
#pragma once
#include "common.cuh"
namespace bitmoe {
// sign: 1-bit sign codes (MOE_FORMAT_SIGN) instead of ternary digits.
int launch_quantize_weights(const float* w, int64_t rows, int64_t k, uint32_t* trits,
                            uint16_t* scales, cudaStream_t stream, bool sign = false);
// Two-level scales (MOE_FORMAT_E16): the per-row anchors, then the digits
// and the 4-bit sub-scale codes.
int launch_quantize_weights_e16(const float* w, int64_t rows, int64_t k, uint32_t* trits, uint32_t* codes,
                                uint16_t* anchors, cudaStream_t stream);
int launch_quant_act_q8(const float* x, int64_t ntok, int k, int8_t* xq, float* xd,
                        cudaStream_t stream);

// One 32-value block of x (one warp): d = amax/127, q = clamp(rint(x/d),
// -127, 127) with IEEE divisions; d = 0 gives q = 0 (pxq_llama README, "PXQ vs
// MXFP4": one scale per 32 values).
__device__ __forceinline__ void quant_act_block(const float* __restrict__ x, int64_t blk, int lane,
                                                int8_t* __restrict__ xq, float* __restrict__ xd) {
  const float v = x[blk * kQBlock + lane];
  const float amax = warp_max(fabsf(v));
  const float d = __fdiv_rn(amax, 127.f);
  int q = 0;
  if (d != 0.f) q = max(-127, min(127, __float2int_rn(__fdiv_rn(v, d))));
  xq[blk * kQBlock + lane] = static_cast<int8_t>(q);
  if (lane == 0) xd[blk] = d;
}
}  // namespace bitmoe
