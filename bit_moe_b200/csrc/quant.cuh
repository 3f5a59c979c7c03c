// quant.cuh -- launchers of the weight and activation quantization kernels.
#pragma once
#include "common.cuh"
namespace bitmoe {
int launch_quantize_weights(const float* w, int64_t rows, int64_t k, uint32_t* trits,
                            uint16_t* scales, cudaStream_t stream);
int launch_quant_act_q8(const float* x, int64_t ntok, int k, int8_t* xq, float* xd,
                        cudaStream_t stream);
}  // namespace bitmoe
