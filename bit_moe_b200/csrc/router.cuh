// router.cuh -- launcher of the router logits and top-k softmax kernels.
#pragma once
#include "common.cuh"
namespace bitmoe {
// logits: scratch [ntok][E] fp32 in device memory.
int launch_route_topk(const float* x, const float* wr, int ntok, int H, int E, int K, int32_t* idx,
                      float* wts, float* logits, cudaStream_t stream);
}  // namespace bitmoe
