// router.cuh -- launcher of the router logits and top-k softmax kernels.
#pragma once
#include "common.cuh"
namespace bitmoe {
// logits: scratch [ntok][E] fp32 in device memory.
int launch_route_topk(const float* x, const float* wr, int ntok, int H, int E, int K, int32_t* idx,
                      float* wts, float* logits, cudaStream_t stream);
// Up to 64 tokens (router_quant_small_ok): the router logits and the int8
// quantization of x (xq [ntok][H], xd [ntok][H/32]) in one kernel.
bool router_quant_small_ok(int ntok, int H);
int launch_router_quant_small(const float* x, const float* wr, int ntok, int H, int E, float* logits,
                              int8_t* xq, float* xd, cudaStream_t stream);
}  // namespace bitmoe
