// prefill.cuh -- launcher of the large-batch (prefill) expert FFN.
#pragma once
#include "decode.cuh"
namespace bitmoe {
int launch_prefill(const DecodeParams& P, cudaStream_t stream);
}  // namespace bitmoe
