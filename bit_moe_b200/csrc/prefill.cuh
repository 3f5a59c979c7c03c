// prefill.cuh -- launcher of the large-batch (prefill) expert FFN.
#pragma once
#include "decode.cuh"
namespace bitmoe {
int launch_prefill(const DecodeParams& P, cudaStream_t stream);
// True if the prefill GEMM takes this layer (ternary format).
bool prefill_tc_supported(const DecodeParams& P);
// Bytes of one activation block of a group of prefill_group_pairs() pairs (split codes, scales, sums).
size_t prefill_block_bytes();
// Most (token, slot) pairs in one group of the prefill GEMM.
int prefill_group_pairs();
}  // namespace bitmoe
