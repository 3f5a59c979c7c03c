// tcmv.cuh -- launcher of the grouped decode mat-vecs on the tensor cores.
#pragma once
#include "decode.cuh"
namespace bitmoe {
// Most 256-weight blocks of a row the tensor-core mat-vecs hold per unit of
// work (hidden and ffn up to 4096).
constexpr int kTcMaxBlocks = 16;
// True if the grouped tensor-core mat-vecs take this layer (ternary format,
// hidden and ffn at most kTcMaxBlocks blocks).
bool tc_ffn_supported(const DecodeParams& P);
// True if the batch is expected to give items of enough pairs for the
// tensor-core mat-vecs to beat the CUDA-core ones (by measurement).
bool tc_ffn_preferred(const DecodeParams& P);
// Gate/up then down over the items of P (grouped or direct mode), chained by
// programmatic dependent launch.
int launch_ffn_tc(const DecodeParams& P, cudaStream_t stream);
}  // namespace bitmoe
