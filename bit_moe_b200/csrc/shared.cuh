// shared.cuh -- launchers of the shared expert's 8-bit quantization and FFN.
#pragma once
#include "common.cuh"
namespace bitmoe {
// The shared expert's matrices in 8-bit blocks of 32 (row-major codes,
// fp16 scale per block): gate/up [ffn][hidden], down [hidden][ffn].
struct SharedParams {
  int hidden, ffn;
  const int8_t* gate_q; const uint16_t* gate_d;
  const int8_t* up_q;   const uint16_t* up_d;
  const int8_t* down_q; const uint16_t* down_d;
};
int launch_quantize_weights_q8(const float* w, int64_t rows, int64_t k, int8_t* q, uint16_t* d,
                               cudaStream_t stream);
size_t shared_ws_bytes(int hidden, int ffn, int ntok);
// y [ntok][hidden] += the shared expert's FFN of xq, xd; ws holds
// shared_ws_bytes(hidden, ffn, ntok) bytes.
int launch_shared_ffn_add(const SharedParams& S, int ntok, const int8_t* xq, const float* xd, float* y, void* ws,
                          cudaStream_t stream);
}  // namespace bitmoe
