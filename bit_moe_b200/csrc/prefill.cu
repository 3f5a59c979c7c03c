// prefill.cu -- large-batch expert FFN: the (token, slot) pairs are grouped
// by expert and each expert's weights are decoded once for every chunk of its
// tokens (Parakon Runtime README, "How it works": prompt processing at large
// batch takes a GEMM path; pxq_llama README, "What's PXQ?": grouped-MoE GEMM).
#include "common.cuh"
#include "prefill.cuh"

namespace bitmoe {

int launch_prefill(const DecodeParams& P, cudaStream_t stream) {
  DecodeParams Q = P;
  Q.direct = 0;
  int rc = launch_group(Q, stream);
  if (rc) return rc;
  return launch_ffn(Q, stream);
}

}  // namespace bitmoe
