// noalloc.cu -- moe_expert_ffn_decode_static: the decode expert FFN with its
// scratch memory in a fixed device array of this library instead of a
// caller-provided workspace.
//
// Who needs this: callers that cannot allocate device memory when they call
// the library -- a plug-in living inside a host application that owns every
// device allocation and hands the plug-in only its inputs and outputs; a
// serving loop that must never enter the CUDA allocator (cudaMalloc can
// synchronize the device and stall other streams); code that runs under a
// fixed device-memory budget fixed at start-up.  For them the library keeps
// kStaticScratchBytes of device memory of its own, reserved when the library
// is loaded onto a GPU and held until the process exits.
#include <mutex>

#include "bitmoe.h"
#include "common.cuh"
#include "decode.cuh"

namespace bitmoe {

// The scratch: status word, intermediate int8 activations, per-slot down
// outputs, arrival counters and grouping tables of one decode call (the same
// layout moe_expert_ffn_decode uses in a caller workspace).
constexpr size_t kStaticScratchBytes = size_t(4) << 20;  // 4 MiB per device
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on each device, looked up on the first
// call made with that device current.  In host code the symbol name stands for
// a host-side shadow, not for device memory, so the address must come from
// cudaGetSymbolAddress.
static std::mutex g_scratch_mu;
static void* g_scratch_ptr[64] = {};

static int static_scratch(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(err));
  if (dev < 0 || dev >= 64) return fail(MOE_ERR_DEVICE, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_static_scratch);
    if (err != cudaSuccess || !p)
      return fail(MOE_ERR_CUDA, "cudaGetSymbolAddress(static scratch): %s", cudaGetErrorString(err));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace bitmoe

using namespace bitmoe;

extern "C" int moe_expert_ffn_decode_static(const moe_layer* layer, int32_t ntok, const int8_t* xq,
                                            const float* xd, const int32_t* idx, const float* wts,
                                            float* y, moe_stream_t stream) {
  // Every argument is checked before the shared array is touched, so a call
  // that is refused leaves it (and any call still using it) alone.
  int rc = check_decode_call("expert_ffn_decode_static", layer, ntok, xq, xd, idx, wts, y);
  if (rc) return rc;
  const size_t need = moe_workspace_bytes(layer, ntok, 0);
  if (need == 0) return fail(MOE_ERR_INVALID_ARG, "expert_ffn_decode_static: invalid layer or ntok");
  if (need > kStaticScratchBytes)
    return fail(MOE_ERR_WORKSPACE,
                "expert_ffn_decode_static: this call needs %zu bytes of scratch, the static scratch "
                "holds %zu (use moe_expert_ffn_decode with a workspace)",
                need, kStaticScratchBytes);
  void* scratch = nullptr;
  rc = static_scratch(&scratch);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The array keeps what the previous call left there.  Counters and the status
  // word must start at zero: clear the whole region this call uses.  The
  // status word is cleared by every call, so device-side reports (bad expert
  // ids) cannot be read back through this entry point.
  cudaError_t err = cudaMemsetAsync(scratch, 0, need, s);
  if (err != cudaSuccess)
    return fail(MOE_ERR_CUDA, "expert_ffn_decode_static: clearing scratch: %s", cudaGetErrorString(err));
  return moe_expert_ffn_decode(layer, ntok, xq, xd, idx, wts, y, scratch, kStaticScratchBytes, stream);
}
