// common.cuh -- shared host/device helpers of libbitmoe (sm_100a only).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdarg>
#include <cstddef>
#include <cstdio>

#include "bitmoe.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ != 1000)
#error "libbitmoe is written for sm_100a only"
#endif

namespace bitmoe {

constexpr int kBlock = 256;      // weights per ternary block
constexpr int kBlockWords = 13;  // packed uint32 words per block
constexpr int kSignWords = 8;    // uint32 words per block of 1-bit sign codes
constexpr int kE16Words = 2;     // uint32 words of 4-bit sub-scale codes per block (two-level scales)
constexpr int kPanel = 32;       // rows per interleaved panel
constexpr int kQBlock = 32;      // activations per int8 block
constexpr int kSubPerBlock = kBlock / kQBlock;  // 8 activation blocks per weight block

constexpr int kMaxHidden = 16384;
constexpr int kMaxFfn = 8192;
constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 32;
constexpr int kMaxDecodeTokens = 64;
constexpr int kMaxDynSmem = 227 * 1024;  // opt-in dynamic shared memory per CTA

// Workspace header: the first 256 bytes hold the device status word.
struct WsHeader {
  int32_t status;    // first error code seen by a kernel (0 = ok)
  int32_t pad[63];   // pad[0]: route counter; pad[1]: route_group counter; pad[3..4]: 64-bit
                     // one-token step tickets;
                     // pad[8..9]: the wait test knob (below)
};
// Test knob of the bounded device waits (moe_debug_wait_knob; zero in every
// fresh workspace): header word kWsKnobMode selects a wait that is made to run
// out, word kWsKnobPolls (if nonzero) replaces the poll budget of the kernels
// that read the knob.
constexpr int kWsKnobMode = 9;   // word index in the header (pad[8])
constexpr int kWsKnobPolls = 10; // pad[9]
constexpr int kKnobStep1Tag = 1; // the one-token step polls for a logit tag that no CTA publishes
constexpr int kKnobTcGather = 2; // the tensor-core mat-vecs' gather warp withholds its first arrival
static_assert(offsetof(WsHeader, pad) + 3 * sizeof(int32_t) == 16, "8-byte aligned ticket counter");
constexpr size_t kWsHeaderBytes = sizeof(WsHeader);

// ---------------------------------------------------------------- host errors
void set_error(const char* fmt, ...);
int fail(int code, const char* fmt, ...);
int check_launch(const char* what);
int check_device();

// Called after every kernel launch: counts it and, while tracing, records an
// event on its stream.
void note_launch(int kernel_id, cudaStream_t stream);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------- launches
// Programmatic dependent launch: a kernel launched this way may start while
// the previous kernel on the stream finishes; it calls pdl_enter() first,
// which waits until the previous kernel has completed (its writes visible)
// and lets the next kernel start launching in turn.  Without a previous PDL
// edge the wait returns at once.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                     Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- device helpers
__device__ __forceinline__ void record_status(int32_t* status, int32_t code) {
  atomicCAS(status, 0, code);
}

// Bounds-checked build (compiled with -DMOE_CHECKED; the tests build it as
// a separate library): MOE_IN(i, n) is true when 0 <= i < n; otherwise it
// records MOE_ERR_BOUNDS in the status word and is false, so that the guarded
// access is skipped.  In the normal build it is always true and costs nothing.
#ifdef MOE_CHECKED
#define MOE_IN(i, n, status) \
  ((static_cast<unsigned long long>(i) < static_cast<unsigned long long>(n)) ? true \
   : (record_status((status), MOE_ERR_BOUNDS), false))
#else
#define MOE_IN(i, n, status) true
#endif

// fp64 -> binary16, round to nearest even, in one conversion.
__device__ __forceinline__ uint16_t f64_to_f16_rn(double x) {
  uint16_t h;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(x));
  return h;
}

__device__ __forceinline__ float f16_bits_to_f32(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

// Streaming 32-bit load that does not allocate in L1 (weights are read once).
__device__ __forceinline__ uint32_t ld_stream_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}

// Order-preserving map of an fp32 value to uint32 (larger value, larger key;
// -0 ranks as +0), and back (-0 comes back as +0).
__device__ __forceinline__ uint32_t f32_key(float v) {
  const uint32_t b = __float_as_uint(v == 0.f ? 0.f : v);  // -0 ranks as +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float f32_unkey(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

}  // namespace bitmoe
