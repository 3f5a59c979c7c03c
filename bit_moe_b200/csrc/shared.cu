// shared.cu -- the shared expert beside the routed ones (sm_100a): an
// always-active FFN kept at higher precision (llama-modchip page, "The
// interesting bit": shared experts stay at 4/5-bit or float precision while
// the routed experts go to 1-bit), read as 8-bit blocks of 32 weights with an
// fp16 scale (the Q8_0 layout of the pxq_llama tensor census), stored
// row-major.  Its output is added to y after the routed experts' combine.
//
// The weights are dense and small next to the routed experts (one expert for
// all tokens), so the mat-vecs are plain dp4a kernels: one warp per output
// row, lane l taking the 32-blocks l, l+32, ... of the row (two 16-byte loads
// of weight codes and of activation codes each), the block sum scaled by both
// block scales and accumulated in fp32, then summed over the warp.
#include "bitmoe.h"
#include "common.cuh"
#include "ptx.cuh"
#include "quant.cuh"
#include "shared.cuh"

namespace bitmoe {

constexpr int kSharedWarps = 8;

// 8-bit weight blocks: d = fp16_RNE(amax / 127) with the division in fp64,
// q = clamp(rint(w / d), -127, 127) with an IEEE fp32 division by the fp16
// value; a block whose d is 0 is all zeros.  One warp per block.
__global__ void k_quantize_weights_q8(const float* __restrict__ w, int64_t nblk, int8_t* __restrict__ q,
                                      uint16_t* __restrict__ d) {
  const int lane = threadIdx.x & 31;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t blk = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); blk < nblk;
       blk += nw) {
    const float v = w[blk * kQBlock + lane];
    const float amax = warp_max(fabsf(v));
    const uint16_t dh = f64_to_f16_rn(static_cast<double>(amax) / 127.0);
    const float df = f16_bits_to_f32(dh);
    int c = 0;
    if (df != 0.f) c = max(-127, min(127, __float2int_rn(__fdiv_rn(v, df))));
    q[blk * kQBlock + lane] = static_cast<int8_t>(c);
    if (lane == 0) d[blk] = dh;
  }
}

// a[t][f] = silu(gate_f . x^_t) * (up_f . x^_t) for every token and row f of
// the shared ffn, requantized in the same kernel: a CTA of 32 warps takes one
// 32-row block of the shared ffn (one row per warp), puts the block's a
// values in shared memory, and one warp quantizes them (as the activation
// quantization) into aq and ad, token by token.
constexpr int kSharedBlockWarps = kQBlock;
__global__ void __launch_bounds__(kSharedBlockWarps * 32) k_shared_gateup_q(SharedParams S, int ntok,
                                                                            const int8_t* __restrict__ xq,
                                                                            const float* __restrict__ xd,
                                                                            int8_t* __restrict__ aq,
                                                                            float* __restrict__ ad) {
  pdl_enter();
  __shared__ float sa[kQBlock];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int H = S.hidden, F = S.ffn;
  for (int blk = blockIdx.x; blk < F / kQBlock; blk += gridDim.x) {
    const int f = blk * kQBlock + warp;
    const int8_t* gq = S.gate_q + static_cast<size_t>(f) * H;
    const int8_t* uq = S.up_q + static_cast<size_t>(f) * H;
    const uint16_t* gd = S.gate_d + static_cast<size_t>(f) * (H / kQBlock);
    const uint16_t* ud = S.up_d + static_cast<size_t>(f) * (H / kQBlock);
    for (int t = 0; t < ntok; ++t) {
      const int8_t* xt = xq + static_cast<size_t>(t) * H;
      const float* dt = xd + static_cast<size_t>(t) * (H / kQBlock);
      float g, u;
      q8_row_dot2(gq, gd, uq, ud, H, xt, dt, lane, g, u);
      if (lane == 0) sa[warp] = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.f, expf(-g))), u);
      __syncthreads();
      if (warp == 0) quant_act_block(sa, 0, lane, aq + static_cast<size_t>(t) * F + blk * kQBlock,
                                     ad + static_cast<size_t>(t) * (F / kQBlock) + blk);
      __syncthreads();
    }
  }
}

// y[t][h] += down_h . a^_t: one warp per row h of hidden.
__global__ void __launch_bounds__(kSharedWarps * 32) k_shared_down_add(SharedParams S, int ntok, const int8_t* __restrict__ aq,
                                                                       const float* __restrict__ ad, float* __restrict__ y) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int H = S.hidden, F = S.ffn;
  const int nw = gridDim.x * kSharedWarps;
  for (int h = blockIdx.x * kSharedWarps + (threadIdx.x >> 5); h < H; h += nw) {
    const int8_t* dq = S.down_q + static_cast<size_t>(h) * F;
    const uint16_t* dd = S.down_d + static_cast<size_t>(h) * (F / kQBlock);
    for (int t = 0; t < ntok; ++t) {
      const float v = q8_row_dot(dq, dd, F, aq + static_cast<size_t>(t) * F, ad + static_cast<size_t>(t) * (F / kQBlock),
                                 lane);
      if (lane == 0) y[static_cast<size_t>(t) * H + h] = __fadd_rn(y[static_cast<size_t>(t) * H + h], v);
    }
  }
}

static unsigned rows_grid(int rows) {
  int64_t g = (static_cast<int64_t>(rows) + kSharedWarps - 1) / kSharedWarps;
  if (g > 148 * 8) g = 148 * 8;
  return static_cast<unsigned>(g);
}

int launch_quantize_weights_q8(const float* w, int64_t rows, int64_t k, int8_t* q, uint16_t* d,
                               cudaStream_t stream) {
  const int64_t nblk = rows * (k / kQBlock);
  int64_t grid = (nblk + 7) / 8;
  if (grid > 148 * 16) grid = 148 * 16;
  k_quantize_weights_q8<<<static_cast<unsigned>(grid), 256, 0, stream>>>(w, nblk, q, d);
  note_launch(MOE_K_QUANTIZE_WEIGHTS, stream);
  return check_launch("quantize_weights_q8");
}

size_t shared_ws_bytes(int hidden, int ffn, int ntok) {
  (void)hidden;
  const size_t aq = align_up(static_cast<size_t>(ntok) * ffn, 256);
  const size_t ad = align_up(sizeof(float) * static_cast<size_t>(ntok) * (ffn / kQBlock), 256);
  return aq + ad;
}

int launch_shared_ffn_add(const SharedParams& S, int ntok, const int8_t* xq, const float* xd, float* y, void* ws,
                          cudaStream_t stream) {
  unsigned char* base = static_cast<unsigned char*>(ws);
  int8_t* aq = reinterpret_cast<int8_t*>(base);
  float* ad = reinterpret_cast<float*>(base + align_up(static_cast<size_t>(ntok) * S.ffn, 256));
  launch_k(k_shared_gateup_q, dim3(static_cast<unsigned>(S.ffn / kQBlock)), dim3(kSharedBlockWarps * 32), 0, stream,
           S, ntok, xq, xd, aq, ad);
  note_launch(MOE_K_SHARED, stream);
  launch_k(k_shared_down_add, dim3(rows_grid(S.hidden)), dim3(kSharedWarps * 32), 0, stream, S, ntok,
           static_cast<const int8_t*>(aq), static_cast<const float*>(ad), y);
  note_launch(MOE_K_SHARED, stream);
  return check_launch("shared_ffn_add");
}

}  // namespace bitmoe
