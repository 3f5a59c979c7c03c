// router.cu -- S2: router logits in a fixed fp32 order and top-k softmax
// (sm_100a).
//
// llama-modchip page, "Key highlights": every top-k expert of a token is
// evaluated, with no dropping.  The routing decision is an integer result
// taken on fp32 logits, so the evaluation order of each logit is fixed: 32
// partial sums (lane l accumulates fused multiply-adds over k = l, l+32, ...
// ascending) followed by xor-butterfly additions at distances 16, 8, 4, 2, 1.
#include <atomic>
#include "bitmoe.h"
#include "common.cuh"
#include "ptx.cuh"
#include "quant.cuh"
#include "router.cuh"
#include "topk.cuh"

namespace bitmoe {

// One warp per (token, expert) logit.  The router matrix rows are read once per
// token by one warp each (coalesced 128-byte loads); many warps run per SM.
__global__ void k_router_logits(const float* __restrict__ x, const float* __restrict__ wr, int ntok,
                                int H, int E, float* __restrict__ logits) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t total = static_cast<int64_t>(ntok) * E;
  for (int64_t pair = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       pair < total; pair += nw) {
    const int t = static_cast<int>(pair / E), e = static_cast<int>(pair % E);
    const float* xr = x + static_cast<int64_t>(t) * H;
    const float* wrow = wr + static_cast<int64_t>(e) * H;
    float p = 0.f;
#pragma unroll 8
    for (int k = lane; k < H; k += 32) p = __fmaf_rn(__ldg(wrow + k), __ldg(xr + k), p);
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) p = __fadd_rn(p, __shfl_xor_sync(0xffffffffu, p, m));
    if (lane == 0) logits[pair] = p;
  }
}

// Many tokens: a CTA computes a tile of 16 tokens x 16 experts (4 experts
// when there are few tokens, so that more CTAs share the work).  The
// evaluation order is the same as above: the chain of lane l (k = l, l+32, ...
// ascending) is kept by lane l of a warp for each (token, expert) pair of the
// warp's micro-tile, and the 32 chains are combined by the same xor
// butterfly.  x and router rows are staged through shared memory in 256-wide
// chunks (double-buffered cp.async), so each row is read from L2 once per tile
// instead of once per logit.
constexpr int kRtT = 16, kRtKC = 256;
// Few tokens: the tiles have little arithmetic per chunk, so the chunks are
// 1024 wide (two stages of 80 KB) to cut the number of copy round trips.
constexpr int kRtKCWide = 1024;

// kW warps per CTA, kWE of them along the experts (kW / kWE along the
// tokens); a lane holds a micro-tile of kMT tokens x kME experts: the CTA
// tile is (kW / kWE) * kMT tokens x kWE * kME experts.
// With xq non-null the CTAs also quantize x to int8 32-blocks, the blocks
// dealt round-robin over all warps of the grid (as k_quant_act_q8 does).
template <int kW, int kWE, int kMT, int kME, int kKC>
__global__ void __launch_bounds__(kW * 32) k_router_logits_tiled(const float* __restrict__ x,
                                                                 const float* __restrict__ wr, int ntok, int H,
                                                                 int E, float* __restrict__ logits,
                                                                 int8_t* __restrict__ xq, float* __restrict__ xd) {
  pdl_enter();
  constexpr int kRtMT = kMT, kRtME = kME, kRtE = kWE * kME, kRtT = (kW / kWE) * kMT;
  extern __shared__ __align__(16) float rsm[];
  float* xs = rsm;                        // [2][kRtT][kKC]
  float* ws = rsm + 2 * kRtT * kKC;     // [2][kRtE][kKC]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blockIdx.x * kRtT, e0 = blockIdx.y * kRtE;
  const int wt = (warp / kWE) * kRtMT;    // warp's first token in the tile
  const int we = (warp % kWE) * kRtME;    // warp's first expert in the tile
  const int nchunk = H / kKC;
  auto stage = [&](int ch, int buf) {
    // (kRtT + kRtE) rows x kKC floats in chunks of 16 bytes
    for (int c = tid; c < (kRtT + kRtE) * (kKC / 4); c += kW * 32) {
      const int row = c / (kKC / 4), q = c % (kKC / 4);
      const bool isx = row < kRtT;
      const int r = isx ? row : row - kRtT;
      const int g = isx ? t0 + r : e0 + r;
      float* dst = (isx ? xs + (buf * kRtT + r) * kKC : ws + (buf * kRtE + r) * kKC) + q * 4;
      if (g < (isx ? ntok : E)) {
        const float* src = (isx ? x : wr) + static_cast<int64_t>(g) * H + ch * kKC + q * 4;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
      } else {
        *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  float acc[kRtMT][kRtME];
#pragma unroll
  for (int i = 0; i < kRtMT; ++i)
#pragma unroll
    for (int j = 0; j < kRtME; ++j) acc[i][j] = 0.f;
  stage(0, 0);
  if (xq) {
    const int64_t nblk = static_cast<int64_t>(ntok) * (H / kQBlock);
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * gridDim.y * kW;
    for (int64_t blk = (static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x) * kW + warp; blk < nblk;
         blk += nwarps)
      quant_act_block(x, blk, lane, xq, xd);
  }
  for (int ch = 0; ch < nchunk; ++ch) {
    const int buf = ch & 1;
    if (ch + 1 < nchunk) {
      stage(ch + 1, buf ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const float* xb = xs + (buf * kRtT + wt) * kKC;
    const float* wb = ws + (buf * kRtE + we) * kKC;
#pragma unroll 2
    for (int k = lane; k < kKC; k += 32) {
      float xv[kRtMT], wv[kRtME];
#pragma unroll
      for (int i = 0; i < kRtMT; ++i) xv[i] = xb[i * kKC + k];
#pragma unroll
      for (int j = 0; j < kRtME; ++j) wv[j] = wb[j * kKC + k];
#pragma unroll
      for (int i = 0; i < kRtMT; ++i)
#pragma unroll
        for (int j = 0; j < kRtME; ++j) acc[i][j] = __fmaf_rn(wv[j], xv[i], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < kRtMT; ++i) {
#pragma unroll
    for (int j = 0; j < kRtME; ++j) {
      float p = acc[i][j];
#pragma unroll
      for (int m = 16; m >= 1; m >>= 1) p = __fadd_rn(p, __shfl_xor_sync(0xffffffffu, p, m));
      const int t = t0 + wt + i, e = e0 + we + j;
      if (lane == 0 && t < ntok && e < E) logits[static_cast<int64_t>(t) * E + e] = p;
    }
  }
}


// One warp per token: the token's logits in registers (kPer per lane), then
// the top-k and the softmax of warp_topk_softmax.
template <int kPer>
__global__ void k_topk_softmax(const float* __restrict__ logits, int ntok, int E, int K,
                               int32_t* __restrict__ idx, float* __restrict__ wts) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= ntok) return;
  uint32_t key[kPer];
  uint32_t need = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane + 32 * i;
    key[i] = 0u;
    if (e < E) {
      key[i] = f32_key(logits[static_cast<int64_t>(t) * E + e]);
      need |= 1u << i;
    }
  }
  int my_e;
  float w;
  warp_topk_softmax<kPer>(key, need, K, lane, my_e, w);
  if (lane < K) {
    idx[static_cast<int64_t>(t) * K + lane] = my_e;
    wts[static_cast<int64_t>(t) * K + lane] = w;
  }
}

template <int kWE, int kMT, int kME, int kKC = kRtKC, int kW = 8>
static void launch_tiled(const float* x, const float* wr, int ntok, int H, int E, float* logits,
                         cudaStream_t stream, int8_t* xq = nullptr, float* xd = nullptr) {
  auto kern = k_router_logits_tiled<kW, kWE, kMT, kME, kKC>;
  constexpr int kT = (kW / kWE) * kMT;
  const size_t smem = sizeof(float) * 2 * (kT + kWE * kME) * kKC;
  static std::atomic<bool> attr_done[64];  // the attribute call is idempotent
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev].load(std::memory_order_relaxed)) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    attr_done[dev].store(true, std::memory_order_relaxed);
  }
  const dim3 grid((ntok + kT - 1) / kT, (E + kWE * kME - 1) / (kWE * kME));
  launch_k(kern, grid, dim3(kW * 32), smem, stream, x, wr, ntok, H, E, logits, xq, xd);
}

int launch_router_logits(const float* x, const float* wr, int ntok, int H, int E, float* logits,
                         cudaStream_t stream) {
  if (H % kRtKC != 0) {
    const int64_t total = static_cast<int64_t>(ntok) * E;
    int64_t grid = (total + 7) / 8;
    if (grid > 148 * 16) grid = 148 * 16;
    launch_k(k_router_logits, dim3(static_cast<unsigned>(grid)), dim3(256), 0, stream, x, wr, ntok, H, E, logits);
  } else if (ntok >= 4 * kRtT && E >= 64) {
    // 32 tokens x 32 experts on 16 warps: an 8 x 8 micro-tile per lane (16
    // shared-memory loads per 64 fused multiply-adds), each staged row used
    // by 32 logits
    launch_tiled<4, 8, 8, kRtKC, 16>(x, wr, ntok, H, E, logits, stream);
  } else if (ntok >= 4 * kRtT) {
    launch_tiled<4, 8, 4>(x, wr, ntok, H, E, logits, stream);  // 16 x 16 tiles
  } else if (H % kRtKCWide == 0) {
    launch_tiled<2, 4, 2, kRtKCWide>(x, wr, ntok, H, E, logits, stream);  // 16 x 4 tiles, wide chunks
  } else {
    launch_tiled<2, 4, 2>(x, wr, ntok, H, E, logits, stream);  // 16 x 4 tiles
  }
  note_launch(MOE_K_ROUTER_LOGITS, stream);
  return check_launch("router_logits");
}

int launch_route_topk(const float* x, const float* wr, int ntok, int H, int E, int K, int32_t* idx,
                      float* wts, float* logits, cudaStream_t stream) {
  int rc = launch_router_logits(x, wr, ntok, H, E, logits, stream);
  if (rc) return rc;
  const dim3 grid((ntok + 3) / 4), block(128);
  if (E <= 128)
    launch_k(k_topk_softmax<4>, grid, block, 0, stream, logits, ntok, E, K, idx, wts);
  else if (E <= 256)
    launch_k(k_topk_softmax<8>, grid, block, 0, stream, logits, ntok, E, K, idx, wts);
  else
    launch_k(k_topk_softmax<32>, grid, block, 0, stream, logits, ntok, E, K, idx, wts);
  note_launch(MOE_K_TOPK, stream);
  return check_launch("route_topk");
}

bool router_quant_small_ok(int ntok, int H) { return ntok <= kMaxDecodeTokens && H % kRtKC == 0; }

int launch_router_quant_small(const float* x, const float* wr, int ntok, int H, int E, float* logits,
                              int8_t* xq, float* xd, cudaStream_t stream) {
  if (!router_quant_small_ok(ntok, H)) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "router_quant: shape");
  if (H % kRtKCWide == 0 && ntok <= kRtT)
    // one token tile: 16 x 2 tiles (all 8 warps along the tokens), so that
    // E/2 CTAs share the router rows instead of E/8
    launch_tiled<1, 2, 2, kRtKCWide>(x, wr, ntok, H, E, logits, stream, xq, xd);
  else if (H % kRtKCWide == 0)
    launch_tiled<2, 4, 2, kRtKCWide>(x, wr, ntok, H, E, logits, stream, xq, xd);  // 16 x 4 tiles, wide chunks
  else
    launch_tiled<2, 4, 2>(x, wr, ntok, H, E, logits, stream, xq, xd);
  note_launch(MOE_K_ROUTER_QUANT, stream);
  return check_launch("router_quant");
}

}  // namespace bitmoe
