// router.cu -- S2: router logits in a fixed fp32 order and top-k softmax
// (sm_100a).
//
// llama-modchip page, "Key highlights": every top-k expert of a token is
// evaluated, with no dropping.  The routing decision is an integer result
// taken on fp32 logits, so the evaluation order of each logit is fixed: 32
// partial sums (lane l accumulates fused multiply-adds over k = l, l+32, ...
// ascending) followed by xor-butterfly additions at distances 16, 8, 4, 2, 1.
#include "bitmoe.h"
#include "common.cuh"
#include "ptx.cuh"
#include "router.cuh"

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

// kWE warps along the experts (8 / kWE along the tokens); a lane holds a
// micro-tile of kMT tokens x kME experts: the CTA tile is 16 tokens x
// kWE*kME experts.
template <int kWE, int kMT, int kME>
__global__ void __launch_bounds__(256) k_router_logits_tiled(const float* __restrict__ x,
                                                             const float* __restrict__ wr, int ntok, int H,
                                                             int E, float* __restrict__ logits) {
  pdl_enter();
  constexpr int kRtMT = kMT, kRtME = kME, kRtE = kWE * kME;
  static_assert((8 / kWE) * kMT == kRtT, "16 tokens per tile");
  extern __shared__ __align__(16) float rsm[];
  float* xs = rsm;                        // [2][kRtT][kRtKC]
  float* ws = rsm + 2 * kRtT * kRtKC;     // [2][kRtE][kRtKC]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blockIdx.x * kRtT, e0 = blockIdx.y * kRtE;
  const int wt = (warp / kWE) * kRtMT;    // warp's first token in the tile
  const int we = (warp % kWE) * kRtME;    // warp's first expert in the tile
  const int nchunk = H / kRtKC;
  auto stage = [&](int ch, int buf) {
    // (kRtT + kRtE) rows x 256 floats = 2048 chunks of 16 bytes, 8 per thread
    for (int c = tid; c < (kRtT + kRtE) * (kRtKC / 4); c += 256) {
      const int row = c / (kRtKC / 4), q = c % (kRtKC / 4);
      const bool isx = row < kRtT;
      const int r = isx ? row : row - kRtT;
      const int g = isx ? t0 + r : e0 + r;
      float* dst = (isx ? xs + (buf * kRtT + r) * kRtKC : ws + (buf * kRtE + r) * kRtKC) + q * 4;
      if (g < (isx ? ntok : E)) {
        const float* src = (isx ? x : wr) + static_cast<int64_t>(g) * H + ch * kRtKC + q * 4;
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
  for (int ch = 0; ch < nchunk; ++ch) {
    const int buf = ch & 1;
    if (ch + 1 < nchunk) {
      stage(ch + 1, buf ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const float* xb = xs + (buf * kRtT + wt) * kRtKC;
    const float* wb = ws + (buf * kRtE + we) * kRtKC;
#pragma unroll 2
    for (int k = lane; k < kRtKC; k += 32) {
      float xv[kRtMT], wv[kRtME];
#pragma unroll
      for (int i = 0; i < kRtMT; ++i) xv[i] = xb[i * kRtKC + k];
#pragma unroll
      for (int j = 0; j < kRtME; ++j) wv[j] = wb[j * kRtKC + k];
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

// One warp per token: top-k by (logit descending, id ascending), then
// w_i = exp(l_i - l_0) / sum_j exp(l_j - l_0) in fp32, summed in rank order.
__global__ void k_topk_softmax(const float* __restrict__ logits, int ntok, int E, int K,
                               int32_t* __restrict__ idx, float* __restrict__ wts) {
  pdl_enter();
  __shared__ float sel_v[4][kMaxTopK];
  __shared__ int sel_e[4][kMaxTopK];
  __shared__ float lgs[4][kMaxExperts];  // the token's logits, read from L2 once
  const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
  const int t = blockIdx.x * 4 + wl;
  if (t >= ntok) return;
  for (int e = lane; e < E; e += 32) lgs[wl][e] = logits[static_cast<int64_t>(t) * E + e];
  __syncwarp();
  const float* lg = lgs[wl];
  uint32_t used = 0;  // bit i: element lane + 32*i already chosen
  for (int r = 0; r < K; ++r) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
    for (int i = 0; i * 32 + lane < E; ++i) {
      if (used & (1u << i)) continue;
      const int e = i * 32 + lane;
      const float v = lg[e];
      if (v > bv || (v == bv && e < be)) { bv = v; be = e; }
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, m);
      const int oe = __shfl_xor_sync(0xffffffffu, be, m);
      if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
    }
    if ((be & 31) == lane) used |= 1u << (be >> 5);
    if (lane == 0) { sel_v[wl][r] = bv; sel_e[wl][r] = be; }
  }
  __syncwarp();
  if (lane == 0) {
    const float l0 = sel_v[wl][0];
    float ex[kMaxTopK];
    float den = 0.f;
    for (int r = 0; r < K; ++r) {
      ex[r] = expf(__fsub_rn(sel_v[wl][r], l0));
      den = __fadd_rn(den, ex[r]);
    }
    for (int r = 0; r < K; ++r) {
      idx[static_cast<int64_t>(t) * K + r] = sel_e[wl][r];
      wts[static_cast<int64_t>(t) * K + r] = __fdiv_rn(ex[r], den);
    }
  }
}

template <int kWE, int kMT, int kME>
static void launch_tiled(const float* x, const float* wr, int ntok, int H, int E, float* logits,
                         cudaStream_t stream) {
  auto kern = k_router_logits_tiled<kWE, kMT, kME>;
  const size_t smem = sizeof(float) * 2 * (kRtT + kWE * kME) * kRtKC;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    attr_done[dev] = true;
  }
  const dim3 grid((ntok + kRtT - 1) / kRtT, (E + kWE * kME - 1) / (kWE * kME));
  launch_k(kern, grid, dim3(256), smem, stream, x, wr, ntok, H, E, logits);
}

int launch_router_logits(const float* x, const float* wr, int ntok, int H, int E, float* logits,
                         cudaStream_t stream) {
  if (H % kRtKC != 0) {
    const int64_t total = static_cast<int64_t>(ntok) * E;
    int64_t grid = (total + 7) / 8;
    if (grid > 148 * 16) grid = 148 * 16;
    launch_k(k_router_logits, dim3(static_cast<unsigned>(grid)), dim3(256), 0, stream, x, wr, ntok, H, E, logits);
  } else if (ntok >= 4 * kRtT) {
    launch_tiled<4, 8, 4>(x, wr, ntok, H, E, logits, stream);  // 16 x 16 tiles
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
  launch_k(k_topk_softmax, dim3((ntok + 3) / 4), dim3(128), 0, stream, logits, ntok, E, K, idx, wts);
  note_launch(MOE_K_TOPK, stream);
  return check_launch("route_topk");
}

}  // namespace bitmoe
