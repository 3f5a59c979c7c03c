// quant.cu -- S0 ternary weight quantization and S1 int8 activation
// quantization (sm_100a).
#include "bitmoe.h"
#include "common.cuh"
#include "quant.cuh"

namespace bitmoe {

constexpr int kQuantWarps = 4;
constexpr int kTileStride = kBlock + 1;  // padded row of the staged tile

// ---------------------------------------------------------------------------
// S0 (Parallax 8B kappa article, "Что именно доступно": ternary routed-expert
// weights).  One warp per (panel, block): the 32 rows x 256 weights are staged
// in shared memory with coalesced loads, then lane r quantizes row r of the
// panel: s = fp16_rn(sum |w| in fp64, ascending k / 256), q = sign(w) where
// |w| >= s/2.  The digits are packed five per byte as ceil(v*256/243) and the
// 13 words of each row are written 128 contiguous bytes per warp store.
// Every lane does the same sequence of operations for its block whatever the
// grid, so the output does not depend on the launch configuration.
// With kFmt = MOE_FORMAT_SIGN the same scale is kept and the codes are 1-bit
// signs (pxq_llama README, "What's PXQ?": the PXQ1 tier): q = -1 where w < 0,
// else +1, bit 8l + i of word j set for q = +1 at weight 32j + 4i + l.
// With kFmt = MOE_FORMAT_E16 (the same README's E16-row scales) the row's
// anchor A comes from k_e16_anchors; per 16-weight block h the code
// c = clamp(rint(16 * mean|w| / A) - 1, 0, 15) goes to `codes` and the
// digits use the block scale A * (c + 1) / 16 (exact in fp32).
// ---------------------------------------------------------------------------
template <int kFmt>
__global__ void __launch_bounds__(kQuantWarps * 32)
    k_quantize_weights(const float* __restrict__ w, int64_t n_items, int k,
                       uint32_t* __restrict__ trits, uint16_t* __restrict__ scales,
                       uint32_t* __restrict__ codes, const uint16_t* __restrict__ anchors) {
  constexpr bool kSign = kFmt == MOE_FORMAT_SIGN, kE16 = kFmt == MOE_FORMAT_E16;
  extern __shared__ __align__(16) float tile_all[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float* tile = tile_all + warp * kPanel * kTileStride;
  const int nb = k / kBlock;
  for (int64_t item = static_cast<int64_t>(blockIdx.x) * kQuantWarps + warp; item < n_items;
       item += static_cast<int64_t>(gridDim.x) * kQuantWarps) {
    const int64_t p = item / nb;
    const int b = static_cast<int>(item % nb);
    for (int r = 0; r < kPanel; ++r) {
      const float4* src =
          reinterpret_cast<const float4*>(w + (p * kPanel + r) * static_cast<int64_t>(k) + b * kBlock);
      const float4 v0 = src[lane], v1 = src[lane + 32];
      float* dst = tile + r * kTileStride;
      dst[4 * lane + 0] = v0.x; dst[4 * lane + 1] = v0.y;
      dst[4 * lane + 2] = v0.z; dst[4 * lane + 3] = v0.w;
      dst[128 + 4 * lane + 0] = v1.x; dst[128 + 4 * lane + 1] = v1.y;
      dst[128 + 4 * lane + 2] = v1.z; dst[128 + 4 * lane + 3] = v1.w;
    }
    __syncwarp();
    const float* row = tile + lane * kTileStride;
    float half = 0.f, af = 0.f;
    uint32_t cw0 = 0, cw1 = 0;
    if constexpr (kE16) {
      af = f16_bits_to_f32(anchors[p * kPanel + lane]);
      const double a = static_cast<double>(af);
      for (int h = 0; h < kBlock / 16; ++h) {
        double sum = 0.0;
        for (int i = 0; i < 16; ++i) sum = __dadd_rn(sum, fabs(static_cast<double>(row[16 * h + i])));
        int c = 0;
        if (a > 0.0) {
          const double t = rint(16.0 * (sum / 16.0) / a) - 1.0;
          c = t < 0.0 ? 0 : (t > 15.0 ? 15 : static_cast<int>(t));
        }
        if (h < 8) cw0 |= static_cast<uint32_t>(c) << (4 * h);
        else cw1 |= static_cast<uint32_t>(c) << (4 * (h - 8));
      }
      codes[(item * kE16Words + 0) * kPanel + lane] = cw0;
      codes[(item * kE16Words + 1) * kPanel + lane] = cw1;
    } else {
      double sum = 0.0;
      for (int kk = 0; kk < kBlock; ++kk) sum = __dadd_rn(sum, fabs(static_cast<double>(row[kk])));
      const uint16_t s = f64_to_f16_rn(sum * (1.0 / 256.0));
      half = 0.5f * f16_bits_to_f32(s);
      scales[item * kPanel + lane] = s;
    }
    if constexpr (kSign) {
#pragma unroll 1
      for (int j = 0; j < kSignWords; ++j) {
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int l = 0; l < 4; ++l)
            if (!(row[32 * j + 4 * i + l] < 0.f)) word |= 1u << (8 * l + i);
        trits[(item * kSignWords + j) * kPanel + lane] = word;
      }
    } else {
#pragma unroll 1
      for (int j = 0; j < kBlockWords; ++j) {
        uint32_t word = 0;
#pragma unroll
        for (int l = 0; l < 4; ++l) {
          int v = 0;
#pragma unroll
          for (int i = 0; i < 5; ++i) {
            const int kk = 20 * j + 4 * i + l;
            int t = 1;  // pad digit: weight 0
            if (kk < kBlock) {
              const float x = row[kk];
              float hk = half;
              if constexpr (kE16) {  // the block scale of weight kk, exact in fp32
                const int hb = kk >> 4;
                const uint32_t c = ((hb < 8 ? cw0 : cw1) >> (4 * (hb & 7))) & 15u;
                hk = 0.5f * (af * static_cast<float>(c + 1)) * 0.0625f;
              }
              if (fabsf(x) >= hk && x != 0.f) t = x > 0.f ? 2 : 0;
            }
            v = 3 * v + t;
          }
          const uint32_t u = static_cast<uint32_t>((v * 256 + 242) / 243);
          word |= u << (8 * l);
        }
        trits[(item * kBlockWords + j) * kPanel + lane] = word;
      }
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// S1 (Parakon Runtime README, "How it works"; pxq_llama README, "PXQ vs MXFP4":
// one scale per 32 values).  One warp per 32-value block: d = amax/127 and
// q = clamp(rint(x/d), -127, 127) with IEEE divisions; d = 0 gives q = 0.
// ---------------------------------------------------------------------------
__global__ void k_quant_act_q8(const float* __restrict__ x, int64_t nblk, int8_t* __restrict__ xq,
                               float* __restrict__ xd) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t blk = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       blk < nblk; blk += warps)
    quant_act_block(x, blk, lane, xq, xd);
}

// The same quantization, four 32-blocks per warp at a time: lane l holds
// values 4l..4l+3 of the four blocks (one 16-byte load), the eight lanes of a
// block reduce its amax, and each lane stores its four codes as one word.
__global__ void k_quant_act_q8_x4(const float* __restrict__ x, int64_t ngroups, int8_t* __restrict__ xq,
                                  float* __restrict__ xd) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); g < ngroups;
       g += warps) {
    const float4 v = reinterpret_cast<const float4*>(x + g * 4 * kQBlock)[lane];
    float am = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
    for (int m = 1; m <= 4; m <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, m));
    const float d = __fdiv_rn(am, 127.f);
    uint32_t packed = 0;
    if (d != 0.f) {
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int q = max(-127, min(127, __float2int_rn(__fdiv_rn(vv[i], d))));
        packed |= (static_cast<uint32_t>(q) & 0xffu) << (8 * i);
      }
    }
    reinterpret_cast<uint32_t*>(xq + g * 4 * kQBlock)[lane] = packed;
    if ((lane & 7) == 0) xd[g * 4 + (lane >> 3)] = d;
  }
}

// Anchors of the two-level scales: one warp per row, lane l taking the
// 16-weight blocks l, l+32, ...; A = fp16_RNE(max over the blocks of
// mean|w|), each mean summed in fp64 in ascending order.
__global__ void k_e16_anchors(const float* __restrict__ w, int64_t rows, int k, uint16_t* __restrict__ anchors) {
  const int lane = threadIdx.x & 31;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += nw) {
    const float* wr = w + r * k;
    double mmax = 0.0;
    for (int h = lane; h < k / 16; h += 32) {
      const float4* src = reinterpret_cast<const float4*>(wr + 16 * h);
      double sum = 0.0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 v = src[q];
        sum = __dadd_rn(sum, fabs(static_cast<double>(v.x)));
        sum = __dadd_rn(sum, fabs(static_cast<double>(v.y)));
        sum = __dadd_rn(sum, fabs(static_cast<double>(v.z)));
        sum = __dadd_rn(sum, fabs(static_cast<double>(v.w)));
      }
      const double m = sum / 16.0;
      if (m > mmax) mmax = m;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const double v = __shfl_xor_sync(0xffffffffu, mmax, o);
      if (v > mmax) mmax = v;
    }
    if (lane == 0) anchors[r] = f64_to_f16_rn(mmax);
  }
}

template <int kFmt>
static int launch_quantize(const float* w, int64_t rows, int64_t k, uint32_t* trits, uint16_t* scales,
                           uint32_t* codes, const uint16_t* anchors, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(kQuantWarps) * kPanel * kTileStride * sizeof(float);
  cudaFuncSetAttribute(k_quantize_weights<kFmt>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  const int64_t n_items = rows / kPanel * (k / kBlock);
  int64_t grid = (n_items + kQuantWarps - 1) / kQuantWarps;
  if (grid > 148 * 16) grid = 148 * 16;
  k_quantize_weights<kFmt><<<static_cast<unsigned>(grid), kQuantWarps * 32, smem, stream>>>(
      w, n_items, static_cast<int>(k), trits, scales, codes, anchors);
  note_launch(MOE_K_QUANTIZE_WEIGHTS, stream);
  return check_launch("quantize_weights");
}

int launch_quantize_weights(const float* w, int64_t rows, int64_t k, uint32_t* trits,
                            uint16_t* scales, cudaStream_t stream, bool sign) {
  if (sign) return launch_quantize<MOE_FORMAT_SIGN>(w, rows, k, trits, scales, nullptr, nullptr, stream);
  return launch_quantize<MOE_FORMAT_TERNARY>(w, rows, k, trits, scales, nullptr, nullptr, stream);
}

int launch_quantize_weights_e16(const float* w, int64_t rows, int64_t k, uint32_t* trits, uint32_t* codes,
                                uint16_t* anchors, cudaStream_t stream) {
  int64_t grid = (rows + 7) / 8;
  if (grid > 148 * 16) grid = 148 * 16;
  k_e16_anchors<<<static_cast<unsigned>(grid), 256, 0, stream>>>(w, rows, static_cast<int>(k), anchors);
  note_launch(MOE_K_QUANTIZE_WEIGHTS, stream);
  if (int rc = check_launch("e16_anchors")) return rc;
  return launch_quantize<MOE_FORMAT_E16>(w, rows, k, trits, nullptr, codes, anchors, stream);
}

int launch_quant_act_q8(const float* x, int64_t ntok, int k, int8_t* xq, float* xd,
                        cudaStream_t stream) {
  const int64_t nblk = ntok * (k / kQBlock);
  const int warps_per_cta = 8;
  const bool vec = k % (4 * kQBlock) == 0 && reinterpret_cast<uintptr_t>(x) % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(xq) % 4 == 0;
  const int64_t units = vec ? nblk / 4 : nblk;
  int64_t grid = (units + warps_per_cta - 1) / warps_per_cta;
  if (grid > 148 * 8) grid = 148 * 8;
  if (vec)
    launch_k(k_quant_act_q8_x4, dim3(static_cast<unsigned>(grid)), dim3(warps_per_cta * 32), 0, stream, x, units, xq,
             xd);
  else
    launch_k(k_quant_act_q8, dim3(static_cast<unsigned>(grid)), dim3(warps_per_cta * 32), 0, stream, x, nblk, xq, xd);
  note_launch(MOE_K_QUANT_ACT, stream);
  return check_launch("quant_act_q8");
}

}  // namespace bitmoe
