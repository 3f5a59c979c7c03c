// prefill.cu -- large-batch expert FFN on the tcgen05 tensor cores (sm_100a).
//
// Parakon Runtime README, "How it works": prompt processing at large batch
// takes a GEMM path over the quantized tiles; pxq_llama README, "What's PXQ?":
// a grouped-MoE GEMM, and "Updates -- 2026-07-19": an int8 prefill tile.
//
// The (token, slot) pairs are grouped by expert and cut into tiles of up to
// kPN pairs.  A tile of the grouped GEMM is 128 weight rows x kPN pairs:
//   - A (128 x 32 per MMA): the weights' base-3 digits t = q + 1 in {0,1,2},
//     decoded in registers from the packed blocks and written straight into
//     tensor memory with tcgen05.st.  Read as e4m3, the bytes 0, 1, 2 are the
//     subnormals 0, 2^-9, 2^-8, i.e. exactly t * 2^-9, so the decoded digits
//     need no conversion at all;
//   - B (32 x kPN): each int8 activation code a = 16*h + l is split into two
//     e4m3 operands, 16*h (h in [-8, 7]) and l (in [0, 15]), both exact; two
//     MMAs accumulate t*16h and t*l into the same fp32 accumulator, which then
//     holds 2^-9 * sum(t*a) exactly (every partial sum is a multiple of 2^-9
//     below 2^4);
//   - one fp32 TMEM accumulator per 32-value sub-block (the activation scale
//     changes every 32 values); the epilogue forms sum(q*a) = 512*D - sum(a)
//     and scales it in fp32 exactly like the decode kernels: sum over
//     sub-blocks of d * sum(q*a), then the fp16 weight scale per 256-block.
// Two warps share each TMEM lane quadrant: both hold the same 32 rows, one
// decodes the first 32 digit columns and fixes up the first half of the
// pairs, the other the rest.
// Gate/up tiles hold 64 gate rows and the 64 matching up rows, so SwiGLU and
// the requantization run in the epilogue (writing the split codes of the down
// input); down tiles write each pair's rows, and a last pass combines the
// top_k slots of every token in slot order.
#include <cuda_fp8.h>

#include "bitmoe.h"
#include "common.cuh"
#include "decode.cuh"
#include "prefill.cuh"
#include "tc.cuh"

namespace bitmoe {

constexpr int kPN = 32;          // pairs per tile (MMA N)
constexpr int kPM = 128;         // weight rows per tile (MMA M)
constexpr int kPThreads = 256;   // two warps per TMEM lane quadrant
constexpr int kPHalf = kPN / 2;  // pairs fixed up by one warp of a quadrant
constexpr int kTmemCols = 256;   // A: columns [0, 64); D: [64, 64 + 4 * kPN)
constexpr int kADcol = 0;
constexpr int kDcol = 64;

struct PrefillSmem {
  uint32_t tmem_base;
  int abort;
  uint64_t bar;
  int pairs[kPN];
  alignas(128) unsigned char Bh[2][kSubPerBlock * kPN * 32];  // 16*h parts, MMA layout, 2 blocks
  alignas(128) unsigned char Bl[2][kSubPerBlock * kPN * 32];  // l parts
  alignas(16) float d[kSubPerBlock][kPN];                      // activation scales of the block
  alignas(16) float na[kSubPerBlock][kPN];                     // minus the code sums
  float xch[64][kPN + 1];                                      // gate results for the up rows
};

// Byte offset of activation code (pair n, k in [0, 32)) of sub-block s in B:
// 8-row x 16-byte core matrices, the two 16-byte halves of K 128 bytes apart,
// consecutive 8-pair groups 256 bytes apart.
__device__ __forceinline__ int b_off(int s, int n, int k) {
  return s * (kPN * 32) + (n >> 3) * 256 + (k >> 4) * 128 + (n & 7) * 16 + (k & 15);
}

// e4m3 bytes of the two parts of an activation code q = 16*h + l.
__device__ __forceinline__ void code_split(int q, uint8_t& hi, uint8_t& lo) {
  const int h = q >> 4;  // floor(q / 16), in [-8, 7]
  const int l = q & 15;
  hi = static_cast<uint8_t>(__nv_cvt_float_to_fp8(static_cast<float>(h * 16), __NV_SATFINITE, __NV_E4M3));
  lo = static_cast<uint8_t>(__nv_cvt_float_to_fp8(static_cast<float>(l), __NV_SATFINITE, __NV_E4M3));
}

// Split codes and per-32-block code sums of the gate/up input: one warp per
// 32-block.
__global__ void k_prefill_prep(DecodeParams P) {
  const int64_t nblk = static_cast<int64_t>(P.ntok) * (P.hidden / kQBlock);
  const int lane = threadIdx.x & 31;
  for (int64_t blk = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32; blk < nblk;
       blk += static_cast<int64_t>(gridDim.x) * blockDim.x / 32) {
    const int q = P.xq[blk * kQBlock + lane];
    uint8_t hi, lo;
    code_split(q, hi, lo);
    P.xh[blk * kQBlock + lane] = hi;
    P.xl[blk * kQBlock + lane] = lo;
    const int sum = __reduce_add_sync(0xffffffffu, q);
    if (lane == 0) P.xsum[blk] = sum;
  }
}

// Digit words [32*kHalf, 32*kHalf + 32) of one packed block (digit word
// 5*j + i holds level i of the four bytes of packed word j): each 16-bit lane
// keeps u * 3^i, whose high byte H_i grows by one base-3 digit per level and
// t_i = H_(i+1) - 3*H_i.  `w` holds packed words [6*kHalf, 6*kHalf + 7).
template <int kHalf>
__device__ __forceinline__ void decode_half(const uint32_t (&w)[7], uint32_t (&dg)[32]) {
#pragma unroll
  for (int jj = 0; jj < 7; ++jj) {
    const int j = 6 * kHalf + jj;
    uint32_t lo = w[jj] & 0x00FF00FFu, hi = (w[jj] >> 8) & 0x00FF00FFu, hp = 0u;
#pragma unroll
    for (int i = 0; i < 5; ++i) {
      if (j == kBlockWords - 1 && i == 4) break;
      lo *= 3u;
      hi *= 3u;
      const uint32_t hn = __byte_perm(lo, hi, 0x7351);
      const int c = 5 * j + i - 32 * kHalf;
      if (c >= 0 && c < 32) dg[c] = hn - 3u * hp;
      hp = hn;
    }
  }
}

template <bool kGU>
__global__ void __launch_bounds__(kPThreads, 2) k_prefill_mma(DecodeParams P) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  PrefillSmem& S = *reinterpret_cast<PrefillSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, half = warp >> 2;
  const int H = P.hidden, F = P.ffn, K = P.top_k;
  const int kdim = kGU ? H : F;               // reduction length
  const int nb = kdim / kBlock;
  const int m_tiles = kGU ? F / 64 : H / kPM;
  const uint32_t idesc = idesc_e4m3(kPM, kPN);

  if (warp == 0) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&S.bar, 1);
    fence_mbar_init();
    S.abort = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = S.tmem_base;
  const uint32_t tlane = tbase + (static_cast<uint32_t>(quad * 32) << 16);  // this warp's lane quadrant
  uint32_t phase = 0;

  const int n_tiles = *P.n_items * m_tiles;
  for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const Item it = P.items[tile / m_tiles];
    const int mt = tile % m_tiles;
    if (tid < kPN) S.pairs[tid] = tid < it.count ? P.pairs[it.start + tid] : -1;
    __syncthreads();
    if (it.expert < 0) {  // ids out of range: their outputs are zero
      if (tid == 0) record_status(P.status, MOE_ERR_BAD_INDEX);
      for (int n = 0; n < it.count; ++n) {
        const int pair = S.pairs[n];
        if (kGU) {
          if (tid < 64) {
            const size_t f = static_cast<size_t>(pair) * F + 64 * mt + tid;
            P.aqh[f] = 0;
            P.aql[f] = 0;
            if ((tid & 31) == 0) {
              P.ad[static_cast<size_t>(pair) * (F / kQBlock) + (64 * mt + tid) / kQBlock] = 0.f;
              P.asum[static_cast<size_t>(pair) * (F / kQBlock) + (64 * mt + tid) / kQBlock] = 0;
            }
          }
        } else if (tid < kPM) {
          P.ye[static_cast<size_t>(pair) * H + kPM * mt + tid] = 0.f;
        }
      }
      __syncthreads();
      continue;
    }
    // this thread's weight row: matrix, panel and row within the panel
    const uint32_t* trits;
    const uint16_t* scales;
    size_t panel;
    if (kGU) {
      const bool up = quad >= 2;
      trits = up ? P.up_trits : P.gate_trits;
      scales = up ? P.up_scales : P.gate_scales;
      panel = (static_cast<size_t>(it.expert) * F + 64 * mt) / kPanel + (quad & 1);
    } else {
      trits = P.down_trits;
      scales = P.down_scales;
      panel = (static_cast<size_t>(it.expert) * H + kPM * mt) / kPanel + quad;
    }
    float y[kPHalf];
#pragma unroll
    for (int n = 0; n < kPHalf; ++n) y[n] = 0.f;

    // Gather block b's split codes of the tile's pairs into B[buf] (zeros for
    // empty pair slots); one commit group per block.
    auto gather = [&](int b, int buf) {
#pragma unroll
      for (int i = 0; i < (2 * kPN * 16) / kPThreads; ++i) {
        const int c = tid + i * kPThreads;
        const int part = c / (kPN * 16), n = (c / 16) % kPN, kc = c & 15;
        unsigned char* dst = (part ? S.Bl[buf] : S.Bh[buf]) + b_off(kc >> 1, n, (kc & 1) * 16);
        const int pair = S.pairs[n];
        if (pair >= 0) {
          const uint8_t* src = kGU ? (part ? P.xl : P.xh) + static_cast<size_t>(pair / K) * H
                                   : (part ? P.aql : P.aqh) + static_cast<size_t>(pair) * F;
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)),
                       "l"(src + b * kBlock + kc * 16)
                       : "memory");
        } else {
          *reinterpret_cast<int4*>(dst) = make_int4(0, 0, 0, 0);
        }
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    uint32_t wn[7];
    uint16_t sn;
    auto load_w = [&](int b) {
      const size_t pb = panel * nb + b;
#pragma unroll
      for (int j = 0; j < 7; ++j)
        wn[j] = ld_stream_u32(trits + (pb * kBlockWords + 6 * half + j) * kPanel + lane);
      sn = scales[pb * kPanel + lane];
    };
    gather(0, 0);
    load_w(0);
    for (int b = 0; b < nb; ++b) {
      const int buf = b & 1;
      uint32_t w[7];
#pragma unroll
      for (int j = 0; j < 7; ++j) w[j] = wn[j];
      const float sw = f16_bits_to_f32(sn);
      // prefetch block b+1 while this block is decoded, multiplied and scaled
      if (b + 1 < nb) {
        gather(b + 1, buf ^ 1);
        load_w(b + 1);
      }
      // ---- A: this warp's 32 digit columns of the rows' block
      {
        uint32_t dg[32];
        if (half == 0) decode_half<0>(w, dg);
        else decode_half<1>(w, dg);
        tmem_st32(tlane + kADcol + 32 * half, dg);
      }
      // ---- scales and code sums of block b
      if (b + 1 < nb) asm volatile("cp.async.wait_group 1;" ::: "memory");
      else asm volatile("cp.async.wait_group 0;" ::: "memory");
      {
        const int s = tid >> 5, n = tid & 31;  // kPThreads == kSubPerBlock * kPN
        const int pair = S.pairs[n];
        float dv = 0.f, av = 0.f;
        if (pair >= 0) {
          const size_t q = kGU ? static_cast<size_t>(pair / K) * (H / kQBlock) + b * kSubPerBlock + s
                               : static_cast<size_t>(pair) * (F / kQBlock) + b * kSubPerBlock + s;
          dv = kGU ? P.xd[q] : P.ad[q];
          av = static_cast<float>(kGU ? P.xsum[q] : P.asum[q]);
        }
        S.d[s][n] = dv;
        S.na[s][n] = -av;
      }
      tc_wait_st();
      fence_proxy_async_shared();
      tc_fence_before();
      __syncthreads();
      float inner[kPHalf];
#pragma unroll
      for (int n = 0; n < kPHalf; ++n) inner[n] = 0.f;
#pragma unroll
      for (int h4 = 0; h4 < 2; ++h4) {
        if (tid == 0 && !*reinterpret_cast<volatile int*>(&S.abort)) {
          tc_fence_after();
#pragma unroll
          for (int s4 = 0; s4 < 4; ++s4) {
            const int s = 4 * h4 + s4;
            const uint32_t dcol = tbase + kDcol + s4 * kPN, acol = tbase + kADcol + 8 * s;
            mma_f8_ts(dcol, acol, smem_desc(smem_u32(S.Bh[buf] + s * (kPN * 32)), 128, 256), idesc, false);
            mma_f8_ts(dcol, acol, smem_desc(smem_u32(S.Bl[buf] + s * (kPN * 32)), 128, 256), idesc, true);
          }
          mma_commit(&S.bar);
        }
        if (!*reinterpret_cast<volatile int*>(&S.abort) && !mbar_wait(&S.bar, phase & 1)) {
          S.abort = 1;
          record_status(P.status, MOE_ERR_TIMEOUT);
        }
        ++phase;
        tc_fence_after();
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) {
          const int s = 4 * h4 + s4;
          uint32_t v[16];
          tmem_ld16(tlane + kDcol + s4 * kPN + kPHalf * half, v);
          tc_wait_ld();
          const float4* dp = reinterpret_cast<const float4*>(&S.d[s][kPHalf * half]);
          const float4* ap = reinterpret_cast<const float4*>(&S.na[s][kPHalf * half]);
#pragma unroll
          for (int n4 = 0; n4 < kPHalf / 4; ++n4) {
            const float4 dd = dp[n4], aa = ap[n4];
            const float dv[4] = {dd.x, dd.y, dd.z, dd.w}, av[4] = {aa.x, aa.y, aa.z, aa.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int n = 4 * n4 + e;
              // 512 * D - sum(a) = sum(q*a), exact; then d * sum(q*a) as in the decode kernels
              const float qa = __fmaf_rn(__uint_as_float(v[n]), 512.f, av[e]);
              inner[n] = __fmaf_rn(dv[e], qa, inner[n]);
            }
          }
        }
        tc_fence_before();
        __syncthreads();
      }
#pragma unroll
      for (int n = 0; n < kPHalf; ++n) y[n] = __fmaf_rn(sw, inner[n], y[n]);
    }

    // ---- epilogue (this warp: rows 32*quad + lane, pairs kPHalf*half + n)
    const int n0 = kPHalf * half;
    if (kGU) {
      if (quad < 2) {
#pragma unroll
        for (int n = 0; n < kPHalf; ++n) S.xch[32 * quad + lane][n0 + n] = y[n];
      }
      __syncthreads();
      if (quad >= 2) {
        const int r = 32 * (quad - 2) + lane;  // f offset within the tile
        const int f = 64 * mt + r;
#pragma unroll
        for (int n = 0; n < kPHalf; ++n) {
          if (n0 + n >= it.count) break;
          const float g = S.xch[r][n0 + n];
          const float a = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.f, expf(-g))), y[n]);
          const float amax = warp_max(fabsf(a));
          const float dd = __fdiv_rn(amax, 127.f);
          int q = 0;
          if (dd != 0.f) q = max(-127, min(127, __float2int_rn(__fdiv_rn(a, dd))));
          const int pair = S.pairs[n0 + n];
          uint8_t hi, lo;
          code_split(q, hi, lo);
          P.aqh[static_cast<size_t>(pair) * F + f] = hi;
          P.aql[static_cast<size_t>(pair) * F + f] = lo;
          const int sum = __reduce_add_sync(0xffffffffu, q);
          if (lane == 0) {
            P.ad[static_cast<size_t>(pair) * (F / kQBlock) + f / kQBlock] = dd;
            P.asum[static_cast<size_t>(pair) * (F / kQBlock) + f / kQBlock] = sum;
          }
        }
      }
    } else {
      const int h = kPM * mt + 32 * quad + lane;
#pragma unroll
      for (int n = 0; n < kPHalf; ++n)
        if (n0 + n < it.count) P.ye[static_cast<size_t>(S.pairs[n0 + n]) * H + h] = y[n];
    }
    __syncthreads();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, kTmemCols);
}

// y[t] = sum_j wts[t][j] * ye[t][j], slots in order.
__global__ void k_combine(DecodeParams P) {
  const int H = P.hidden, K = P.top_k;
  const int64_t total = static_cast<int64_t>(P.ntok) * H;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / H, h = i % H;
    float y = 0.f;
    for (int j = 0; j < K; ++j) y = __fmaf_rn(P.wts[t * K + j], P.ye[(t * K + j) * H + h], y);
    P.y[i] = y;
  }
}

static size_t prefill_smem() {
  // at least 80 KB so that no more than two CTAs (2 x 256 TMEM columns) share an SM
  const size_t s = sizeof(PrefillSmem) + 1024;
  return s < 80 * 1024 ? 80 * 1024 : s;
}

int launch_prefill(const DecodeParams& P0, cudaStream_t stream) {
  DecodeParams P = P0;
  P.direct = 0;
  P.group_chunk = kPN;
  int rc = launch_group(P, stream);
  if (rc) return rc;
  static bool attrs_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attrs_done[dev]) {
    cudaFuncSetAttribute(k_prefill_mma<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
    cudaFuncSetAttribute(k_prefill_mma<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
    attrs_done[dev] = true;
  }
  int n_sm = 148;
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  const size_t smem = prefill_smem();
  k_prefill_prep<<<2 * n_sm, 256, 0, stream>>>(P);
  note_launch(MOE_K_PREFILL_PREP, stream);
  k_prefill_mma<true><<<2 * n_sm, kPThreads, smem, stream>>>(P);
  note_launch(MOE_K_PREFILL_GATEUP, stream);
  k_prefill_mma<false><<<2 * n_sm, kPThreads, smem, stream>>>(P);
  note_launch(MOE_K_PREFILL_DOWN, stream);
  k_combine<<<4 * n_sm, 256, 0, stream>>>(P);
  note_launch(MOE_K_COMBINE, stream);
  return check_launch("expert_ffn_prefill");
}

}  // namespace bitmoe
