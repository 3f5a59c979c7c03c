// prefill.cu -- large-batch expert FFN on the tcgen05 tensor cores (sm_100a).
//
// Parakon Runtime README, "How it works": prompt processing at large batch
// takes a GEMM path over the quantized tiles; pxq_llama README, "What's PXQ?":
// a grouped-MoE GEMM, and "Updates -- 2026-07-19": an int8 prefill tile.
//
// The (token, slot) pairs are grouped by expert and cut into tiles of up to
// kPN pairs.  A tile of the grouped GEMM is 128 weight rows x kPN pairs:
//   - A (128 x 32 per MMA): the weights' base-3 digits t = q + 1 as u8,
//     decoded in registers from the packed blocks (one thread per row) and
//     written straight into tensor memory with tcgen05.st -- the expanded
//     weights never exist in HBM or shared memory;
//   - B (32 x kPN): the pairs' int8 activation codes, gathered with cp.async
//     into the K-major core-matrix layout of shared memory;
//   - one tcgen05.mma kind::i8 per 32-value sub-block into its own int32 TMEM
//     accumulator (the activation scale changes every 32 values), read back
//     with tcgen05.ld and scaled in fp32 exactly like the decode kernels:
//     sum over sub-blocks of d * (sum t*a - sum a), then the fp16 weight
//     scale per 256-block.
// Gate/up tiles hold 64 gate rows and the 64 matching up rows, so SwiGLU and
// the int8 requantization of a run in the epilogue; down tiles write each
// pair's rows, and a last pass combines the top_k slots of every token in
// slot order.
#include "bitmoe.h"
#include "common.cuh"
#include "decode.cuh"
#include "prefill.cuh"
#include "tc.cuh"

namespace bitmoe {

constexpr int kPN = 32;          // pairs per tile (MMA N)
constexpr int kPM = 128;         // weight rows per tile (MMA M)
constexpr int kPThreads = 128;   // one thread per row
constexpr int kTmemCols = 256;   // A: columns [0, 64); D: [64, 64 + 4 * kPN)
constexpr int kADcol = 0;
constexpr int kDcol = 64;

struct PrefillSmem {
  uint32_t tmem_base;
  int abort;
  uint64_t bar;
  int pairs[kPN];
  alignas(128) unsigned char B[kSubPerBlock * kPN * 32];  // activation codes, MMA layout
  float d[kSubPerBlock][kPN];                              // activation scales
  int as[kSubPerBlock][kPN];                               // sums of the codes
  float xch[64][kPN + 1];                                  // gate results for the up rows
};

// Byte offset of activation code (pair n, k in [0, 32)) of sub-block s in B:
// 8-row x 16-byte core matrices, the two 16-byte halves of K 128 bytes apart,
// consecutive 8-pair groups 256 bytes apart.
__device__ __forceinline__ int b_off(int s, int n, int k) {
  return s * (kPN * 32) + (n >> 3) * 256 + (k >> 4) * 128 + (n & 7) * 16 + (k & 15);
}

template <bool kGU>
__global__ void __launch_bounds__(kPThreads, 1) k_prefill_mma(DecodeParams P) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  PrefillSmem& S = *reinterpret_cast<PrefillSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = P.hidden, F = P.ffn, K = P.top_k;
  const int kdim = kGU ? H : F;               // reduction length
  const int nb = kdim / kBlock;
  const int m_tiles = kGU ? F / 64 : H / kPM;
  const uint32_t idesc = idesc_i8(kPM, kPN);

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
  const uint32_t tlane = tbase + (static_cast<uint32_t>(warp * 32) << 16);  // this warp's lane quadrant
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
          for (int r = tid; r < 64; r += kPThreads) {
            P.aq[static_cast<size_t>(pair) * F + 64 * mt + r] = 0;
            if ((r & 31) == 0) P.ad[static_cast<size_t>(pair) * (F / kQBlock) + (64 * mt + r) / kQBlock] = 0.f;
          }
        } else {
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
      const bool up = warp >= 2;
      trits = up ? P.up_trits : P.gate_trits;
      scales = up ? P.up_scales : P.gate_scales;
      panel = (static_cast<size_t>(it.expert) * F + 64 * mt) / kPanel + (warp & 1);
    } else {
      trits = P.down_trits;
      scales = P.down_scales;
      panel = (static_cast<size_t>(it.expert) * H + kPM * mt) / kPanel + warp;
    }
    float y[kPN];
#pragma unroll
    for (int n = 0; n < kPN; ++n) y[n] = 0.f;

    for (int b = 0; b < nb; ++b) {
      // ---- B: gather the pairs' codes of block b (zeros for empty slots)
      for (int c = tid; c < kPN * 16; c += kPThreads) {
        const int n = c >> 4, kc = c & 15;
        unsigned char* dst = S.B + b_off(kc >> 1, n, (kc & 1) * 16);
        const int pair = S.pairs[n];
        if (pair >= 0) {
          const int8_t* row = kGU ? P.xq + static_cast<size_t>(pair / K) * H : P.aq + static_cast<size_t>(pair) * F;
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)),
                       "l"(row + b * kBlock + kc * 16)
                       : "memory");
        } else {
          *reinterpret_cast<int4*>(dst) = make_int4(0, 0, 0, 0);
        }
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      // ---- A: decode this row's block into 64 digit words (groups of 4)
      const size_t pb = panel * nb + b;
      uint32_t w[kBlockWords];
#pragma unroll
      for (int j = 0; j < kBlockWords; ++j) w[j] = ld_stream_u32(trits + (pb * kBlockWords + j) * kPanel + lane);
      const float sw = f16_bits_to_f32(scales[pb * kPanel + lane]);
      uint32_t digits[64];
#pragma unroll
      for (int j = 0; j < kBlockWords; ++j) {
        uint32_t lo = w[j] & 0x00FF00FFu, hi = (w[j] >> 8) & 0x00FF00FFu, hp = 0u;
#pragma unroll
        for (int i = 0; i < 5; ++i) {
          if (j == kBlockWords - 1 && i == 4) break;
          lo *= 3u;
          hi *= 3u;
          const uint32_t hn = __byte_perm(lo, hi, 0x7351);
          digits[5 * j + i] = hn - 3u * hp;
          hp = hn;
        }
      }
      tmem_st64(tlane + kADcol, digits);
      // ---- scales and code sums of block b
      asm volatile("cp.async.wait_group 0;" ::: "memory");
      __syncthreads();
      for (int q = tid; q < kSubPerBlock * kPN; q += kPThreads) {
        const int s = q / kPN, n = q % kPN;
        const int pair = S.pairs[n];
        float dv = 0.f;
        int sum = 0;
        if (pair >= 0) {
          dv = kGU ? P.xd[static_cast<size_t>(pair / K) * (H / kQBlock) + b * kSubPerBlock + s]
                   : P.ad[static_cast<size_t>(pair) * (F / kQBlock) + b * kSubPerBlock + s];
          const int4 lo4 = *reinterpret_cast<const int4*>(S.B + b_off(s, n, 0));
          const int4 hi4 = *reinterpret_cast<const int4*>(S.B + b_off(s, n, 16));
          sum = __dp4a(lo4.x, 0x01010101, sum); sum = __dp4a(lo4.y, 0x01010101, sum);
          sum = __dp4a(lo4.z, 0x01010101, sum); sum = __dp4a(lo4.w, 0x01010101, sum);
          sum = __dp4a(hi4.x, 0x01010101, sum); sum = __dp4a(hi4.y, 0x01010101, sum);
          sum = __dp4a(hi4.z, 0x01010101, sum); sum = __dp4a(hi4.w, 0x01010101, sum);
        }
        S.d[s][n] = dv;
        S.as[s][n] = sum;
      }
      tc_wait_st();
      fence_proxy_async_shared();
      tc_fence_before();
      __syncthreads();
      float inner[kPN];
#pragma unroll
      for (int n = 0; n < kPN; ++n) inner[n] = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        if (tid == 0 && !*reinterpret_cast<volatile int*>(&S.abort)) {
          tc_fence_after();
#pragma unroll
          for (int s4 = 0; s4 < 4; ++s4) {
            const int s = 4 * half + s4;
            mma_i8_ts(tbase + kDcol + s4 * kPN, tbase + kADcol + 8 * s,
                      smem_desc(smem_u32(S.B + s * (kPN * 32)), 128, 256), idesc, false);
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
          const int s = 4 * half + s4;
          uint32_t v[32];
          tmem_ld32(tlane + kDcol + s4 * kPN, v);
          tc_wait_ld();
#pragma unroll
          for (int n = 0; n < kPN; ++n)
            inner[n] = __fmaf_rn(S.d[s][n], static_cast<float>(static_cast<int>(v[n]) - S.as[s][n]), inner[n]);
        }
        tc_fence_before();
        __syncthreads();
      }
#pragma unroll
      for (int n = 0; n < kPN; ++n) y[n] = __fmaf_rn(sw, inner[n], y[n]);
    }

    // ---- epilogue
    if (kGU) {
      if (warp < 2) {
#pragma unroll
        for (int n = 0; n < kPN; ++n) S.xch[tid][n] = y[n];
      }
      __syncthreads();
      if (warp >= 2) {
        const int r = tid - 64;               // f offset within the tile
        const int f = 64 * mt + r;
#pragma unroll
        for (int n = 0; n < kPN; ++n) {
          if (n >= it.count) break;
          const float g = S.xch[r][n];
          const float a = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.f, expf(-g))), y[n]);
          const float amax = warp_max(fabsf(a));
          const float dd = __fdiv_rn(amax, 127.f);
          int q = 0;
          if (dd != 0.f) q = max(-127, min(127, __float2int_rn(__fdiv_rn(a, dd))));
          const int pair = S.pairs[n];
          P.aq[static_cast<size_t>(pair) * F + f] = static_cast<int8_t>(q);
          if (lane == 0) P.ad[static_cast<size_t>(pair) * (F / kQBlock) + f / kQBlock] = dd;
        }
      }
    } else {
      const int h = kPM * mt + tid;
#pragma unroll
      for (int n = 0; n < kPN; ++n)
        if (n < it.count) P.ye[static_cast<size_t>(S.pairs[n]) * H + h] = y[n];
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
  k_prefill_mma<true><<<2 * n_sm, kPThreads, smem, stream>>>(P);
  note_launch(MOE_K_PREFILL_GATEUP, stream);
  k_prefill_mma<false><<<2 * n_sm, kPThreads, smem, stream>>>(P);
  note_launch(MOE_K_PREFILL_DOWN, stream);
  k_combine<<<4 * n_sm, 256, 0, stream>>>(P);
  note_launch(MOE_K_COMBINE, stream);
  return check_launch("expert_ffn_prefill");
}

}  // namespace bitmoe
