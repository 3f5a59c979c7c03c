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
// The activations of a tile are laid out once per (group, 256-block) in HBM
// exactly as shared memory holds them (split codes in the MMA's core-matrix
// layout, then the scales and code sums of the group's pairs): for gate/up by a
// gather pass over x^, for down by the gate/up epilogue itself.  One bulk copy
// (TMA) then brings each block's 18 KB into a shared-memory stage.
// The kernel is persistent (one CTA per SM) and warp-specialized: decode
// warps write the digits of block i while the MMAs of block i-1 run and the
// fixup warps drain the accumulators of earlier half blocks; mbarriers pass
// each stage along (digits: 2 TMEM stages, activations: 3 shared-memory
// stages, accumulators: 2 TMEM stages of half a block).
// Gate/up tiles hold 64 gate rows and the 64 matching up rows, so SwiGLU and
// the requantization run in the epilogue; down tiles write each pair's rows,
// and a last pass combines the top_k slots of every token in slot order.
#include <atomic>
#include <cuda_fp8.h>

#include "bitmoe.h"
#include "common.cuh"
#include "decode.cuh"
#include "digits.cuh"
#include "prefill.cuh"
#include "tc.cuh"

namespace bitmoe {

constexpr int kPN = 64;           // pairs per tile (MMA N)
constexpr int kPM = 128;          // weight rows per tile (MMA M)
// Warp roles of a CTA (one CTA per SM, persistent over the tiles):
constexpr int kWDec = 0;          // warps 0-3: decode the digits into TMEM (thread = row)
constexpr int kWFix = 4;          // warps 4-19: accumulator fixup and epilogue (thread = row,
constexpr int kFixWarps = 16;     //   warp 4 + 4f + q: rows of quadrant q, pairs [8f, 8f + 8))
constexpr int kFixPairs = kPN / (kFixWarps / 4);
constexpr int kWGat = 20;         // warp 20: lane 0 brings the activation blocks in (bulk copies)
constexpr int kWMma = 21;         // warp 21: lane 0 issues the MMAs
constexpr int kPThreads = 22 * 32;
constexpr int kAStages = 2;       // digit stages in TMEM, 64 columns each
constexpr int kBStages = 3;       // code / scale stages in shared memory
constexpr int kQSub = 2;          // sub-blocks per accumulator stage (a quarter of a block)
constexpr int kDStages = 3;       // accumulator stages in flight
constexpr int kTmemCols = 512;
constexpr int kAcol = 0;          // A stage a: columns [64a, 64a + 64)
constexpr int kDSub = kPN;        // D columns per sub-block: one fp32 accumulator per pair
constexpr int kDcol = 128;        // D stage d: columns [128 + kQSub*kDSub*d, 128 + kQSub*kDSub*(d+1))
static_assert(kDcol + kDStages * kQSub * kDSub <= 512, "tensor memory columns");

// One 256-wide block of a tile's activations, identical in HBM and in shared
// memory: the split codes in the MMA layout, then per sub-block the pairs'
// scales and code sums (negated).
struct BStage {
  unsigned char codes[2][kSubPerBlock * kPN * 32];  // 16*h parts, then l parts, MMA layout
  float d[kSubPerBlock][kPN];                        // activation scales
  float nsa[kSubPerBlock][kPN];                      // minus the code sums
};
constexpr int kBTile = static_cast<int>(sizeof(BStage));
static_assert(kBTile % 128 == 0, "bulk copies of whole stages");

struct PrefillSmem {
  uint64_t a_full[kAStages], a_empty[kAStages];
  uint64_t b_full[kBStages], b_empty[kBStages], s_empty[kBStages];
  uint64_t d_full[kDStages], d_empty[kDStages];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  alignas(128) BStage st[kBStages];
  float xch[64][kPN + 1];  // gate results for the up rows
};

// Byte offset of activation code (pair n, k in [0, 32)) of sub-block s in one
// part's B operand: 8-row x 16-byte core matrices, the two 16-byte halves of K
// 128 bytes apart, consecutive 8-pair groups 256 bytes apart.
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

// The gate/up activation blocks of every group: thread (n, s) of a CTA
// splits the 32 codes of sub-block s of pair n's token and adds them up.
__global__ void __launch_bounds__(kPN * kSubPerBlock) k_prefill_gather(DecodeParams P) {
  pdl_enter();
  const int H = P.hidden, K = P.top_k, nb = H / kBlock;
  const int64_t work = static_cast<int64_t>(*P.n_items) * nb;
  const int n = threadIdx.x >> 3, s = threadIdx.x & 7;
  for (int64_t w = blockIdx.x; w < work; w += gridDim.x) {
    const Item it = P.items[w / nb];
    const int b = static_cast<int>(w % nb);
    BStage* dst = reinterpret_cast<BStage*>(P.bgu) + w;
    const int pair = n < it.count ? P.pairs[it.start + n] : -1;
    int4 c[2] = {make_int4(0, 0, 0, 0), make_int4(0, 0, 0, 0)};
    float d = 0.f;
    if (pair >= 0) {
      const int8_t* src = P.xq + static_cast<size_t>(pair / K) * H + b * kBlock + s * kQBlock;
      c[0] = *reinterpret_cast<const int4*>(src);
      c[1] = *reinterpret_cast<const int4*>(src + 16);
      d = P.xd[static_cast<size_t>(pair / K) * (H / kQBlock) + b * kSubPerBlock + s];
    }
    int sum = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int8_t* q = reinterpret_cast<const int8_t*>(&c[h]);
      int4 hv, lv;
      uint8_t* hb = reinterpret_cast<uint8_t*>(&hv);
      uint8_t* lb = reinterpret_cast<uint8_t*>(&lv);
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        code_split(q[k], hb[k], lb[k]);
        sum += q[k];
      }
      *reinterpret_cast<int4*>(dst->codes[0] + b_off(s, n, 16 * h)) = hv;
      *reinterpret_cast<int4*>(dst->codes[1] + b_off(s, n, 16 * h)) = lv;
    }
    dst->d[s][n] = d;
    dst->nsa[s][n] = -static_cast<float>(sum);
  }
}

// Two independent fp32 fused multiply-adds, round to nearest each, in one
// packed instruction: (r0, r1) = (a0*b0 + c0, a1*b1 + c1).
__device__ __forceinline__ void fma2(float& r0, float& r1, float a0, float a1, float b0, float b1, float c0,
                                     float c1) {
  asm("{\n\t.reg .b64 a, b, c, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 c, {%6, %7};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(r0), "=f"(r1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

// Tile t of the grouped GEMM: item (expert, pairs) and 128-row tile index.
struct TileInfo {
  Item it;
  int mt;
};
__device__ __forceinline__ TileInfo tile_info(const DecodeParams& P, int t, int m_tiles) {
  TileInfo T;
  T.it = P.items[t / m_tiles];
  T.mt = t % m_tiles;
  return T;
}

// The row of this thread in a tile (quadrant q, lane): matrix and panel.
template <bool kGU>
__device__ __forceinline__ void tile_row(const DecodeParams& P, const TileInfo& T, int q, const uint32_t*& trits,
                                         const uint16_t*& scales, size_t& panel) {
  if (kGU) {
    const bool up = q >= 2;
    trits = up ? P.up_trits : P.gate_trits;
    scales = up ? P.up_scales : P.gate_scales;
    panel = (static_cast<size_t>(T.it.expert) * P.ffn + 64 * T.mt) / kPanel + (q & 1);
  } else {
    trits = P.down_trits;
    scales = P.down_scales;
    panel = (static_cast<size_t>(T.it.expert) * P.hidden + kPM * T.mt) / kPanel + q;
  }
}

// The gate/up epilogue's output for pairs [n0, n0 + kFixPairs) at ffn row f of a
// tile: each lane (32 consecutive f, one 32-block) requantizes the SwiGLU
// values a[] (absent pairs and bad groups: zeros) and writes the split codes,
// scale and code sum into the down input's activation block of the group.
__device__ __forceinline__ void write_down_codes(const DecodeParams& P, int mt, int item, int r, int n0,
                                                 const float* a, int count, int lane) {
  const int F = P.ffn;
  const int f = 64 * mt + r;
  const int bf = f / kBlock, sub = (f % kBlock) / kQBlock;
  BStage* dst = reinterpret_cast<BStage*>(P.bdn) + static_cast<size_t>(item) * (F / kBlock) + bf;
#pragma unroll
  for (int n = 0; n < kFixPairs; ++n) {
    const int np = n0 + n;
    float dd = 0.f;
    int qq = 0;
    if (a != nullptr && np < count) {
      const float amax = warp_max(fabsf(a[n]));
      dd = __fdiv_rn(amax, 127.f);
      if (dd != 0.f) qq = max(-127, min(127, __float2int_rn(__fdiv_rn(a[n], dd))));
    }
    uint8_t hi, lo;
    code_split(qq, hi, lo);
    dst->codes[0][b_off(sub, np, lane)] = hi;
    dst->codes[1][b_off(sub, np, lane)] = lo;
    const int sum = __reduce_add_sync(0xffffffffu, qq);
    if (lane == 0) {
      dst->d[sub][np] = dd;
      dst->nsa[sub][np] = -static_cast<float>(sum);
    }
  }
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, PrefillSmem& S, int32_t* status) {
  if (*reinterpret_cast<volatile int*>(&S.abort)) return false;
  if (mbar_wait_sleep(bar, parity)) return true;
  *reinterpret_cast<volatile int*>(&S.abort) = 1;
  record_status(status, MOE_ERR_TIMEOUT);
  return false;
}

template <bool kGU>
__global__ void __launch_bounds__(kPThreads, 1) k_prefill_mma(DecodeParams P) {
  pdl_enter();
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  PrefillSmem& S = *reinterpret_cast<PrefillSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = P.hidden, F = P.ffn;
  const int kdim = kGU ? H : F;               // reduction length
  const int nb = kdim / kBlock;
  const int m_tiles = kGU ? F / 64 : H / kPM;
  const int n_tiles = *P.n_items * m_tiles;

  if (warp == 0) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < kAStages; ++i) { mbar_init(&S.a_full[i], 4); mbar_init(&S.a_empty[i], 1); }
    for (int i = 0; i < kBStages; ++i) {
      mbar_init(&S.b_full[i], 1);
      mbar_init(&S.b_empty[i], 1);
      mbar_init(&S.s_empty[i], kFixWarps);
    }
    for (int i = 0; i < kDStages; ++i) { mbar_init(&S.d_full[i], 1); mbar_init(&S.d_empty[i], kFixWarps); }
    mbar_init(&S.mma_done, 1);
    fence_mbar_init();
    S.abort = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = S.tmem_base;

  if (warp >= kWDec && warp < kWFix) {
    // ------------------------------------------------ decode: digits -> TMEM
    const uint32_t tlane = tbase + (static_cast<uint32_t>(warp * 32) << 16);
    // the CTA's sequence of (tile, block): the next one's words are loaded
    // while the current one is decoded
    int t = blockIdx.x, b = 0;
    auto skip_bad = [&]() {
      while (t < n_tiles && P.items[t / m_tiles].expert < 0) t += gridDim.x;
    };
    auto load = [&](int tt, int bb, uint32_t (&w)[kBlockWords]) {
      const TileInfo T = tile_info(P, tt, m_tiles);
      const uint32_t* trits;
      const uint16_t* scales;
      size_t panel;
      tile_row<kGU>(P, T, warp, trits, scales, panel);
      const size_t pb = panel * nb + bb;
#pragma unroll
      for (int j = 0; j < kBlockWords; ++j) w[j] = ld_stream_u32(trits + (pb * kBlockWords + j) * kPanel + lane);
    };
    skip_bad();
    uint32_t wn[kBlockWords];
    if (t < n_tiles) load(t, 0, wn);
    for (uint32_t i = 0; t < n_tiles; ++i) {
      uint32_t w[kBlockWords];
#pragma unroll
      for (int j = 0; j < kBlockWords; ++j) w[j] = wn[j];
      // advance to the next (tile, block) and start its loads
      int tn = t, bn = b + 1;
      if (bn == nb) {
        bn = 0;
        tn += gridDim.x;
        while (tn < n_tiles && P.items[tn / m_tiles].expert < 0) tn += gridDim.x;
      }
      if (tn < n_tiles) load(tn, bn, wn);
      const int a = i % kAStages;
      if (!wait_or_abort(&S.a_empty[a], ((i / kAStages) & 1u) ^ 1u, S, P.status)) break;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t w7[7], dg[32];
#pragma unroll
        for (int jj = 0; jj < 7; ++jj) w7[jj] = w[6 * h + jj];
        if (h == 0) digit_half<0>(w7, dg);
        else digit_half<1>(w7, dg);
        tmem_st32(tlane + kAcol + 64 * a + 32 * h, dg);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.a_full[a]);
      t = tn;
      b = bn;
    }
  } else if (warp < kWGat) {
    // ------------------------------------------------ fixup and epilogue
    const int q = (warp - kWFix) & 3, f16 = (warp - kWFix) >> 2;  // lane quadrant, pair group
    const uint32_t tlane = tbase + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x) {
      const TileInfo T = tile_info(P, t, m_tiles);
      // pair n of the tile: lane n & 31 of mp[n >> 5]
      const int mp0 = lane < T.it.count ? P.pairs[T.it.start + lane] : -1;
      const int mp1 = lane + 32 < T.it.count ? P.pairs[T.it.start + lane + 32] : -1;
      auto pair_at = [&](int n) { return __shfl_sync(0xffffffffu, n < 32 ? mp0 : mp1, n & 31); };
      if (T.it.expert < 0) {  // ids out of range: their outputs are zero
        if (warp == kWFix && lane == 0) record_status(P.status, MOE_ERR_BAD_INDEX);
        if (kGU) {
          if (q >= 2) write_down_codes(P, T.mt, t / m_tiles, 32 * (q - 2) + lane, kFixPairs * f16, nullptr, 0, lane);
        } else {
          for (int n = kFixPairs * f16; n < kFixPairs * f16 + kFixPairs; ++n) {
            const int pair = pair_at(n);
            if (n < T.it.count) P.ye[static_cast<size_t>(pair) * H + kPM * T.mt + 32 * q + lane] = 0.f;
          }
        }
        continue;
      }
      const uint32_t* trits;
      const uint16_t* scales;
      size_t panel;
      tile_row<kGU>(P, T, q, trits, scales, panel);
      float y[kFixPairs];
#pragma unroll
      for (int n = 0; n < kFixPairs; ++n) y[n] = 0.f;
      uint16_t sn = scales[(panel * nb) * kPanel + lane];
      bool ok = true;
      for (int b = 0; b < nb && ok; ++b, ++i) {
        const float sw = f16_bits_to_f32(sn);
        if (b + 1 < nb) sn = scales[(panel * nb + b + 1) * kPanel + lane];
        const int bs = i % kBStages;
        if (!wait_or_abort(&S.b_full[bs], (i / kBStages) & 1u, S, P.status)) { ok = false; break; }
        float inner[kFixPairs];
#pragma unroll
        for (int n = 0; n < kFixPairs; ++n) inner[n] = 0.f;
#pragma unroll 1
        for (int h = 0; h < kSubPerBlock / kQSub; ++h) {
          const uint32_t j2 = (kSubPerBlock / kQSub) * i + h;
          const int ds = j2 % kDStages;
          if (!wait_or_abort(&S.d_full[ds], (j2 / kDStages) & 1u, S, P.status)) { ok = false; break; }
          tc_fence_after();
          // kQSub sub-blocks x this warp's pairs, one sub-block at a time; the
          // stage goes back to the MMA once the last one is in registers
#pragma unroll
          for (int s2 = 0; s2 < kQSub; ++s2) {
            uint32_t v[kFixPairs];
            tmem_ld16(tlane + kDcol + kQSub * kDSub * ds + kDSub * s2 + kFixPairs * f16, v);
            tc_wait_ld();
            if (s2 == kQSub - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&S.d_empty[ds]);
            }
            const int s = kQSub * h + s2;
            const float4* dp = reinterpret_cast<const float4*>(&S.st[bs].d[s][kFixPairs * f16]);
            const float4* ap = reinterpret_cast<const float4*>(&S.st[bs].nsa[s][kFixPairs * f16]);
#pragma unroll
            for (int n4 = 0; n4 < kFixPairs / 4; ++n4) {
              const float4 dd = dp[n4], aa = ap[n4];
              // 512 * D - sum(a) = sum(q*a), exact; then d * sum(q*a) as in the decode kernels
              const uint32_t* vv = &v[4 * n4];
              float q0, q1, q2, q3;
              fma2(q0, q1, __uint_as_float(vv[0]), __uint_as_float(vv[1]), 512.f, 512.f, aa.x, aa.y);
              fma2(q2, q3, __uint_as_float(vv[2]), __uint_as_float(vv[3]), 512.f, 512.f, aa.z, aa.w);
              fma2(inner[4 * n4], inner[4 * n4 + 1], dd.x, dd.y, q0, q1, inner[4 * n4], inner[4 * n4 + 1]);
              fma2(inner[4 * n4 + 2], inner[4 * n4 + 3], dd.z, dd.w, q2, q3, inner[4 * n4 + 2], inner[4 * n4 + 3]);
            }
          }
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.s_empty[bs]);
#pragma unroll
        for (int n = 0; n < kFixPairs; ++n) y[n] = __fmaf_rn(sw, inner[n], y[n]);
      }
      if (!ok) break;
      // ---- epilogue (rows 32*q + lane, pairs [kFixPairs*f16, kFixPairs*f16 + kFixPairs))
      if (kGU) {
        if (q < 2) {
#pragma unroll
          for (int n = 0; n < kFixPairs; ++n) S.xch[32 * q + lane][kFixPairs * f16 + n] = y[n];
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kFixWarps * 32) : "memory");
        if (q >= 2) {
          const int r = 32 * (q - 2) + lane;  // f offset within the tile
          float a[kFixPairs];
#pragma unroll
          for (int n = 0; n < kFixPairs; ++n) {
            const float g = S.xch[r][kFixPairs * f16 + n];
            a[n] = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.f, expf(-g))), y[n]);
          }
          write_down_codes(P, T.mt, t / m_tiles, r, kFixPairs * f16, a, T.it.count, lane);
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kFixWarps * 32) : "memory");
      } else {
        const int hrow = kPM * T.mt + 32 * q + lane;
#pragma unroll
        for (int n = 0; n < kFixPairs; ++n) {
          const int np = kFixPairs * f16 + n;
          const int pair = pair_at(np);
          if (np < T.it.count) P.ye[static_cast<size_t>(pair) * H + hrow] = y[n];
        }
      }
    }
  } else if (warp == kWGat && lane == 0) {
    // ------------------------------------------------ activation blocks: one bulk copy each
    const unsigned char* src = kGU ? P.bgu : P.bdn;
    const uint64_t pol = policy_evict_last();  // each block serves all the group's row tiles
    uint32_t i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x) {
      const int item = t / m_tiles;
      if (P.items[item].expert < 0) continue;
      bool ok = true;
      for (int b = 0; b < nb; ++b, ++i) {
        const int bs = i % kBStages;
        const uint32_t par = ((i / kBStages) & 1u) ^ 1u;
        if (!wait_or_abort(&S.b_empty[bs], par, S, P.status) || !wait_or_abort(&S.s_empty[bs], par, S, P.status)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&S.b_full[bs], kBTile);
        bulk_g2s(&S.st[bs], src + (static_cast<size_t>(item) * nb + b) * kBTile, kBTile, &S.b_full[bs], pol);
      }
      if (!ok) break;
    }
  } else if (warp == kWMma && lane == 0) {
    // ------------------------------------------------ MMA issue
    const uint32_t idesc = idesc_e4m3(kPM, kPN);
    uint32_t i = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      if (P.items[t / m_tiles].expert < 0) continue;
      for (int b = 0; b < nb; ++b, ++i) {
        const int a = i % kAStages, bs = i % kBStages;
        if (!wait_or_abort(&S.a_full[a], (i / kAStages) & 1u, S, P.status) ||
            !wait_or_abort(&S.b_full[bs], (i / kBStages) & 1u, S, P.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t bdesc0 = smem_desc(smem_u32(S.st[bs].codes[0]), 128, 256);
        const uint64_t bdesc1 = smem_desc(smem_u32(S.st[bs].codes[1]), 128, 256);
        for (int h = 0; h < kSubPerBlock / kQSub; ++h) {
          const uint32_t j2 = (kSubPerBlock / kQSub) * i + h;
          const int ds = j2 % kDStages;
          if (!wait_or_abort(&S.d_empty[ds], ((j2 / kDStages) & 1u) ^ 1u, S, P.status)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int s2 = 0; s2 < kQSub; ++s2) {
            const int s = kQSub * h + s2;
            // start address field (bits 0-13, address >> 4) advanced by the sub-block's offset
            const uint64_t off = static_cast<uint64_t>((s * kPN * 32) >> 4);
            const uint32_t dcol = tbase + kDcol + kQSub * kDSub * ds + kDSub * s2, acol = tbase + kAcol + 64 * a + 8 * s;
            mma_f8_ts(dcol, acol, bdesc0 + off, idesc, false);
            mma_f8_ts(dcol, acol, bdesc1 + off, idesc, true);
          }
          mma_commit(&S.d_full[ds]);
        }
        if (!ok) break;
        mma_commit(&S.a_empty[a]);
        mma_commit(&S.b_empty[bs]);
      }
    }
    // every MMA has completed before the columns are released
    mma_commit(&S.mma_done);
    if (!mbar_wait(&S.mma_done, 0)) record_status(P.status, MOE_ERR_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, kTmemCols);
}

// y[t] = sum_j wts[t][j] * ye[t][j], slots in order; four h per thread
// (16-byte loads and stores; hidden is a multiple of 256).
__global__ void k_combine(DecodeParams P) {
  pdl_enter();
  const int H = P.hidden, K = P.top_k, H4 = H / 4;
  const int64_t total = static_cast<int64_t>(P.ntok) * H4;
  const float4* ye = reinterpret_cast<const float4*>(P.ye);
  float4* y = reinterpret_cast<float4*>(P.y);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / H4, h4 = i % H4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < K; ++j) {
      const float w = P.wts[t * K + j];
      const float4 v = __ldcs(ye + (t * K + j) * H4 + h4);
      acc.x = __fmaf_rn(w, v.x, acc.x);
      acc.y = __fmaf_rn(w, v.y, acc.y);
      acc.z = __fmaf_rn(w, v.z, acc.z);
      acc.w = __fmaf_rn(w, v.w, acc.w);
    }
    y[i] = acc;
  }
}

static size_t prefill_smem() {
  // more than half of the SM's shared memory, so that one CTA (holding all 512
  // TMEM columns) runs per SM
  const size_t s = sizeof(PrefillSmem) + 1024;
  return s < 120 * 1024 ? 120 * 1024 : s;
}

size_t prefill_block_bytes() { return kBTile; }
int prefill_group_pairs() { return kPN; }

int launch_prefill(const DecodeParams& P0, cudaStream_t stream) {
  DecodeParams P = P0;
  P.direct = 0;
  P.group_chunk = kPN;
  int rc = launch_group(P, stream);
  if (rc) return rc;
  static std::atomic<bool> attrs_done[64];  // the attribute calls are idempotent
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attrs_done[dev].load(std::memory_order_relaxed)) {
    cudaFuncSetAttribute(k_prefill_mma<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
    cudaFuncSetAttribute(k_prefill_mma<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
    attrs_done[dev].store(true, std::memory_order_relaxed);
  }
  int n_sm = 148;
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  const size_t smem = prefill_smem();
  launch_k(k_prefill_gather, dim3(4 * n_sm), dim3(kPN * kSubPerBlock), 0, stream, P);
  note_launch(MOE_K_PREFILL_GATHER, stream);
  launch_k(k_prefill_mma<true>, dim3(n_sm), dim3(kPThreads), smem, stream, P);
  note_launch(MOE_K_PREFILL_GATEUP, stream);
  launch_k(k_prefill_mma<false>, dim3(n_sm), dim3(kPThreads), smem, stream, P);
  note_launch(MOE_K_PREFILL_DOWN, stream);
  launch_k(k_combine, dim3(4 * n_sm), dim3(256), 0, stream, P);
  note_launch(MOE_K_COMBINE, stream);
  return check_launch("expert_ffn_prefill");
}

}  // namespace bitmoe
