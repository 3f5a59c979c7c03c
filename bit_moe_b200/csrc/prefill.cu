// prefill.cu -- large-batch expert FFN on the tcgen05 tensor cores (sm_100a).
//
// Parakon Runtime README, "How it works": prompt processing at large batch
// takes a GEMM path over the quantized tiles; pxq_llama README, "What's PXQ?":
// a grouped-MoE GEMM, and "Updates -- 2026-07-19": an int8 prefill tile.
//
// The (token, slot) pairs are grouped by expert and cut into groups of up to
// kPN = 64 pairs.  A tile of the grouped GEMM is 128 weight rows x one group,
// one tcgen05.mma kind::i8 (M = 128, N = 64, K = 32) per 32-value sub-block:
//   - A (tensor memory): the weights' base-3 digits t = q + 1 in {0, 1, 2} as
//     u8, decoded in registers from the packed blocks (digits.cuh) and written
//     straight into tensor memory -- the expanded weights exist nowhere else;
//   - B (shared memory): the group's int8 activation codes as s8;
//   - D (tensor memory): int32, exact (|sum(t * a)| < 2^13).  The fixup adds
//     the integer 0x4B400000 to each sum, so that its bits read as the fp32
//     value 12582912 + sum(t * a) exactly; one fp32 subtraction of
//     m = 12582912 + sum(a) then gives sum(q * a) exactly, and the fixup
//     scales it as every decode kernel does: per block
//     inner = sum_s fma(d_s, sum_s(q * a), inner), per row and pair
//     y = fma(s_b, inner, y) over the blocks in order.
// 64-pair groups keep a fixup warp's 16 pairs (inner, y and one sub-block's
// sums) in registers; a tcgen05.mma of N = 64 costs the issue of one of N = 16
// on B200, so the grouped GEMM is bound by the fixup, not the tensor cores.
// The activations of a tile are laid out once per (group, 256-block) in HBM
// exactly as shared memory holds them (codes in the MMA's core-matrix layout,
// then the scales and m of the group's pairs): for gate/up by a gather pass
// over x^, for down by the gate/up epilogue itself.  One bulk copy (TMA) brings
// each block's 40 KB into a shared-memory stage; the weights stream through
// an 8-stage ring of bulk copies (one per 32-row panel and block).
// The kernel is persistent (one CTA per SM) and warp-specialized: decode
// warps write the digits of block i while the MMAs of block i-1 run and the
// fixup warps drain the accumulators sub-block by sub-block; mbarriers pass
// each stage along, and every wait is bounded.
// Gate/up tiles hold 64 gate rows and the 64 matching up rows, so SwiGLU and
// the requantization run in the epilogue; down tiles write each pair's rows,
// and a last pass combines the top_k slots of every token in slot order.
#include <atomic>

#include "bitmoe.h"
#include "common.cuh"
#include "decode.cuh"
#include "digits.cuh"
#include "prefill.cuh"
#include "tc.cuh"

namespace bitmoe {

constexpr int kPN = 64;           // pairs per group (MMA N)
constexpr int kPM = 128;          // weight rows per tile (MMA M)
// Warp roles of a CTA (one CTA per SM, persistent over the tiles):
constexpr int kWDec = 0;          // warps 0-3: decode the digits into TMEM (thread = row)
constexpr int kWFix = 4;          // warps 4-19: accumulator fixup and epilogue (thread = row,
constexpr int kFixWarps = 16;     //   warp 4 + 4f + q: rows of quadrant q, pairs [16f, 16f + 16))
constexpr int kFixPairs = kPN / (kFixWarps / 4);
constexpr int kWCopyW = 20;       // warp 20: lane 0 brings the weight blocks in (bulk copies)
constexpr int kWCopyB = 21;       // warp 21: lane 0 brings the activation blocks in (bulk copies)
constexpr int kWMma = 22;         // warp 22: lane 0 issues the MMAs
constexpr int kPThreads = 23 * 32;
constexpr int kWStages = 8;       // weight ring: one block of the tile's 4 panels per stage
constexpr int kAStages = 2;       // digit stages in TMEM, 64 columns each
constexpr int kBStages = 4;       // activation stages in shared memory
constexpr int kDSub = 2;          // sub-blocks per accumulator stage
constexpr int kDStages = 3;       // accumulator stages in TMEM, kDSub * kPN columns each
constexpr int kTmemCols = 512;
constexpr int kAcol = 0;          // A stage a: columns [64a, 64a + 64)
constexpr int kDcol = 128;        // D stage d: columns [128 + kDSub*kPN*d, 128 + kDSub*kPN*(d+1))
static_assert(kDcol + kDStages * kDSub * kPN <= kTmemCols, "tensor memory columns");
static_assert(kSubPerBlock % kDSub == 0, "whole sub-blocks per stage");
constexpr int kPanelBytes = kBlockWords * kPanel * 4;
constexpr uint32_t kMagic = 0x4B400000u;  // bits of 12582912.0f
constexpr float kMagicF = 12582912.0f;

// One 256-wide block of a group's activations, identical in HBM and in shared
// memory: the codes in the MMA layout, then per sub-block the pairs' scales
// and m = 12582912 + sum of the codes.
struct BStage {
  unsigned char codes[kSubPerBlock * kPN * 32];
  float d[kSubPerBlock][kPN];
  float m[kSubPerBlock][kPN];
};
constexpr int kBTile = static_cast<int>(sizeof(BStage));
static_assert(kBTile % 128 == 0, "bulk copies of whole stages");

struct PrefillSmem {
  uint64_t w_full[kWStages], w_empty[kWStages];
  uint64_t a_full[kAStages], a_empty[kAStages];
  uint64_t b_full[kBStages], b_empty[kBStages];
  uint64_t d_full[kDStages], d_empty[kDStages];
  uint64_t fx_bar[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  alignas(128) uint32_t w[kWStages][4][kBlockWords * kPanel];  // packed words, [panel][word][row]
  alignas(16) uint16_t wsc[kWStages][4][kPanel];                // fp16 block scales, [panel][row]
  alignas(16) uint32_t wc[kWStages][4][kE16Words * kPanel];     // two-level scales: 4-bit codes, [panel][word][row]
  alignas(128) BStage st[kBStages];
  alignas(128) unsigned char neg1[kPM * 32];  // A operand of all -1 (s8): D = -sum(a) before the digits' MMA
  float xch[2][64][kPN + 1];  // the tile's gate and up results, [row][pair], for the epilogue
};

// Byte offset of activation code (pair n, k in [0, 32)) of sub-block s: 8-row
// x 16-byte core matrices, the two 16-byte halves of K 128 bytes apart,
// consecutive 8-pair groups 256 bytes apart.
__device__ __forceinline__ int b_off(int s, int n, int k) {
  return s * (kPN * 32) + (n >> 3) * 256 + (k >> 4) * 128 + (n & 7) * 16 + (k & 15);
}

// The gate/up activation blocks of every group: thread (n, s) of a CTA copies
// the 32 codes of sub-block s of pair n's token and adds them up.
__global__ void __launch_bounds__(kPN * kSubPerBlock) k_prefill_gather(DecodeParams P) {
  pdl_enter();
  const int H = P.hidden, K = P.top_k, nb = H / kBlock;
  const int64_t work = static_cast<int64_t>(*P.n_items) * nb;
  const int n = threadIdx.x >> 3, s = threadIdx.x & 7;
  for (int64_t w = blockIdx.x; w < work; w += gridDim.x) {
    const Item it = P.items[w / nb];
    const int b = static_cast<int>(w % nb);
    if (!MOE_IN(w / nb, P.ntok * P.top_k / kPN + P.n_experts + 1, P.status)) continue;
    BStage* dst = reinterpret_cast<BStage*>(P.bgu) + w;
    const int pair = n < it.count && MOE_IN(it.start + n, P.ntok * P.top_k, P.status) ? P.pairs[it.start + n] : -1;
    int4 c[2] = {make_int4(0, 0, 0, 0), make_int4(0, 0, 0, 0)};
    float d = 0.f;
    if (pair >= 0 && pair_ok(P, pair)) {
      const int8_t* src = P.xq + static_cast<size_t>(pair / K) * H + b * kBlock + s * kQBlock;
      c[0] = *reinterpret_cast<const int4*>(src);
      c[1] = *reinterpret_cast<const int4*>(src + 16);
      d = P.xd[static_cast<size_t>(pair / K) * (H / kQBlock) + b * kSubPerBlock + s];
    }
    int sum = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      sum = __dp4a(c[h].x, 0x01010101, sum);
      sum = __dp4a(c[h].y, 0x01010101, sum);
      sum = __dp4a(c[h].z, 0x01010101, sum);
      sum = __dp4a(c[h].w, 0x01010101, sum);
      *reinterpret_cast<int4*>(dst->codes + b_off(s, n, 16 * h)) = c[h];
    }
    dst->d[s][n] = d;
    dst->m[s][n] = kMagicF + static_cast<float>(sum);
  }
}

// Two independent fp32 operations, round to nearest each, in one packed
// instruction: (r0, r1) = (a0*b0 + c0, a1*b1 + c1), and (a0 - b0, a1 - b1).
__device__ __forceinline__ void fma2(float& r0, float& r1, float a0, float a1, float b0, float b1, float c0,
                                     float c1) {
  asm("{\n\t.reg .b64 a, b, c, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 c, {%6, %7};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(r0), "=f"(r1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void sub2(float& r0, float& r1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "sub.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(r0), "=f"(r1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Tile t of the grouped GEMM: item (expert, pairs) and 128-row tile index.
struct TileInfo {
  Item it;
  int item, mt;
};
__device__ __forceinline__ bool tile_info(const DecodeParams& P, int t, int m_tiles, TileInfo& T) {
  T.item = t / m_tiles;
  if (T.item >= *P.n_items) return false;
  T.it = P.items[T.item];
  T.mt = t % m_tiles;
  return true;
}

// Panel p (0..3) of a tile: gate/up tiles are gate panels 2mt, 2mt+1 then up
// panels 2mt, 2mt+1 of the expert; down tiles are panels 4mt..4mt+3.
template <bool kGU>
__device__ __forceinline__ size_t tile_panel_index(const DecodeParams& P, const TileInfo& T, int p) {
  if (kGU) return static_cast<size_t>(T.it.expert) * (P.ffn / kPanel) + 2 * T.mt + (p & 1);
  return static_cast<size_t>(T.it.expert) * (P.hidden / kPanel) + 4 * T.mt + p;
}
template <bool kGU>
__device__ __forceinline__ const uint32_t* panel_trits(const DecodeParams& P, int p) {
  return kGU ? (p < 2 ? P.gate_trits : P.up_trits) : P.down_trits;
}
template <bool kGU>
__device__ __forceinline__ const uint16_t* panel_scales(const DecodeParams& P, int p) {
  return kGU ? (p < 2 ? P.gate_scales : P.up_scales) : P.down_scales;
}
template <bool kGU>
__device__ __forceinline__ const uint32_t* panel_codes(const DecodeParams& P, int p) {
  return kGU ? (p < 2 ? P.gate_codes : P.up_codes) : P.down_codes;
}
// Packed words per 256-weight block of a 32-row panel, by weight format.
__host__ __device__ constexpr int pf_words(int fmt) { return fmt == MOE_FORMAT_SIGN ? kSignWords : kBlockWords; }

// The gate/up epilogue's output for pairs [n0, n0 + kNP) at ffn row f of a
// tile: each lane (32 consecutive f, one 32-block) requantizes the SwiGLU
// values a[] (absent pairs and bad groups: zeros) and writes the codes, scale
// and m into the down input's activation block of the group.
template <bool kDbg, int kNP>
__device__ __forceinline__ void write_down_codes(const DecodeParams& P, int mt, int item, int r, int n0,
                                                 const float* a, const Item& it, int lane) {
  const int F = P.ffn;
  const int f = 64 * mt + r;
  const int bf = f / kBlock, sub = (f % kBlock) / kQBlock;
  if (!MOE_IN(item, P.ntok * P.top_k / kPN + P.n_experts + 1, P.status) || !MOE_IN(bf, F / kBlock, P.status)) return;
  BStage* dst = reinterpret_cast<BStage*>(P.bdn) + static_cast<size_t>(item) * (F / kBlock) + bf;
#pragma unroll 4
  for (int n = 0; n < kNP; ++n) {
    const int np = n0 + n;
    float dd = 0.f;
    int qq = 0;
    if (a != nullptr && np < it.count) {
      const float amax = warp_max(fabsf(a[n]));
      dd = __fdiv_rn(amax, 127.f);
      if (dd != 0.f) qq = max(-127, min(127, __float2int_rn(__fdiv_rn(a[n], dd))));
    }
    dst->codes[b_off(sub, np, lane)] = static_cast<unsigned char>(static_cast<int8_t>(qq));
    const int sum = __reduce_add_sync(0xffffffffu, qq);
    if (lane == 0) {
      dst->d[sub][np] = dd;
      dst->m[sub][np] = kMagicF + static_cast<float>(sum);
    }
    if (kDbg && np < it.count && pair_ok(P, P.pairs[it.start + np]))  // test hook: the SwiGLU codes
      P.aq[static_cast<size_t>(P.pairs[it.start + np]) * F + f] = static_cast<int8_t>(qq);
  }
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, PrefillSmem& S, int32_t* status) {
  if (*reinterpret_cast<volatile int*>(&S.abort)) return false;
  if (mbar_wait_sleep(bar, parity)) return true;
  *reinterpret_cast<volatile int*>(&S.abort) = 1;
  record_status(status, MOE_ERR_TIMEOUT);
  return false;
}

// kFmt: the weights' format (MOE_FORMAT_*); kDbg: the test hook's
// instantiation, which also writes the exact block sums.
template <int kFmt, bool kGU, bool kDbg>
__global__ void __launch_bounds__(kPThreads, 1) k_prefill_mma(DecodeParams P) {
  constexpr bool kE16 = kFmt == MOE_FORMAT_E16, kSgn = kFmt == MOE_FORMAT_SIGN;
  constexpr int kWords = pf_words(kFmt);
  pdl_enter();
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  PrefillSmem& S = *reinterpret_cast<PrefillSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = P.hidden, F = P.ffn;
  const int kdim = kGU ? H : F;               // reduction length
  const int nb = kdim / kBlock;
  const int m_tiles = kGU ? F / 64 : H / kPM;

  if (warp == 0) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    // a weight stage is free once the 4 decode warps have its words and the 16
    // fixup warps its scales
    for (int i = 0; i < kWStages; ++i) { mbar_init(&S.w_full[i], 1); mbar_init(&S.w_empty[i], 4 + kFixWarps); }
    for (int i = 0; i < kAStages; ++i) { mbar_init(&S.a_full[i], 4); mbar_init(&S.a_empty[i], 1); }
    for (int i = 0; i < kBStages; ++i) { mbar_init(&S.b_full[i], 1); mbar_init(&S.b_empty[i], 1 + kFixWarps); }
    for (int i = 0; i < kDStages; ++i) { mbar_init(&S.d_full[i], 1); mbar_init(&S.d_empty[i], kFixWarps); }
    for (int i = 0; i < 2; ++i) mbar_init(&S.fx_bar[i], kFixWarps);
    mbar_init(&S.mma_done, 1);
    fence_mbar_init();
    S.abort = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = S.tmem_base;
  for (int i = tid; i < kPM * 32 / 4; i += kPThreads) reinterpret_cast<uint32_t*>(S.neg1)[i] = 0xFFFFFFFFu;
  fence_proxy_async_shared();  // read by the tensor cores
  if (warp >= kWFix && warp < kWFix + kFixWarps) {
    // every accumulator column starts out holding the offset 0x4B400000
    const int q = (warp - kWFix) & 3, n0 = kFixPairs * ((warp - kWFix) >> 2);
    for (int c = 0; c < kDStages * kDSub; ++c)
      tmem_st16_fill(tbase + (static_cast<uint32_t>(q * 32) << 16) + kDcol + kPN * c + n0, kMagic);
    tc_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp >= kWDec && warp < kWFix) {
    // ------------------------------------------------ decode: digits -> TMEM
    const uint32_t tlane = tbase + (static_cast<uint32_t>(warp * 32) << 16);
    uint32_t wi = 0;
    TileInfo T;
    for (int t = blockIdx.x; tile_info(P, t, m_tiles, T); t += gridDim.x) {
      if (T.it.expert < 0) continue;
      bool ok = true;
      for (int b = 0; b < nb; ++b, ++wi) {
        const int ws = wi % kWStages, a = wi % kAStages;
        if (!wait_or_abort(&S.w_full[ws], (wi / kWStages) & 1u, S, P.status)) { ok = false; break; }
        uint32_t w[kWords], cw[kE16Words];
#pragma unroll
        for (int j = 0; j < kWords; ++j) w[j] = S.w[ws][warp][j * kPanel + lane];
        if (kE16) {
#pragma unroll
          for (int u = 0; u < kE16Words; ++u) cw[u] = S.wc[ws][warp][u * kPanel + lane];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.w_empty[ws]);
        if (!wait_or_abort(&S.a_empty[a], ((wi / kAStages) & 1u) ^ 1u, S, P.status)) { ok = false; break; }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // digit word c (weights 4c..4c+3 of the block) into column 32h + c
          uint32_t dg[32];
          if (kSgn) {
            // sign bits: word j holds weights 32j + 4i + l in bit 8l + i; the
            // digit byte is 2t (t = the bit), so that with the -1 MMA the sum
            // is sum((2t - 1) * a) = sum(q * a)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
#pragma unroll
              for (int i = 0; i < 8; ++i) dg[8 * jj + i] = ((w[4 * h + jj] >> i) & 0x01010101u) << 1;
          } else {
            uint32_t w7[7];
#pragma unroll
            for (int jj = 0; jj < 7; ++jj) w7[jj] = w[6 * h + jj];
            if (h == 0) digit_half<0>(w7, dg);
            else digit_half<1>(w7, dg);
            if (kE16) {
              // two-level scales: the signed byte q * (c + 1) of the weight's
              // 16-block (t * (c + 1) + 0x80 - (c + 1) stays in [0x70, 0x90]
              // per byte, so no carry crosses a byte; the xor makes it s8)
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                const int hb = (32 * h + c) >> 2;
                const uint32_t m1 = ((cw[hb >> 3] >> (4 * (hb & 7))) & 15u) + 1u;
                dg[c] = (dg[c] * m1 + (0x80u - m1) * 0x01010101u) ^ 0x80808080u;
              }
            }
          }
          tmem_st32(tlane + kAcol + 64 * a + 32 * h, dg);
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.a_full[a]);
      }
      if (!ok) break;
    }
  } else if (warp < kWFix + kFixWarps) {
    // ------------------------------------------------ fixup and epilogue
    const int q = (warp - kWFix) & 3, f = (warp - kWFix) >> 2;  // lane quadrant, pair group
    const int n0 = kFixPairs * f;
    const uint32_t tlane = tbase + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t bi = 0, si = 0, ep = 0;
    TileInfo T;
    for (int t = blockIdx.x; tile_info(P, t, m_tiles, T); t += gridDim.x) {
      if (T.it.expert < 0) {  // ids out of range: their outputs are zero
        if (warp == kWFix && lane == 0) record_status(P.status, MOE_ERR_BAD_INDEX);
        if (kGU) {
          if (q >= 2) write_down_codes<kDbg, kFixPairs>(P, T.mt, T.item, 32 * (q - 2) + lane, n0, nullptr, T.it, lane);
        } else {
          for (int n = n0; n < n0 + kFixPairs && n < T.it.count; ++n)
            if (pair_ok(P, P.pairs[T.it.start + n]))
              P.ye[static_cast<size_t>(P.pairs[T.it.start + n]) * H + kPM * T.mt + 32 * q + lane] = 0.f;
        }
        continue;
      }
      bool ok = true;
      float y[kFixPairs];
#pragma unroll
      for (int n = 0; n < kFixPairs; ++n) y[n] = 0.f;
      // two-level scales: the row's anchor A / 16 takes the place of the
      // block scale (y = sum over blocks of fma(A/16, inner, y))
      const float a16 = kE16 ? __fmul_rn(f16_bits_to_f32(panel_scales<kGU>(P, q)[tile_panel_index<kGU>(P, T, q) *
                                                                                kPanel + lane]), 0.0625f)
                             : 0.f;
      for (int b = 0; b < nb && ok; ++b, ++bi) {
        // the row's block scale from the weight stage of this block
        const int ws = bi % kWStages;
        if (!wait_or_abort(&S.w_full[ws], (bi / kWStages) & 1u, S, P.status)) { ok = false; break; }
        const float sw = kE16 ? a16 : f16_bits_to_f32(S.wsc[ws][q][lane]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.w_empty[ws]);
        const int bs = bi % kBStages;
        if (!wait_or_abort(&S.b_full[bs], (bi / kBStages) & 1u, S, P.status)) { ok = false; break; }
        float inner[kFixPairs];
#pragma unroll
        for (int n = 0; n < kFixPairs; ++n) inner[n] = 0.f;
#pragma unroll 1
        for (int h = 0; h < kSubPerBlock / kDSub; ++h, ++si) {
          const int ds = si % kDStages;
          if (!wait_or_abort(&S.d_full[ds], (si / kDStages) & 1u, S, P.status)) { ok = false; break; }
          tc_fence_after();
          // both sub-blocks' sums in one round trip to tensor memory, then
          // the stage goes back to the MMA
          uint32_t vv[kDSub][kFixPairs];
#pragma unroll
          for (int s2 = 0; s2 < kDSub; ++s2) tmem_ld16(tlane + kDcol + kDSub * kPN * ds + kPN * s2 + n0, vv[s2]);
          tc_wait_ld();
          // the stage goes back holding the offset again
#pragma unroll
          for (int s2 = 0; s2 < kDSub; ++s2) tmem_st16_fill(tlane + kDcol + kDSub * kPN * ds + kPN * s2 + n0, kMagic);
          tc_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.d_empty[ds]);
#pragma unroll
          for (int s2 = 0; s2 < kDSub; ++s2) {
            const int s = kDSub * h + s2;
            const uint32_t (&v)[kFixPairs] = vv[s2];
            const float* dp = &S.st[bs].d[s][n0];
            if (kDbg) {  // test hook: the exact block sums
#pragma unroll
              for (int e = 0; e < kFixPairs; ++e) {
                const int np = n0 + e;
                if (np >= T.it.count) continue;
                const int pair = P.pairs[T.it.start + np];
                const int isum = static_cast<int>(__fsub_rn(__uint_as_float(v[e]), kMagicF));
                const int sg = b * kSubPerBlock + s;
                if (kGU) {
                  const int fr = 64 * T.mt + 32 * (q & 1) + lane;
                  P.dbg_isum_gu[((static_cast<size_t>(pair) * 2 + (q >> 1)) * F + fr) * (H / kQBlock) + sg] = isum;
                } else {
                  const int hr = kPM * T.mt + 32 * q + lane;
                  P.dbg_isum_dn[(static_cast<size_t>(pair) * H + hr) * (F / kQBlock) + sg] = isum;
                }
              }
            }
#pragma unroll
            for (int n4 = 0; n4 < kFixPairs / 4; ++n4) {
              const float4 dd = reinterpret_cast<const float4*>(dp)[n4];
              const int nn = 4 * n4;
              // D (0x4B400000 + sum(q*a)) as fp32 minus 12582912 = sum(q*a),
              // exact; then d * sum(q*a) as in the decode kernels
              float i0, i1, i2, i3;
              sub2(i0, i1, __uint_as_float(v[nn]), __uint_as_float(v[nn + 1]), kMagicF, kMagicF);
              sub2(i2, i3, __uint_as_float(v[nn + 2]), __uint_as_float(v[nn + 3]), kMagicF, kMagicF);
              fma2(inner[nn], inner[nn + 1], dd.x, dd.y, i0, i1, inner[nn], inner[nn + 1]);
              fma2(inner[nn + 2], inner[nn + 3], dd.z, dd.w, i2, i3, inner[nn + 2], inner[nn + 3]);
            }
          }
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.b_empty[bs]);
        // y = fma(sw, inner, y) over the blocks in order
#pragma unroll
        for (int n = 0; n < kFixPairs; ++n) y[n] = __fmaf_rn(sw, inner[n], y[n]);
      }
      if (!ok) break;
      // ---- epilogue (rows 32*q + lane, pairs [n0, n0 + kFixPairs))
      if (kGU) {
        // gate rows (q < 2) and up rows (q >= 2) go to the exchange; then
        // every fixup warp takes one 32-row block of f and 8 pairs: SwiGLU
        // and the requantization of those (block, pair) columns
#pragma unroll
        for (int n = 0; n < kFixPairs; ++n) S.xch[q >> 1][32 * (q & 1) + lane][n0 + n] = y[n];
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.fx_bar[0]);
        if (!wait_or_abort(&S.fx_bar[0], ep & 1u, S, P.status)) break;
        {
          constexpr int kEpPairs = kPN * 2 / kFixWarps;  // 8 pairs per warp and row block
          const int fw = warp - kWFix;
          const int r = 32 * (fw & 1) + lane;            // f offset within the tile
          const int e0 = kEpPairs * (fw >> 1);
          // the SwiGLU value replaces g in the exchange (each entry is read
          // and written by its own thread)
#pragma unroll
          for (int n = 0; n < kEpPairs; ++n) {
            const float g = S.xch[0][r][e0 + n];
            S.xch[0][r][e0 + n] = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.f, expf(-g))), S.xch[1][r][e0 + n]);
          }
          write_down_codes<kDbg, kEpPairs>(P, T.mt, T.item, r, e0, &S.xch[0][r][e0], T.it, lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.fx_bar[1]);
        if (!wait_or_abort(&S.fx_bar[1], ep & 1u, S, P.status)) break;
        ++ep;
      } else {
        const int hrow = kPM * T.mt + 32 * q + lane;
#pragma unroll
        for (int n = 0; n < kFixPairs; ++n)
          if (n0 + n < T.it.count && pair_ok(P, P.pairs[T.it.start + n0 + n]))
            P.ye[static_cast<size_t>(P.pairs[T.it.start + n0 + n]) * H + hrow] = y[n];
      }
    }
  } else if (warp == kWCopyW && lane == 0) {
    // ------------------------------------------------ weight blocks: 4 bulk copies each
    const uint64_t pol = policy_evict_first();
    uint32_t wi = 0;
    bool ok = true;
    TileInfo T;
    for (int t = blockIdx.x; ok && tile_info(P, t, m_tiles, T); t += gridDim.x) {
      if (T.it.expert < 0) continue;
      // per block and panel: the packed words, then the fp16 block scales
      // (two-level scales: the 4-bit code words; the anchors are per row)
      constexpr uint32_t kWBytes = kWords * kPanel * 4;
      constexpr uint32_t kSBytes = kE16 ? kE16Words * kPanel * 4 : kPanel * 2;
      const uint32_t* src[4];
      const void* ssrc[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const size_t pi = tile_panel_index<kGU>(P, T, p);
        src[p] = panel_trits<kGU>(P, p) + pi * nb * kWords * kPanel;
        if (kE16) ssrc[p] = panel_codes<kGU>(P, p) + pi * nb * kE16Words * kPanel;
        else ssrc[p] = panel_scales<kGU>(P, p) + pi * nb * kPanel;
      }
      for (int b = 0; b < nb; ++b, ++wi) {
        const int ws = wi % kWStages;
        if (!wait_or_abort(&S.w_empty[ws], ((wi / kWStages) & 1u) ^ 1u, S, P.status)) { ok = false; break; }
        mbar_arrive_expect_tx(&S.w_full[ws], 4 * (kWBytes + kSBytes));
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          bulk_g2s(S.w[ws][p], src[p] + static_cast<size_t>(b) * kWords * kPanel, kWBytes, &S.w_full[ws], pol);
          void* sdst = kE16 ? static_cast<void*>(S.wc[ws][p]) : static_cast<void*>(S.wsc[ws][p]);
          bulk_g2s(sdst, static_cast<const unsigned char*>(ssrc[p]) + static_cast<size_t>(b) * kSBytes, kSBytes,
                   &S.w_full[ws], pol);
        }
      }
    }
    for (uint32_t k = wi > kWStages ? wi - kWStages : 0; k < wi; ++k)  // copies still in flight land
      if (!mbar_wait(&S.w_full[k % kWStages], (k / kWStages) & 1u)) record_status(P.status, MOE_ERR_TIMEOUT);
  } else if (warp == kWCopyB && lane == 0) {
    // ------------------------------------------------ activation blocks: one bulk copy each
    const unsigned char* src = kGU ? P.bgu : P.bdn;
    const uint64_t pol = policy_evict_last();  // each block serves all the group's row tiles
    uint32_t bi = 0;
    bool ok = true;
    TileInfo T;
    for (int t = blockIdx.x; ok && tile_info(P, t, m_tiles, T); t += gridDim.x) {
      if (T.it.expert < 0) continue;
      for (int b = 0; b < nb; ++b, ++bi) {
        const int bs = bi % kBStages;
        if (!wait_or_abort(&S.b_empty[bs], ((bi / kBStages) & 1u) ^ 1u, S, P.status)) { ok = false; break; }
        mbar_arrive_expect_tx(&S.b_full[bs], kBTile);
        bulk_g2s(&S.st[bs], src + (static_cast<size_t>(T.item) * nb + b) * kBTile, kBTile, &S.b_full[bs], pol);
      }
    }
    for (uint32_t k = bi > kBStages ? bi - kBStages : 0; k < bi; ++k)
      if (!mbar_wait(&S.b_full[k % kBStages], (k / kBStages) & 1u)) record_status(P.status, MOE_ERR_TIMEOUT);
  } else if (warp == kWMma && lane == 0) {
    // ------------------------------------------------ MMA issue
    const uint32_t idesc = idesc_i8(kPM, kPN);
    const uint32_t idesc_neg = idesc_i8(kPM, kPN, true);  // A signed
    const uint64_t ndesc = smem_desc(smem_u32(S.neg1), 128, 256);
    uint32_t bi = 0, si = 0;
    bool ok = true;
    TileInfo T;
    for (int t = blockIdx.x; ok && tile_info(P, t, m_tiles, T); t += gridDim.x) {
      if (T.it.expert < 0) continue;
      for (int b = 0; b < nb; ++b, ++bi) {
        const int a = bi % kAStages, bs = bi % kBStages;
        if (!wait_or_abort(&S.a_full[a], (bi / kAStages) & 1u, S, P.status) ||
            !wait_or_abort(&S.b_full[bs], (bi / kBStages) & 1u, S, P.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t bdesc = smem_desc(smem_u32(S.st[bs].codes), 128, 256);
        for (int h = 0; h < kSubPerBlock / kDSub; ++h, ++si) {
          const int ds = si % kDStages;
          if (!wait_or_abort(&S.d_empty[ds], ((si / kDStages) & 1u) ^ 1u, S, P.status)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int s2 = 0; s2 < kDSub; ++s2) {
            // onto the offset: -sum(a) (all -1 A operand), then sum(t * a)
            // (sign codes: sum(2t * a)); two-level scales: the signed bytes
            // q * (c + 1) in one MMA
            const int s = kDSub * h + s2;
            const uint32_t dcol = tbase + kDcol + kDSub * kPN * ds + kPN * s2;
            const uint64_t bsub = bdesc + static_cast<uint64_t>((s * kPN * 32) >> 4);
            if (kE16) {
              mma_i8_ts(dcol, tbase + kAcol + 64 * a + 8 * s, bsub, idesc_neg, true);
            } else {
              mma_i8_ss(dcol, ndesc, bsub, idesc_neg, true);
              mma_i8_ts(dcol, tbase + kAcol + 64 * a + 8 * s, bsub, idesc, true);
            }
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
// (16-byte loads and stores; hidden is a multiple of 256): CTAs take tokens,
// threads the token's float4 columns.
__global__ void k_combine(DecodeParams P) {
  pdl_enter();
  const int H4 = P.hidden / 4, K = P.top_k;
  const float4* ye = reinterpret_cast<const float4*>(P.ye);
  float4* y = reinterpret_cast<float4*>(P.y);
  for (int t = blockIdx.x; t < P.ntok; t += gridDim.x) {
    const float* wt = P.wts + static_cast<size_t>(t) * K;
    const float4* src = ye + static_cast<size_t>(t) * K * H4;
    for (int h4 = threadIdx.x; h4 < H4; h4 += blockDim.x) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
      for (int j = 0; j < K; ++j) {
        const float w = wt[j];
        const float4 v = __ldcs(src + static_cast<size_t>(j) * H4 + h4);
        acc.x = __fmaf_rn(w, v.x, acc.x);
        acc.y = __fmaf_rn(w, v.y, acc.y);
        acc.z = __fmaf_rn(w, v.z, acc.z);
        acc.w = __fmaf_rn(w, v.w, acc.w);
      }
      y[static_cast<size_t>(t) * H4 + h4] = acc;
    }
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
bool prefill_tc_supported(const DecodeParams& P) {
  return P.format == MOE_FORMAT_TERNARY || P.format == MOE_FORMAT_SIGN || P.format == MOE_FORMAT_E16;
}

// The gate/up and down GEMM launches of one weight format.
template <int kFmt>
static void launch_gemms(const DecodeParams& P, bool dbg, int dev, int n_sm, cudaStream_t stream) {
  static std::atomic<bool> attrs_done[64];  // the attribute calls are idempotent
  if (dev >= 0 && dev < 64 && !attrs_done[dev].load(std::memory_order_relaxed)) {
    cudaFuncSetAttribute(k_prefill_mma<kFmt, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
    cudaFuncSetAttribute(k_prefill_mma<kFmt, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
    cudaFuncSetAttribute(k_prefill_mma<kFmt, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
    cudaFuncSetAttribute(k_prefill_mma<kFmt, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
    attrs_done[dev].store(true, std::memory_order_relaxed);
  }
  const size_t smem = prefill_smem();
  launch_k(dbg ? k_prefill_mma<kFmt, true, true> : k_prefill_mma<kFmt, true, false>, dim3(n_sm), dim3(kPThreads), smem,
           stream, P);
  note_launch(MOE_K_PREFILL_GATEUP, stream);
  launch_k(dbg ? k_prefill_mma<kFmt, false, true> : k_prefill_mma<kFmt, false, false>, dim3(n_sm), dim3(kPThreads),
           smem, stream, P);
  note_launch(MOE_K_PREFILL_DOWN, stream);
}

int launch_prefill(const DecodeParams& P0, cudaStream_t stream) {
  DecodeParams P = P0;
  P.direct = 0;
  P.group_chunk = kPN;
  if (!prefill_tc_supported(P)) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "prefill: weight format %d", P.format);
  int rc = launch_group(P, stream);
  if (rc) return rc;
  int dev = 0;
  cudaGetDevice(&dev);
  int n_sm = 148;
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  launch_k(k_prefill_gather, dim3(4 * n_sm), dim3(kPN * kSubPerBlock), 0, stream, P);
  note_launch(MOE_K_PREFILL_GATHER, stream);
  const bool dbg = P.dbg_isum_gu != nullptr;
  if (P.format == MOE_FORMAT_SIGN) launch_gemms<MOE_FORMAT_SIGN>(P, dbg, dev, n_sm, stream);
  else if (P.format == MOE_FORMAT_E16) launch_gemms<MOE_FORMAT_E16>(P, dbg, dev, n_sm, stream);
  else launch_gemms<MOE_FORMAT_TERNARY>(P, dbg, dev, n_sm, stream);
  launch_k(k_combine, dim3(4 * n_sm), dim3(256), 0, stream, P);
  note_launch(MOE_K_COMBINE, stream);
  return check_launch("expert_ffn_prefill");
}

}  // namespace bitmoe
