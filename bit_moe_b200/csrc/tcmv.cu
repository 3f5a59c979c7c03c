// tcmv.cu -- grouped decode mat-vecs of the expert FFN on the tcgen05 tensor
// cores (sm_100a): the gate+up mat-vec with the SwiGLU and int8
// requantization epilogue, and the down mat-vec with the top-k combine, for
// items of up to kChunk (token, slot) pairs routed to one expert.
//
// Parakon Runtime README, "How it works": decode multiplies the packed blocks
// in place against int8 activations; pxq_llama README, "What's PXQ?": gate/up
// fusion and a grouped-MoE path; "PXQ vs MXFP4": one fixup per 32-value
// activation block.  On B200 the dot products of a decode mat-vec need not
// cost CUDA-core instructions: the base-3 digits of a 128-row tile are
// written into tensor memory and one tcgen05.mma kind::i8 per 32-value
// sub-block multiplies them with the item's int8 codes:
//   - A (128 x 32 per MMA, tensor memory): digits t = q + 1 in {0, 1, 2} as
//     u8, decoded in registers (digits.cuh) by 8 warps, two per TMEM lane
//     quadrant, each half a block;
//   - B (32 x 16, shared memory): the item's pairs' codes as s8 (rows past
//     the item's pairs hold stale codes whose results are never read);
//   - D (128 x 16 int32, tensor memory): the exact block sums sum(t * a) of
//     every row, pair and sub-block; the fixup warps form
//     sum(q * a) = sum(t * a) - sum(a) and scale them in fp32 exactly as the
//     CUDA-core decode kernels do (ternary_dot.cuh): per block
//     inner = sum_s fma(d_s, isum_s, inner), then per row
//     chain_w = fma(s_b, inner, chain_w) over the blocks b = w mod 8 (gate/up)
//     or one chain over all blocks (down), and the gate/up chains are summed
//     in order -- so a token gives the same bits here as through the one-token
//     step or the CUDA-core kernels.
// The weights stream through an 8-stage shared-memory ring filled by bulk
// copies (one per 32-row panel and block); the activation codes of each
// unit of work are gathered by one warp into one of two buffers while the
// previous unit computes.  Warp roles (one CTA of 19 warps per SM, persistent
// over the units; every wait bounded):
//   warps 0-7  : digits -> TMEM A stages (thread = row)
//   warps 8-15 : D -> fixup, chains, epilogue (thread = row, 4 pairs a warp)
//   warp 16    : lane 0 issues the weight bulk copies
//   warp 17    : gathers the codes, scales and code sums of the item's pairs
//   warp 18    : lane 0 issues the MMAs
#include <atomic>

#include "bitmoe.h"
#include "common.cuh"
#include "decode.cuh"
#include "digits.cuh"
#include "tc.cuh"
#include "tcmv.cuh"

namespace bitmoe {

constexpr int kTP = kChunk;           // most pairs of an item
constexpr int kTN = 16;               // MMA N (the smallest for M = 128)
constexpr int kTM = 128;              // MMA M: weight rows of a tile
constexpr int kTWStages = 8;          // weight ring: one block of the tile's 4 panels per stage
constexpr int kTAStages = 3;          // digit stages in TMEM, 64 columns each
constexpr int kTDStages = 2;          // accumulator stages in TMEM, 8 sub-blocks x 16 columns
constexpr int kTAcol = 0;
constexpr int kTDcol = kTAStages * 64;
constexpr int kTDStageCols = kSubPerBlock * kTN;
constexpr int kTTmemCols = 512;
static_assert(kTDcol + kTDStages * kTDStageCols <= kTTmemCols, "tensor memory columns");
constexpr int kTFix0 = 8;             // first fixup warp
constexpr int kTFixWarps = 8;
constexpr int kTFixPairs = kTP / 2;   // pairs per fixup warp
constexpr int kTCopy = 16, kTGat = 17, kTMma = 18;
constexpr int kTThreads = 19 * 32;
constexpr int kTGatherBatch = 8;      // 16-byte code chunks a gather lane has in flight
constexpr int kPanelBlockBytes = kBlockWords * kPanel * 4;
constexpr int kTBBlock = kSubPerBlock * kTN * 32;  // B bytes of one block

struct TcSmem {
  uint64_t w_full[kTWStages], w_empty[kTWStages];
  uint64_t a_full[kTAStages], a_empty[kTAStages];
  uint64_t d_full[kTDStages], d_empty[kTDStages];
  uint64_t b_full[2], b_empty[2];
  uint64_t fx_bar[2];  // the fixup warps' two meeting points of a gate/up epilogue
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  uint32_t checks;  // checks of a bounded mbarrier wait before it gives up
  int knob;         // the wait test knob's mode
  alignas(128) uint32_t w[kTWStages][4][kBlockWords * kPanel];   // packed words, [panel][word][row]
  alignas(16) uint16_t wsc[kTWStages][4][kPanel];                 // fp16 block scales, [panel][row]
  alignas(128) unsigned char B[2][kTcMaxBlocks][kTBBlock];         // codes, MMA layout
  alignas(16) float dsc[2][kTcMaxBlocks][kSubPerBlock][kTP];      // activation scales
  alignas(16) int sa[2][kTcMaxBlocks][kSubPerBlock][kTP];         // code sums
  float xch[64][kTP + 1];                                          // gate results for the up rows
};

// Byte offset of code (pair n, k in [0, 32)) of sub-block s in a block's B:
// 8-row x 16-byte core matrices, K halves 128 bytes apart, the two 8-row
// groups 256 bytes apart, sub-blocks 512 bytes apart.
__device__ __forceinline__ int tb_off(int s, int n, int k) {
  return s * (kTN * 32) + (n >> 3) * 256 + (k >> 4) * 128 + (n & 7) * 16 + (k & 15);
}

// Unit u of the grid's work: item, 128-row tile and block phase.  Unit ks of
// a tile takes the blocks b = ks, ks + ks_n, ... (ks_n divides 8, so each unit
// holds whole gate/up chains).
struct TcUnit {
  Item it;
  int item, mt, ks, nbu;
};

__device__ __forceinline__ bool tc_unit(const DecodeParams& P, int u, int m_tiles, int ks_n, int nb, TcUnit& U) {
  const int per = m_tiles * ks_n;
  U.item = u / per;
  if (!fetch_item(P, U.item, U.it)) return false;
  const int r = u % per;
  U.mt = r / ks_n;
  U.ks = r % ks_n;
  U.nbu = (nb - U.ks + ks_n - 1) / ks_n;
  return true;
}

// Packed words of panel p (0..3) of the unit's tile at block 0.
template <bool kGU>
__device__ __forceinline__ const uint32_t* tile_panel(const DecodeParams& P, const TcUnit& U, int p, int nb) {
  size_t panel;
  const uint32_t* base;
  if (kGU) {
    base = p < 2 ? P.gate_trits : P.up_trits;
    panel = static_cast<size_t>(U.it.expert) * (P.ffn / kPanel) + 2 * U.mt + (p & 1);
  } else {
    base = P.down_trits;
    panel = static_cast<size_t>(U.it.expert) * (P.hidden / kPanel) + 4 * U.mt + p;
  }
  return base + panel * nb * kBlockWords * kPanel;
}

template <bool kGU>
__device__ __forceinline__ const uint16_t* tile_scales(const DecodeParams& P, const TcUnit& U, int p, int nb) {
  size_t panel;
  const uint16_t* base;
  if (kGU) {
    base = p < 2 ? P.gate_scales : P.up_scales;
    panel = static_cast<size_t>(U.it.expert) * (P.ffn / kPanel) + 2 * U.mt + (p & 1);
  } else {
    base = P.down_scales;
    panel = static_cast<size_t>(U.it.expert) * (P.hidden / kPanel) + 4 * U.mt + p;
  }
  return base + panel * nb * kPanel;
}

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, TcSmem& S, int32_t* status) {
  if (*reinterpret_cast<volatile int*>(&S.abort)) return false;
  if (mbar_wait_sleep(bar, parity, S.checks)) return true;
  *reinterpret_cast<volatile int*>(&S.abort) = 1;
  record_status(status, MOE_ERR_TIMEOUT);
  return false;
}

// Gather warp: the codes of the unit's pairs for its blocks into buffer buf,
// with the scales and the code sums of every (block, sub-block, pair).
template <bool kGU>
__device__ __forceinline__ void tc_gather(const DecodeParams& P, TcSmem& S, int buf, const TcUnit& U, int ks_n,
                                          int lane) {
  const int kdim = kGU ? P.hidden : P.ffn;
  const int count = U.it.count;
  // lane n < count holds pair n's row of codes and scales
  const int8_t* my_q = nullptr;
  const float* my_d = nullptr;
  if (lane < count) {
    const int pair = item_pair(P, U.it, lane);
    if (kGU) {
      const int t = pair / P.top_k;
      my_q = P.xq + static_cast<size_t>(t) * kdim;
      my_d = P.xd + static_cast<size_t>(t) * (kdim / kQBlock);
    } else {
      my_q = P.aq + static_cast<size_t>(pair) * kdim;
      my_d = P.ad + static_cast<size_t>(pair) * (kdim / kQBlock);
    }
  }
  const int total = U.nbu * count * 16;  // 16-byte chunks: (block i, pair n, sub-block s, K half)
  for (int c0 = 0; c0 < total; c0 += 32 * kTGatherBatch) {
    int4 v[kTGatherBatch];
#pragma unroll
    for (int g = 0; g < kTGatherBatch; ++g) {
      const int c = c0 + 32 * g + lane;
      const int cc = c < total ? c : 0;
      const int kh = cc & 1, s = (cc >> 1) & 7, n = (cc >> 4) % count, i = (cc >> 4) / count;
      const int b = U.ks + i * ks_n;
      const int8_t* q = reinterpret_cast<const int8_t*>(
          __shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(my_q), n));
      v[g] = make_int4(0, 0, 0, 0);
      if (c < total) v[g] = __ldcg(reinterpret_cast<const int4*>(q + b * kBlock + s * kQBlock + kh * 16));
    }
#pragma unroll
    for (int g = 0; g < kTGatherBatch; ++g) {
      const int c = c0 + 32 * g + lane;
      const int cc = c < total ? c : 0;
      const int kh = cc & 1, s = (cc >> 1) & 7, n = (cc >> 4) % count, i = (cc >> 4) / count;
      const int b = U.ks + i * ks_n;
      const float* dsrc = reinterpret_cast<const float*>(
          __shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(my_d), n));
      int sum = 0;
      sum = __dp4a(v[g].x, 0x01010101, sum);
      sum = __dp4a(v[g].y, 0x01010101, sum);
      sum = __dp4a(v[g].z, 0x01010101, sum);
      sum = __dp4a(v[g].w, 0x01010101, sum);
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);  // the two K halves are neighbouring lanes
      if (c < total) {
        *reinterpret_cast<int4*>(&S.B[buf][i][tb_off(s, n, 16 * kh)]) = v[g];
        if (kh == 0) {
          S.sa[buf][i][s][n] = sum;
          S.dsc[buf][i][s][n] = __ldcg(dsrc + b * kSubPerBlock + s);
        }
      }
    }
  }
}

// One block of the fixup for NC pairs of a fixup warp: the exact sums of its
// pairs (D columns n0 .. n0 + NC of each sub-block), the stage handed back
// to the MMA, then per pair inner = sum_s fma(d_s, sum_s(t*a) - sum_s(a), inner)
// and chain w = fma(s_b, inner, chain w).
template <int NC, int kChains, bool kDbg, bool kGU = (kChains == 8)>
__device__ __forceinline__ void fix_block(const DecodeParams& P, TcSmem& S, uint32_t dcol, int buf, int i, int n0,
                                          int nc, int w, float sw, float (&acc)[kChains][kTFixPairs],
                                          const TcUnit& U, int b, int q, int lane, uint64_t* d_empty) {
  uint32_t v[kSubPerBlock][NC];
#pragma unroll
  for (int s = 0; s < kSubPerBlock; ++s) {
    if constexpr (NC == 4) tmem_ld4(dcol + kTN * s, v[s]);
    else if constexpr (NC == 2) tmem_ld2(dcol + kTN * s, v[s]);
    else tmem_ld1(dcol + kTN * s, v[s]);
  }
  tc_wait_ld();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(d_empty);
  float inner[NC];
#pragma unroll
  for (int n = 0; n < NC; ++n) inner[n] = 0.f;
  int32_t* dbg = kGU ? P.dbg_isum_gu : P.dbg_isum_dn;
#pragma unroll
  for (int s = 0; s < kSubPerBlock; ++s) {
#pragma unroll
    for (int n = 0; n < NC; ++n) {
      const int isum = static_cast<int>(v[s][n]) - S.sa[buf][i][s][n0 + n];
      inner[n] = __fmaf_rn(S.dsc[buf][i][s][n0 + n], static_cast<float>(isum), inner[n]);
      if (kDbg && n < nc) {  // test hook: the exact block sums
        const int pair = item_pair(P, U.it, n0 + n);
        const int sg = b * kSubPerBlock + s;
        if (kGU) {
          const int f = 64 * U.mt + 32 * (q & 1) + lane;
          dbg[((static_cast<size_t>(pair) * 2 + (q >> 1)) * P.ffn + f) * (P.hidden / kQBlock) + sg] = isum;
        } else {
          const int h = kTM * U.mt + 32 * q + lane;
          dbg[(static_cast<size_t>(pair) * P.hidden + h) * (P.ffn / kQBlock) + sg] = isum;
        }
      }
    }
  }
#pragma unroll
  for (int c = 0; c < kChains; ++c)
    if (c == w) {
#pragma unroll
      for (int n = 0; n < NC; ++n) acc[c][n] = __fmaf_rn(sw, inner[n], acc[c][n]);
    }
}

// kDbg: the test hook's instantiation, which also writes the exact block sums.
template <bool kGU, bool kDbg>
__global__ void __launch_bounds__(kTThreads, 1) k_tcmv(DecodeParams P, int ks_n) {
  pdl_enter();
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  TcSmem& S = *reinterpret_cast<TcSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = P.hidden, F = P.ffn;
  const int kdim = kGU ? H : F;
  const int nb = kdim / kBlock;
  const int m_tiles = kGU ? F / 64 : H / kTM;

  if (warp == 0) {
    tmem_alloc(&S.tmem_base, kTTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    // a weight stage is free once the 8 decode warps have its words and the 8
    // fixup warps its scales
    for (int i = 0; i < kTWStages; ++i) { mbar_init(&S.w_full[i], 1); mbar_init(&S.w_empty[i], 8 + kTFixWarps); }
    for (int i = 0; i < kTAStages; ++i) { mbar_init(&S.a_full[i], 8); mbar_init(&S.a_empty[i], 1); }
    for (int i = 0; i < kTDStages; ++i) { mbar_init(&S.d_full[i], 1); mbar_init(&S.d_empty[i], kTFixWarps); }
    for (int i = 0; i < 2; ++i) { mbar_init(&S.b_full[i], 1); mbar_init(&S.b_empty[i], 1 + kTFixWarps); }
    for (int i = 0; i < 2; ++i) mbar_init(&S.fx_bar[i], kTFixWarps);
    mbar_init(&S.mma_done, 1);
    fence_mbar_init();
    S.abort = 0;
    const int32_t* knob = reinterpret_cast<const int32_t*>(P.status);
    S.knob = knob[kWsKnobMode];
    S.checks = knob[kWsKnobPolls] ? static_cast<uint32_t>(knob[kWsKnobPolls]) : (1u << 17);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = S.tmem_base;

  if (warp < kTFix0) {
    // ------------------------------------------------ digits -> TMEM
    const int q = warp & 3, hh = warp >> 2;
    const uint32_t tl = tbase + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t wi = 0, ai = 0;
    TcUnit U;
    for (int u = blockIdx.x; tc_unit(P, u, m_tiles, ks_n, nb, U); u += gridDim.x) {
      if (U.it.expert < 0) continue;
      bool ok = true;
      for (int i = 0; i < U.nbu; ++i, ++wi, ++ai) {
        const int ws = wi % kTWStages;
        if (!tc_wait(&S.w_full[ws], (wi / kTWStages) & 1u, S, P.status)) { ok = false; break; }
        uint32_t w7[7];
#pragma unroll
        for (int jj = 0; jj < 7; ++jj) w7[jj] = S.w[ws][q][(6 * hh + jj) * kPanel + lane];
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.w_empty[ws]);
        const int as = ai % kTAStages;
        if (!tc_wait(&S.a_empty[as], ((ai / kTAStages) & 1u) ^ 1u, S, P.status)) { ok = false; break; }
        uint32_t dg[32];
        if (hh == 0) digit_half<0>(w7, dg);
        else digit_half<1>(w7, dg);
        tmem_st32(tl + kTAcol + 64 * as + 32 * hh, dg);
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.a_full[as]);
      }
      if (!ok) break;
    }
  } else if (warp < kTFix0 + kTFixWarps) {
    // ------------------------------------------------ fixup, chains, epilogue
    const int q = warp & 3, hp = (warp - kTFix0) >> 2;
    const uint32_t tl = tbase + (static_cast<uint32_t>(q * 32) << 16);
    constexpr int kChains = kGU ? 8 : 1;
    uint32_t ug = 0, di = 0, wi = 0;
    TcUnit U;
    for (int u = blockIdx.x; tc_unit(P, u, m_tiles, ks_n, nb, U); u += gridDim.x) {
      const int n0 = kTFixPairs * hp;
      if (U.it.expert < 0) {  // ids out of range: their outputs are zero
        if (q == 0 && hp == 0 && lane == 0) record_status(P.status, MOE_ERR_BAD_INDEX);
        if (kGU) {
          if (q >= 2) {
            for (int n = n0; n < n0 + kTFixPairs && n < U.it.count; ++n) {
              const int pair = item_pair(P, U.it, n);
              if (!pair_ok(P, pair)) continue;
              P.aq[static_cast<size_t>(pair) * F + 64 * U.mt + 32 * (q - 2) + lane] = 0;
              if (lane == 0) P.ad[static_cast<size_t>(pair) * (F / kQBlock) + 2 * U.mt + (q - 2)] = 0.f;
            }
          }
        } else {
          for (int n = n0; n < n0 + kTFixPairs && n < U.it.count; ++n)
            if (pair_ok(P, item_pair(P, U.it, n)))
              P.ye[static_cast<size_t>(item_pair(P, U.it, n)) * H + kTM * U.mt + 32 * q + lane] = 0.f;
          __threadfence();
          __syncwarp();
          for (int n = n0; n < n0 + kTFixPairs && n < U.it.count; ++n)
            arrive_and_combine(P, item_pair(P, U.it, n), 4 * U.mt + q, lane);
        }
        continue;
      }
      const int buf = ug & 1;
      if (!tc_wait(&S.b_full[buf], (ug >> 1) & 1u, S, P.status)) break;
      const int nc = min(kTFixPairs, U.it.count - n0);  // this warp's pairs of the item
      float acc[kChains][kTFixPairs];
#pragma unroll
      for (int w = 0; w < kChains; ++w)
#pragma unroll
        for (int n = 0; n < kTFixPairs; ++n) acc[w][n] = 0.f;
      bool ok = true;
      for (int i = 0; i < U.nbu; ++i, ++di, ++wi) {
        const int b = U.ks + i * ks_n;
        // the row's block scale from the weight stage of this block
        const int ws = wi % kTWStages;
        if (!tc_wait(&S.w_full[ws], (wi / kTWStages) & 1u, S, P.status)) { ok = false; break; }
        const float sw = f16_bits_to_f32(S.wsc[ws][q][lane]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.w_empty[ws]);
        const int ds = di % kTDStages;
        if (!tc_wait(&S.d_full[ds], (di / kTDStages) & 1u, S, P.status)) { ok = false; break; }
        tc_fence_after();
        // only this warp's pairs of the item (a warp with none just passes the stage on)
        const uint32_t dcol = tl + kTDcol + kTDStageCols * ds + n0;
        const int w = kGU ? (b & 7) : 0;
        if (nc >= 3) fix_block<4, kChains, kDbg>(P, S, dcol, buf, i, n0, nc, w, sw, acc, U, b, q, lane, &S.d_empty[ds]);
        else if (nc == 2) fix_block<2, kChains, kDbg>(P, S, dcol, buf, i, n0, nc, w, sw, acc, U, b, q, lane, &S.d_empty[ds]);
        else if (nc == 1) fix_block<1, kChains, kDbg>(P, S, dcol, buf, i, n0, nc, w, sw, acc, U, b, q, lane, &S.d_empty[ds]);
        else {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.d_empty[ds]);
        }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.b_empty[buf]);
      ++ug;
      // ---- epilogue (rows 32*q + lane of the tile, pairs [n0, n0 + 4))
      if (kGU) {
        float r[kTFixPairs];
#pragma unroll
        for (int n = 0; n < kTFixPairs; ++n) {
          r[n] = 0.f;
#pragma unroll
          for (int c = 0; c < kChains; ++c) r[n] = __fadd_rn(r[n], acc[c][n]);
        }
        if (q < 2) {
#pragma unroll
          for (int n = 0; n < kTFixPairs; ++n) S.xch[32 * q + lane][n0 + n] = r[n];
        }
        // meet the other fixup warps (bounded wait: a warp that gave up
        // cannot leave the others waiting for ever)
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.fx_bar[0]);
        if (!tc_wait(&S.fx_bar[0], (ug - 1) & 1u, S, P.status)) break;
        if (q >= 2) {
          const int rr = 32 * (q - 2) + lane;  // f offset within the tile
          for (int n = 0; n < kTFixPairs && n0 + n < U.it.count; ++n) {
            const float g = S.xch[rr][n0 + n];
            const float a = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.f, expf(-g))), r[n]);
            const float amax = warp_max(fabsf(a));
            const float dd = __fdiv_rn(amax, 127.f);
            int qq = 0;
            if (dd != 0.f) qq = max(-127, min(127, __float2int_rn(__fdiv_rn(a, dd))));
            const int pair = item_pair(P, U.it, n0 + n);
            if (pair_ok(P, pair)) {
              P.aq[static_cast<size_t>(pair) * F + 64 * U.mt + rr] = static_cast<int8_t>(qq);
              if (lane == 0) P.ad[static_cast<size_t>(pair) * (F / kQBlock) + 2 * U.mt + (q - 2)] = dd;
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.fx_bar[1]);
        if (!tc_wait(&S.fx_bar[1], (ug - 1) & 1u, S, P.status)) break;
      } else {
        const int hrow = kTM * U.mt + 32 * q + lane;
        for (int n = 0; n < kTFixPairs && n0 + n < U.it.count; ++n)
          if (pair_ok(P, item_pair(P, U.it, n0 + n)))
            P.ye[static_cast<size_t>(item_pair(P, U.it, n0 + n)) * H + hrow] = acc[0][n];
        __threadfence();
        __syncwarp();
        for (int n = 0; n < kTFixPairs && n0 + n < U.it.count; ++n)
          arrive_and_combine(P, item_pair(P, U.it, n0 + n), 4 * U.mt + q, lane);
      }
    }
  } else if (warp == kTCopy) {
    // ------------------------------------------------ weight bulk copies
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      uint32_t wi = 0;
      TcUnit U;
      bool ok = true;
      for (int u = blockIdx.x; ok && tc_unit(P, u, m_tiles, ks_n, nb, U); u += gridDim.x) {
        if (U.it.expert < 0) continue;
        const uint32_t* src[4];
        const uint16_t* ssrc[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          src[p] = tile_panel<kGU>(P, U, p, nb);
          ssrc[p] = tile_scales<kGU>(P, U, p, nb);
        }
        for (int i = 0; i < U.nbu; ++i, ++wi) {
          const int b = U.ks + i * ks_n;
          const int ws = wi % kTWStages;
          if (!tc_wait(&S.w_empty[ws], ((wi / kTWStages) & 1u) ^ 1u, S, P.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&S.w_full[ws], 4 * (kPanelBlockBytes + kPanel * 2));
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            bulk_g2s(S.w[ws][p], src[p] + static_cast<size_t>(b) * kBlockWords * kPanel, kPanelBlockBytes,
                     &S.w_full[ws], pol);
            bulk_g2s(S.wsc[ws][p], ssrc[p] + static_cast<size_t>(b) * kPanel, kPanel * 2, &S.w_full[ws], pol);
          }
        }
      }
      // the copies still in flight land before the CTA leaves (after a
      // timeout elsewhere; normally the decode warps have waited for them)
      for (uint32_t k = wi > kTWStages ? wi - kTWStages : 0; k < wi; ++k)
        if (!mbar_wait(&S.w_full[k % kTWStages], (k / kTWStages) & 1u)) record_status(P.status, MOE_ERR_TIMEOUT);
    }
  } else if (warp == kTGat) {
    // ------------------------------------------------ activation gather
    uint32_t ug = 0;
    TcUnit U;
    for (int u = blockIdx.x; tc_unit(P, u, m_tiles, ks_n, nb, U); u += gridDim.x) {
      if (U.it.expert < 0) continue;
      const int buf = ug & 1;
      if (!tc_wait(&S.b_empty[buf], ((ug >> 1) & 1u) ^ 1u, S, P.status)) break;
      tc_gather<kGU>(P, S, buf, U, ks_n, lane);
      fence_proxy_async_shared();  // the codes are read by the tensor cores
      __syncwarp();
      // (the wait test knob withholds the first arrival: the MMA and fixup
      // waits for it run out)
      if (lane == 0 && !(ug == 0 && S.knob == kKnobTcGather)) mbar_arrive(&S.b_full[buf]);
      ++ug;
    }
  } else if (warp == kTMma && lane == 0) {
    // ------------------------------------------------ MMA issue
    const uint32_t idesc = idesc_i8(kTM, kTN);
    uint32_t ug = 0, ai = 0, di = 0;
    TcUnit U;
    bool ok = true;
    for (int u = blockIdx.x; ok && tc_unit(P, u, m_tiles, ks_n, nb, U); u += gridDim.x) {
      if (U.it.expert < 0) continue;
      const int buf = ug & 1;
      if (!tc_wait(&S.b_full[buf], (ug >> 1) & 1u, S, P.status)) break;
      tc_fence_after();
      for (int i = 0; i < U.nbu; ++i, ++ai, ++di) {
        const int as = ai % kTAStages, ds = di % kTDStages;
        if (!tc_wait(&S.a_full[as], (ai / kTAStages) & 1u, S, P.status) ||
            !tc_wait(&S.d_empty[ds], ((di / kTDStages) & 1u) ^ 1u, S, P.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t bdesc = smem_desc(smem_u32(S.B[buf][i]), 128, 256);
#pragma unroll
        for (int s = 0; s < kSubPerBlock; ++s)
          mma_i8_ts(tbase + kTDcol + kTDStageCols * ds + kTN * s, tbase + kTAcol + 64 * as + 8 * s,
                    bdesc + static_cast<uint64_t>((s * kTN * 32) >> 4), idesc, false);
        mma_commit(&S.d_full[ds]);
        mma_commit(&S.a_empty[as]);
      }
      if (!ok) break;
      mma_commit(&S.b_empty[buf]);
      ++ug;
    }
    // every MMA has completed before the columns are released
    mma_commit(&S.mma_done);
    if (!mbar_wait(&S.mma_done, 0)) record_status(P.status, MOE_ERR_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, kTTmemCols);
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
static size_t tc_smem() {
  // more than half of the SM's shared memory, so that one CTA (holding all 512
  // TMEM columns) runs per SM
  const size_t s = sizeof(TcSmem) + 1024;
  return s < 120 * 1024 ? 120 * 1024 : s;
}

bool tc_ffn_supported(const DecodeParams& P) {
  return P.format == MOE_FORMAT_TERNARY && P.hidden / kBlock <= kTcMaxBlocks && P.ffn / kBlock <= kTcMaxBlocks &&
         P.hidden % kTM == 0 && P.ffn % 64 == 0;
}

bool tc_ffn_preferred(const DecodeParams& P) {
  // measured on B200: with 1-2 pairs per expert (the 8- and 16-token decode
  // batches) the CUDA-core grouped kernels are faster; the tensor-core path
  // is kept for the test hook until its decode warps keep the MMA fed
  (void)P;
  return false;
}

int launch_ffn_tc(const DecodeParams& P, cudaStream_t stream) {
  static std::atomic<bool> attrs_done[64];  // the attribute calls are idempotent
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attrs_done[dev].load(std::memory_order_relaxed)) {
    cudaFuncSetAttribute(k_tcmv<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
    cudaFuncSetAttribute(k_tcmv<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
    cudaFuncSetAttribute(k_tcmv<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
    cudaFuncSetAttribute(k_tcmv<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
    attrs_done[dev].store(true, std::memory_order_relaxed);
  }
  int n_sm = 148;
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  const size_t smem = tc_smem();
  const bool dbg = P.dbg_isum_gu != nullptr;
  launch_k(dbg ? k_tcmv<true, true> : k_tcmv<true, false>, dim3(n_sm), dim3(kTThreads), smem, stream, P, 1);
  note_launch(MOE_K_TC_GATEUP, stream);
  launch_k(dbg ? k_tcmv<false, true> : k_tcmv<false, false>, dim3(n_sm), dim3(kTThreads), smem, stream, P, 1);
  note_launch(MOE_K_TC_DOWN, stream);
  return check_launch("expert_ffn (tensor cores)");
}

}  // namespace bitmoe
