// decode.cu -- expert FFN on CUDA cores: fused gate+up mat-vec with a SwiGLU
// and int8 requantization epilogue, then the down mat-vec with the weighted
// top-k combine (sm_100a).
//
// Parakon Runtime README, "How it works": decode uses fused mat-vec kernels
// that read the quantized blocks directly from VRAM and accumulate against
// int8-quantized activations.  pxq_llama README, "Updates -- 2026-07-28": gate
// and up are computed together with the SiLU unary; "What's PXQ?": gate/up
// fusion, K-split decode and a grouped-MoE path.
//
// Work is cut into items: up to kChunk (token, slot) pairs routed to the same
// expert.  With one token every slot is its own item (direct mode); with more
// tokens a grouping pass collects the pairs of each expert so that the
// expert's weights stream from HBM once per step and every decoded digit word
// serves all pairs of the item.
#include <atomic>
#include <cub/block/block_scan.cuh>

#include "bitmoe.h"
#include "common.cuh"
#include "decode.cuh"
#include "ptx.cuh"
#include "quant.cuh"
#include "tcmv.cuh"
#include "ternary_dot.cuh"
#include "topk.cuh"

namespace bitmoe {

size_t group_ws_layout(int E, int npairs, size_t off, GroupWs* G) {
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  G->items = take(sizeof(Item) * static_cast<size_t>(npairs));
  G->n_items = take(sizeof(int32_t));
  G->pairs = take(sizeof(int32_t) * static_cast<size_t>(npairs));
  G->scratch = take(sizeof(int32_t) * 2 * static_cast<size_t>(E + 1));
  return off;
}

// ---------------------------------------------------------------------------
// Grouping (S6): count the pairs of each expert, scan, cut each expert's pairs
// into items of at most kChunk, and scatter the pair ids.  Ids outside
// [0, E) form one extra group with expert -1 (their outputs are zero).
// One CTA of 1024 threads.
// ---------------------------------------------------------------------------
constexpr int kGroupThreads = 1024;

// sidx: the pairs' expert ids in shared memory where the caller has them
// (else they are read from P.idx).
__device__ __forceinline__ void group_body(const DecodeParams& P, const int* sidx = nullptr) {
  using Scan = cub::BlockScan<int, kGroupThreads>;
  __shared__ typename Scan::TempStorage scan_tmp;
  __shared__ int cnt[kMaxExperts + 1];
  __shared__ int off[kMaxExperts + 1];
  __shared__ int fill[kMaxExperts + 1];
  const int E = P.n_experts, npairs = P.ntok * P.top_k, tid = threadIdx.x;
  for (int e = tid; e <= E; e += kGroupThreads) { cnt[e] = 0; fill[e] = 0; }
  __syncthreads();
  // eight ids per thread in flight at a time (the counts' atomics would
  // otherwise hold each load back)
  constexpr int kU = 8;
  for (int p0 = tid; p0 < npairs; p0 += kU * kGroupThreads) {
    int ev[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int p = p0 + u * kGroupThreads;
      ev[u] = p < npairs ? (sidx ? sidx[p] : __ldcg(P.idx + p)) : 0;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (p0 + u * kGroupThreads >= npairs) continue;
      int e = ev[u];
      if (e < 0 || e >= E) { record_status(P.status, MOE_ERR_BAD_INDEX); e = E; }
      atomicAdd(&cnt[e], 1);
    }
  }
  __syncthreads();
  // groups 0..E handled two per thread (E + 1 <= 2 * kGroupThreads)
  int c[2], ic[2], o[2], io[2];
  for (int r = 0; r < 2; ++r) {
    const int e = 2 * tid + r;
    c[r] = e <= E ? cnt[e] : 0;
    ic[r] = (c[r] + P.group_chunk - 1) / P.group_chunk;
  }
  int tot_c = 0, tot_i = 0;
  Scan(scan_tmp).ExclusiveSum(c[0] + c[1], o[0], tot_c);
  __syncthreads();
  Scan(scan_tmp).ExclusiveSum(ic[0] + ic[1], io[0], tot_i);
  o[1] = o[0] + c[0];
  io[1] = io[0] + ic[0];
  Item* items = const_cast<Item*>(P.items);
  for (int r = 0; r < 2; ++r) {
    const int e = 2 * tid + r;
    if (e > E) continue;
    off[e] = o[r];
    for (int i = 0; i < ic[r]; ++i) {
      Item it;
      it.expert = e == E ? -1 : e;
      it.start = o[r] + i * P.group_chunk;
      it.count = min(P.group_chunk, c[r] - i * P.group_chunk);
      it.pad = 0;
      items[io[r] + i] = it;
    }
  }
  if (tid == 0) *const_cast<int32_t*>(P.n_items) = tot_i;
  __syncthreads();
  int32_t* pairs = const_cast<int32_t*>(P.pairs);
  for (int p0 = tid; p0 < npairs; p0 += kU * kGroupThreads) {
    int ev[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int p = p0 + u * kGroupThreads;
      ev[u] = p < npairs ? (sidx ? sidx[p] : __ldcg(P.idx + p)) : 0;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int p = p0 + u * kGroupThreads;
      if (p >= npairs) continue;
      int e = ev[u];
      if (e < 0 || e >= E) e = E;
      pairs[off[e] + atomicAdd(&fill[e], 1)] = p;
    }
  }
}

__global__ void __launch_bounds__(kGroupThreads) k_group(DecodeParams P) {
  pdl_enter();
  group_body(P);
}

// Up to kMaxDecodeTokens tokens: warp w takes the top-k and softmax of tokens
// w, w + 32, ... (warp_topk_softmax, as k_topk_softmax), then the CTA groups
// the pairs.
template <int kPer>
__global__ void __launch_bounds__(kGroupThreads) k_topk_group(DecodeParams P, const float* __restrict__ logits,
                                                              float* __restrict__ wts) {
  pdl_enter();
  __shared__ int sidx[kMaxDecodeTokens * kMaxTopK];  // the ids again for the grouping
  const int lane = threadIdx.x & 31;
  const int E = P.n_experts, K = P.top_k;
  for (int t = threadIdx.x >> 5; t < P.ntok; t += kGroupThreads / 32) {
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
      const_cast<int32_t*>(P.idx)[static_cast<int64_t>(t) * K + lane] = my_e;
      sidx[t * K + lane] = my_e;
      wts[static_cast<int64_t>(t) * K + lane] = w;
    }
  }
  __syncthreads();
  group_body(P, sidx);
}

// S1 + S2 + S6 of a decode batch in one launch.  CTA (i, c) copies router
// rows [i*EW, (i+1)*EW) and tokens [c*TT, (c+1)*TT) of x into shared memory
// (one bulk copy each, so the CTA pays one copy latency), computes those
// logits with the fixed evaluation order of the router kernels (one warp per
// logit: lane l's chain over k = l, l+32, ... ascending, then the xor
// butterfly), and quantizes its share of the tile's 32-blocks of x.  The last
// CTA to finish (a ticket counter that it resets) takes every token's top-k
// and softmax (warp_topk_softmax, one warp per token) and groups the pairs
// by expert (group_body).  No CTA waits for another.
template <int kPer>
__global__ void __launch_bounds__(kGroupThreads) k_route_group(DecodeParams P, const float* __restrict__ x,
                                                               const float* __restrict__ wr,
                                                               float* __restrict__ logits,
                                                               float* __restrict__ wts, uint32_t* ticket,
                                                               int EW, int TT) {
  extern __shared__ __align__(128) unsigned char rsm[];
  __shared__ int sidx[kMaxDecodeTokens * kMaxTopK];
  const int H = P.hidden, E = P.n_experts, T = P.ntok, K = P.top_k;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nwarp = blockDim.x >> 5;
  uint64_t* bar = reinterpret_cast<uint64_t*>(rsm);
  int* flag = reinterpret_cast<int*>(rsm + 8);
  float* wsm = reinterpret_cast<float*>(rsm + 128);  // [EW][H]
  float* xsm = wsm + static_cast<size_t>(EW) * H;    // [TT][H]
  const int e0 = blockIdx.x * EW, ne = min(EW, E - e0);
  const int t0 = blockIdx.y * TT, nt = min(TT, T - t0);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // the router rows are caller data that no kernel of this library writes:
  // their copy starts before the dependency wait
  if (tid == 0) {
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(ne + nt) * H * 4);
    bulk_g2s(wsm, wr + static_cast<size_t>(e0) * H, static_cast<uint32_t>(ne) * H * 4, bar, policy_evict_first());
  }
  pdl_wait();
  if (tid == 0)
    bulk_g2s(xsm, x + static_cast<size_t>(t0) * H, static_cast<uint32_t>(nt) * H * 4, bar, policy_evict_last());
  pdl_launch_dependents();
  const bool ok = mbar_wait(bar, 0);
  if (!ok) {
    // the copies must land before the CTA exits; the counter still counts
    // this CTA, and the status tells the caller that the step is void
    if (tid == 0) record_status(P.status, MOE_ERR_TIMEOUT);
    mbar_wait(bar, 0);
  } else {
    // micro-tiles of up to 2 tokens x 2 experts per warp: each value a lane
    // loads from shared memory feeds two of the logits' chains (shared
    // memory bandwidth, not the chains, bounds one logit per warp)
    const int mtn = (nt + 1) / 2, men = (ne + 1) / 2;
    for (int mt = warp; mt < mtn * men; mt += nwarp) {
      const int ti = (mt / men) * 2, ei = (mt % men) * 2;
      const bool t1 = ti + 1 < nt, e1 = ei + 1 < ne;
      const float* w0 = wsm + static_cast<size_t>(ei) * H;
      const float* w1 = e1 ? w0 + H : w0;
      const float* x0 = xsm + static_cast<size_t>(ti) * H;
      const float* x1 = t1 ? x0 + H : x0;
      float p00 = 0.f, p01 = 0.f, p10 = 0.f, p11 = 0.f;
#pragma unroll 4
      for (int k = lane; k < H; k += 32) {
        const float a0 = x0[k], a1 = x1[k], b0 = w0[k], b1 = w1[k];
        p00 = __fmaf_rn(b0, a0, p00);
        p01 = __fmaf_rn(b1, a0, p01);
        p10 = __fmaf_rn(b0, a1, p10);
        p11 = __fmaf_rn(b1, a1, p11);
      }
#pragma unroll
      for (int m = 16; m >= 1; m >>= 1) {
        p00 = __fadd_rn(p00, __shfl_xor_sync(0xffffffffu, p00, m));
        p01 = __fadd_rn(p01, __shfl_xor_sync(0xffffffffu, p01, m));
        p10 = __fadd_rn(p10, __shfl_xor_sync(0xffffffffu, p10, m));
        p11 = __fadd_rn(p11, __shfl_xor_sync(0xffffffffu, p11, m));
      }
      if (lane == 0) {
        float* l0 = logits + static_cast<size_t>(t0 + ti) * E + e0 + ei;
        l0[0] = p00;
        if (e1) l0[1] = p01;
        if (t1) l0[E] = p10;
        if (t1 && e1) l0[E + 1] = p11;
      }
    }
    // the tile's 32-blocks of x, dealt over the CTAs that hold it from the
    // last warp down (the first warps take the logits)
    const int nblk = nt * (H / kQBlock);
    for (int blk = (nwarp - 1 - warp) * gridDim.x + blockIdx.x; blk < nblk; blk += gridDim.x * nwarp)
      quant_act_block(xsm, blk, lane, const_cast<int8_t*>(P.xq) + static_cast<size_t>(t0) * H,
                      const_cast<float*>(P.xd) + static_cast<size_t>(t0) * (H / kQBlock));
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) *flag = (atomicAdd(ticket, 1u) == gridDim.x * gridDim.y - 1) ? 1 : 0;
  __syncthreads();
  if (!*flag) return;
  __threadfence();
  if (tid == 0) atomicExch(ticket, 0u);  // every CTA has taken its ticket
  for (int t = warp; t < T; t += nwarp) {
    uint32_t key[kPer];
    uint32_t need = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = lane + 32 * i;
      key[i] = 0u;
      if (e < E) {
        key[i] = f32_key(__ldcg(logits + static_cast<size_t>(t) * E + e));
        need |= 1u << i;
      }
    }
    int my_e;
    float w;
    warp_topk_softmax<kPer>(key, need, K, lane, my_e, w);
    if (lane < K) {
      const_cast<int32_t*>(P.idx)[static_cast<size_t>(t) * K + lane] = my_e;
      sidx[t * K + lane] = my_e;
      wts[static_cast<size_t>(t) * K + lane] = w;
    }
  }
  __syncthreads();
  group_body(P, sidx);
}

// ---------------------------------------------------------------------------
// S3 + S4: gate and up of one item for one 32-row panel of the ffn dimension.
// The 8 warps split the 256-blocks of the hidden dimension; the per-warp
// partial rows are summed in warp order; warp n then applies SwiGLU to pair
// n's 32 rows and requantizes them (one 32-block of a) to int8.
// grid: (ffn/32, items), block: kGateUpWarps*32.
// ---------------------------------------------------------------------------
template <int NT, int kFmt>
__device__ __forceinline__ void gateup_run(const DecodeParams& P, const Item& item, int panel,
                                           unsigned char* smem) {
  constexpr int kWords = WordsPerBlock<kFmt == MOE_FORMAT_SIGN>::value;
  const int H = P.hidden, F = P.ffn;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int* q4 = reinterpret_cast<int*>(smem);
  float* d = reinterpret_cast<float*>(q4 + (H / 4) * NT);
  int* as = reinterpret_cast<int*>(d + (H / kQBlock) * NT);
  float* red = reinterpret_cast<float*>(as + (H / kQBlock) * NT);  // [2][warps][NT][32]
  for (int n = 0; n < NT; ++n) {
    if (n < item.count) {
      const int t = item_pair(P, item, n) / P.top_k;
      stage_act<NT>(P.xq + static_cast<size_t>(t) * H, P.xd + static_cast<size_t>(t) * (H / kQBlock),
                    H, n, q4, d, as, threadIdx.x, blockDim.x);
    } else {
      zero_act<NT>(H, n, q4, d, as, threadIdx.x, blockDim.x);
    }
  }
  __syncthreads();
  const int nb = H / kBlock;
  const size_t pb0 = (static_cast<size_t>(item.expert) * (F / kPanel) + panel) * nb;
  const uint32_t* const tw[2] = {P.gate_trits + pb0 * kWords * kPanel + lane,
                                 P.up_trits + pb0 * kWords * kPanel + lane};
  const uint16_t* const ts[2] = {P.gate_scales + pb0 * kPanel + lane, P.up_scales + pb0 * kPanel + lane};
  float out[2][NT];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int n = 0; n < NT; ++n) out[m][n] = 0.f;
  if constexpr (kFmt == MOE_FORMAT_E16) {
    // per-row fp16 anchors, 4-bit sub-scale codes per 16 weights
    const size_t row = static_cast<size_t>(item.expert) * F + panel * kPanel + lane;
    const uint32_t* const tc[2] = {P.gate_codes + pb0 * kE16Words * kPanel + lane,
                                   P.up_codes + pb0 * kE16Words * kPanel + lane};
    const float a16[2] = {f16_bits_to_f32(P.gate_scales[row]) * 0.0625f, f16_bits_to_f32(P.up_scales[row]) * 0.0625f};
    if constexpr (NT >= 4) {
      // many vectors: gate, then up (each matrix's sums are independent, so
      // the results are those of the joint pass, in fewer registers)
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const uint32_t* const tw1[1] = {tw[m]};
        const uint32_t* const tc1[1] = {tc[m]};
        const float a1[1] = {a16[m]};
        float o1[1][NT];
#pragma unroll
        for (int n = 0; n < NT; ++n) o1[0][n] = 0.f;
        panel_dot_e16<1, NT>(tw1, tc1, a1, warp, nb, kGateUpWarps, q4, d, o1);
#pragma unroll
        for (int n = 0; n < NT; ++n) out[m][n] = o1[0][n];
      }
    } else {
      panel_dot_e16<2, NT>(tw, tc, a16, warp, nb, kGateUpWarps, q4, d, out);
    }
  } else if constexpr (NT >= 4) {
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const uint32_t* const tw1[1] = {tw[m]};
      const uint16_t* const ts1[1] = {ts[m]};
      float o1[1][NT];
#pragma unroll
      for (int n = 0; n < NT; ++n) o1[0][n] = 0.f;
      panel_dot<1, NT, kFmt == MOE_FORMAT_SIGN>(tw1, ts1, warp, nb, kGateUpWarps, q4, d, as, o1);
#pragma unroll
      for (int n = 0; n < NT; ++n) out[m][n] = o1[0][n];
    }
  } else {
    panel_dot<2, NT, kFmt == MOE_FORMAT_SIGN>(tw, ts, warp, nb, kGateUpWarps, q4, d, as, out);
  }
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int n = 0; n < NT; ++n) red[((m * kGateUpWarps + warp) * NT + n) * 32 + lane] = out[m][n];
  __syncthreads();
  if (warp < item.count) {
    const int n = warp;
    float g = 0.f, u = 0.f;
    for (int w = 0; w < kGateUpWarps; ++w) {
      g = __fadd_rn(g, red[((0 * kGateUpWarps + w) * NT + n) * 32 + lane]);
      u = __fadd_rn(u, red[((1 * kGateUpWarps + w) * NT + n) * 32 + lane]);
    }
    const float a = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.f, expf(-g))), u);
    const float amax = warp_max(fabsf(a));
    const float dd = __fdiv_rn(amax, 127.f);
    int q = 0;
    if (dd != 0.f) q = max(-127, min(127, __float2int_rn(__fdiv_rn(a, dd))));
    const int pair = item_pair(P, item, n);
    if (pair_ok(P, pair)) {
      P.aq[static_cast<size_t>(pair) * F + panel * kPanel + lane] = static_cast<int8_t>(q);
      if (lane == 0) P.ad[static_cast<size_t>(pair) * (F / kQBlock) + panel] = dd;
    }
  }
}

// Four CTAs per SM (at most 64 registers a thread): the items of a decode
// batch are mostly single pairs, whose path needs few registers; the rare
// 8-pair path spills a little.
template <int NTMAX, int kFmt>
__global__ void __launch_bounds__(kGateUpWarps * 32, 4) k_gateup(DecodeParams P) {
  pdl_enter();
  extern __shared__ __align__(16) unsigned char smem[];
  Item item;
  if (!fetch_item(P, blockIdx.y, item)) return;
  const int panel = blockIdx.x;
  if (item.expert < 0) {
    if (threadIdx.x == 0) record_status(P.status, MOE_ERR_BAD_INDEX);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < item.count) {
      const int pair = item_pair(P, item, warp);
      if (pair_ok(P, pair)) {
        P.aq[static_cast<size_t>(pair) * P.ffn + panel * kPanel + lane] = 0;
        if (lane == 0) P.ad[static_cast<size_t>(pair) * (P.ffn / kQBlock) + panel] = 0.f;
      }
    }
    return;
  }
  if constexpr (NTMAX == 1) {
    gateup_run<1, kFmt>(P, item, panel, smem);
  } else {
    if (item.count <= 1) gateup_run<1, kFmt>(P, item, panel, smem);
    else if (item.count <= 2) gateup_run<2, kFmt>(P, item, panel, smem);
    else if (item.count <= 4) gateup_run<4, kFmt>(P, item, panel, smem);
    else gateup_run<8, kFmt>(P, item, panel, smem);
  }
}

// ---------------------------------------------------------------------------
// S5: down mat-vec of one item for kDownWarps 32-row panels of the hidden
// dimension (one panel per warp), written per pair to ye; the CTA that
// completes the last of a token's top_k slots for a panel combines
// y[t] = sum_j wts[t][j] * ye[t][j] over the slots in order.
// grid: (hidden/32/kDownWarps, items), block: kDownWarps*32.
// ---------------------------------------------------------------------------
template <int NT, int kFmt>
__device__ __forceinline__ void down_run(const DecodeParams& P, const Item& item, int pgroup,
                                         unsigned char* smem) {
  constexpr int kWords = WordsPerBlock<kFmt == MOE_FORMAT_SIGN>::value;
  const int H = P.hidden, F = P.ffn;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int* q4 = reinterpret_cast<int*>(smem);
  float* d = reinterpret_cast<float*>(q4 + (F / 4) * NT);
  int* as = reinterpret_cast<int*>(d + (F / kQBlock) * NT);
  for (int n = 0; n < NT; ++n) {
    if (n < item.count) {
      const int pair = item_pair(P, item, n);
      stage_act<NT>(P.aq + static_cast<size_t>(pair) * F, P.ad + static_cast<size_t>(pair) * (F / kQBlock),
                    F, n, q4, d, as, threadIdx.x, blockDim.x);
    } else {
      zero_act<NT>(F, n, q4, d, as, threadIdx.x, blockDim.x);
    }
  }
  __syncthreads();
  const int panel = pgroup * kDownWarps + warp;
  const int nb = F / kBlock;
  const size_t pb0 = (static_cast<size_t>(item.expert) * (H / kPanel) + panel) * nb;
  const uint32_t* const tw[1] = {P.down_trits + pb0 * kWords * kPanel + lane};
  const uint16_t* const ts[1] = {P.down_scales + pb0 * kPanel + lane};
  float out[1][NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) out[0][n] = 0.f;
  if constexpr (kFmt == MOE_FORMAT_E16) {
    const size_t row = static_cast<size_t>(item.expert) * H + panel * kPanel + lane;
    const uint32_t* const tc[1] = {P.down_codes + pb0 * kE16Words * kPanel + lane};
    const float a16[1] = {f16_bits_to_f32(P.down_scales[row]) * 0.0625f};
    panel_dot_e16<1, NT>(tw, tc, a16, 0, nb, 1, q4, d, out);
  } else {
    panel_dot<1, NT, kFmt == MOE_FORMAT_SIGN>(tw, ts, 0, nb, 1, q4, d, as, out);
  }
#pragma unroll
  for (int n = 0; n < NT; ++n)
    if (n < item.count)
      if (pair_ok(P, item_pair(P, item, n)))
        P.ye[static_cast<size_t>(item_pair(P, item, n)) * H + panel * kPanel + lane] = out[0][n];
  __threadfence();
  __syncwarp();
  for (int n = 0; n < item.count; ++n) arrive_and_combine(P, item_pair(P, item, n), panel, lane);
}

// Eight CTAs per SM (at most 64 registers a thread, which leaves room for the
// prefetched next block of weight words in panel_dot).
template <int NTMAX, int kFmt>
__global__ void __launch_bounds__(kDownWarps * 32, 8) k_down(DecodeParams P) {
  pdl_enter();
  extern __shared__ __align__(16) unsigned char smem[];
  Item item;
  if (!fetch_item(P, blockIdx.y, item)) return;
  const int pgroup = blockIdx.x;
  if (item.expert < 0) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int panel = pgroup * kDownWarps + warp;
    for (int n = 0; n < item.count; ++n)
      if (pair_ok(P, item_pair(P, item, n)))
        P.ye[static_cast<size_t>(item_pair(P, item, n)) * P.hidden + panel * kPanel + lane] = 0.f;
    __threadfence();
    __syncwarp();
    for (int n = 0; n < item.count; ++n) arrive_and_combine(P, item_pair(P, item, n), panel, lane);
    return;
  }
  if constexpr (NTMAX == 1) {
    down_run<1, kFmt>(P, item, pgroup, smem);
  } else {
    if (item.count <= 1) down_run<1, kFmt>(P, item, pgroup, smem);
    else if (item.count <= 2) down_run<2, kFmt>(P, item, pgroup, smem);
    else if (item.count <= 4) down_run<4, kFmt>(P, item, pgroup, smem);
    else down_run<8, kFmt>(P, item, pgroup, smem);
  }
}

// ---------------------------------------------------------------------------
// Test hook: the mat-vec core on one matrix, with the exact block sums.
// grid: (rows/32, ntok), block: kGateUpWarps*32; warps split the blocks.
// ---------------------------------------------------------------------------
template <int kFmt>
__global__ void __launch_bounds__(kGateUpWarps * 32)
    k_debug_matvec(const uint32_t* __restrict__ trits, const uint16_t* __restrict__ scales,
                   const uint32_t* __restrict__ codes, int rows, int k, const int8_t* __restrict__ xq,
                   const float* __restrict__ xd, float* __restrict__ out, int32_t* __restrict__ isum) {
  extern __shared__ __align__(16) unsigned char smem[];
  int* q4 = reinterpret_cast<int*>(smem);
  float* d = reinterpret_cast<float*>(q4 + k / 4);
  int* as = reinterpret_cast<int*>(d + k / kQBlock);
  float* red = reinterpret_cast<float*>(as + k / kQBlock);
  const int panel = blockIdx.x, t = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  stage_act<1>(xq + static_cast<size_t>(t) * k, xd + static_cast<size_t>(t) * (k / kQBlock), k, 0, q4,
               d, as, threadIdx.x, blockDim.x);
  __syncthreads();
  const int nb = k / kBlock;
  const int r = panel * kPanel + lane;
  const size_t pb0 = static_cast<size_t>(panel) * nb;
  const uint32_t* const tw[1] = {trits + pb0 * WordsPerBlock<kFmt == MOE_FORMAT_SIGN>::value * kPanel + lane};
  const uint16_t* const ts[1] = {scales + pb0 * kPanel + lane};
  float o[1][1] = {{0.f}};
  int32_t* isum_row = isum ? isum + (static_cast<size_t>(t) * rows + r) * (k / kQBlock) : nullptr;
  if constexpr (kFmt == MOE_FORMAT_E16) {
    const uint32_t* const tc[1] = {codes + pb0 * kE16Words * kPanel + lane};
    const float a16[1] = {f16_bits_to_f32(scales[r]) * 0.0625f};
    panel_dot_e16<1, 1>(tw, tc, a16, warp, nb, kGateUpWarps, q4, d, o, isum_row, 0);
  } else {
    panel_dot<1, 1, kFmt == MOE_FORMAT_SIGN>(tw, ts, warp, nb, kGateUpWarps, q4, d, as, o, isum_row, 0);
  }
  red[warp * 32 + lane] = o[0][0];
  __syncthreads();
  if (warp == 0) {
    float acc = 0.f;
    for (int w = 0; w < kGateUpWarps; ++w) acc = __fadd_rn(acc, red[w * 32 + lane]);
    out[static_cast<size_t>(t) * rows + r] = acc;
  }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
// Raise the dynamic shared-memory limit of every kernel in this file to the
// opt-in maximum, once per device (so no attribute call happens inside a
// stream capture).
static void init_kernel_attrs() {
  constexpr int kMaxDev = 64;
  static std::atomic<bool> done[kMaxDev];  // the attribute calls are idempotent
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < kMaxDev && done[dev].load(std::memory_order_relaxed)) return;
  const void* kernels[] = {
      reinterpret_cast<const void*>(&k_gateup<1, 0>),     reinterpret_cast<const void*>(&k_gateup<kChunk, 0>),
      reinterpret_cast<const void*>(&k_down<1, 0>),       reinterpret_cast<const void*>(&k_down<kChunk, 0>),
      reinterpret_cast<const void*>(&k_gateup<1, 1>),     reinterpret_cast<const void*>(&k_gateup<kChunk, 1>),
      reinterpret_cast<const void*>(&k_down<1, 1>),       reinterpret_cast<const void*>(&k_down<kChunk, 1>),
      reinterpret_cast<const void*>(&k_gateup<1, 2>),     reinterpret_cast<const void*>(&k_gateup<kChunk, 2>),
      reinterpret_cast<const void*>(&k_down<1, 2>),       reinterpret_cast<const void*>(&k_down<kChunk, 2>),
      reinterpret_cast<const void*>(&k_debug_matvec<0>),  reinterpret_cast<const void*>(&k_debug_matvec<1>),
      reinterpret_cast<const void*>(&k_debug_matvec<2>)};
  for (const void* k : kernels)
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
  if (dev >= 0 && dev < kMaxDev) done[dev].store(true, std::memory_order_relaxed);
}

int launch_group(const DecodeParams& P, cudaStream_t stream) {
  launch_k(k_group, dim3(1), dim3(kGroupThreads), 0, stream, P);
  note_launch(MOE_K_GROUP, stream);
  return check_launch("group");
}

// Shape of k_route_group: EW experts and TT tokens per CTA with their rows
// in shared memory, in one wave of at most n_sm CTAs, the fewest rows per
// CTA first (the least copying per SM), then the most CTAs.  False if no
// shape fits one wave.
static bool route_group_shape(int H, int E, int T, int n_sm, size_t smem_cap, int* EW, int* TT) {
  const size_t row = static_cast<size_t>(H) * 4;
  int best_rows = 0, best_grid = 0;
  for (int tt = T;; tt = (tt + 1) / 2) {
    for (int ew = 1; ew <= E && ew <= 64; ++ew) {
      const int64_t grid = static_cast<int64_t>((E + ew - 1) / ew) * ((T + tt - 1) / tt);
      if (grid > n_sm || 128 + (ew + tt) * row > smem_cap) continue;
      const int rows = ew + tt;
      if (best_rows == 0 || rows < best_rows || (rows == best_rows && grid > best_grid)) {
        best_rows = rows;
        best_grid = static_cast<int>(grid);
        *EW = ew;
        *TT = tt;
      }
    }
    if (tt == 1) break;
  }
  return best_rows > 0;
}

// Largest dynamic shared memory of k_route_group: the opt-in limit less its
// static arrays.
template <int kPer>
static size_t route_group_cap() {
  static std::atomic<size_t> cap{0};  // the same on every device of one architecture
  size_t c = cap.load(std::memory_order_relaxed);
  if (c == 0) {
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, k_route_group<kPer>) != cudaSuccess) return 0;
    const size_t stat = fa.sharedSizeBytes + 1024;
    c = stat < static_cast<size_t>(kMaxDynSmem) ? kMaxDynSmem - stat : 0;
    cap.store(c, std::memory_order_relaxed);
  }
  return c;
}

bool route_group_ok(const DecodeParams& P, int n_sm) {
  if (P.ntok < 1 || P.ntok > kMaxDecodeTokens || P.hidden % kQBlock) return false;
  const size_t cap = P.n_experts <= 128 ? route_group_cap<4>()
                     : P.n_experts <= 256 ? route_group_cap<8>() : route_group_cap<32>();
  int ew = 0, tt = 0;
  return route_group_shape(P.hidden, P.n_experts, P.ntok, n_sm, cap, &ew, &tt);
}

template <int kPer>
static int launch_route_group_k(const DecodeParams& P, const float* x, const float* wr, float* logits,
                                float* wts, uint32_t* ticket, int n_sm, cudaStream_t stream) {
  const size_t cap = route_group_cap<kPer>();
  int EW = 0, TT = 0;
  if (!route_group_shape(P.hidden, P.n_experts, P.ntok, n_sm, cap, &EW, &TT))
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "route_group: no one-wave shape");
  const size_t smem = 128 + static_cast<size_t>(EW + TT) * P.hidden * 4;
  static std::atomic<bool> done[64];  // the attribute call is idempotent
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !done[dev].load(std::memory_order_relaxed)) {
    cudaFuncSetAttribute(k_route_group<kPer>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(cap));
    done[dev].store(true, std::memory_order_relaxed);
  }
  const dim3 grid((P.n_experts + EW - 1) / EW, (P.ntok + TT - 1) / TT);
  launch_k(k_route_group<kPer>, grid, dim3(kGroupThreads), smem, stream, P, x, wr, logits, wts, ticket, EW, TT);
  note_launch(MOE_K_ROUTE_GROUP, stream);
  return check_launch("route_group");
}

int launch_route_group(const DecodeParams& P, const float* x, const float* wr, float* logits, float* wts,
                       uint32_t* ticket, int n_sm, cudaStream_t stream) {
  if (P.n_experts <= 128) return launch_route_group_k<4>(P, x, wr, logits, wts, ticket, n_sm, stream);
  if (P.n_experts <= 256) return launch_route_group_k<8>(P, x, wr, logits, wts, ticket, n_sm, stream);
  return launch_route_group_k<32>(P, x, wr, logits, wts, ticket, n_sm, stream);
}

int launch_topk_group(const DecodeParams& P, const float* logits, float* wts, cudaStream_t stream) {
  if (P.ntok > kMaxDecodeTokens) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "topk_group: more than %d tokens", kMaxDecodeTokens);
  const int E = P.n_experts;
  if (E <= 128) launch_k(k_topk_group<4>, dim3(1), dim3(kGroupThreads), 0, stream, P, logits, wts);
  else if (E <= 256) launch_k(k_topk_group<8>, dim3(1), dim3(kGroupThreads), 0, stream, P, logits, wts);
  else launch_k(k_topk_group<32>, dim3(1), dim3(kGroupThreads), 0, stream, P, logits, wts);
  note_launch(MOE_K_TOPK_GROUP, stream);
  return check_launch("topk_group");
}

template <int kFmt>
static void launch_ffn_fmt(const DecodeParams& P, cudaStream_t stream) {
  const int npairs = P.ntok * P.top_k;
  if (P.direct) {
    const size_t s1 = ActSmem<1>::bytes(P.hidden) + 2 * kGateUpWarps * 1 * 32 * 4;
    const size_t s2 = ActSmem<1>::bytes(P.ffn);
    launch_k(k_gateup<1, kFmt>, dim3(P.ffn / kPanel, npairs), dim3(kGateUpWarps * 32), s1, stream, P);
    note_launch(MOE_K_GATEUP, stream);
    launch_k(k_down<1, kFmt>, dim3(P.hidden / kPanel / kDownWarps, npairs), dim3(kDownWarps * 32), s2, stream, P);
    note_launch(MOE_K_DOWN, stream);
  } else {
    const size_t s1 = ActSmem<kChunk>::bytes(P.hidden) + 2 * kGateUpWarps * kChunk * 32 * 4;
    const size_t s2 = ActSmem<kChunk>::bytes(P.ffn);
    launch_k(k_gateup<kChunk, kFmt>, dim3(P.ffn / kPanel, npairs), dim3(kGateUpWarps * 32), s1, stream, P);
    note_launch(MOE_K_GATEUP, stream);
    launch_k(k_down<kChunk, kFmt>, dim3(P.hidden / kPanel / kDownWarps, npairs), dim3(kDownWarps * 32), s2, stream,
             P);
    note_launch(MOE_K_DOWN, stream);
  }
}

int launch_ffn(const DecodeParams& P, cudaStream_t stream) {
  if (!P.direct && P.group_chunk != kChunk) return fail(MOE_ERR_INVALID_ARG, "expert_ffn: items of %d pairs", P.group_chunk);
  // ternary layers of batches whose items hold many pairs: the tensor-core
  // mat-vecs (a tcgen05.mma of N <= 64 costs the same as one of N = 16, so
  // they pay only when the items are large)
  if (!P.direct && tc_ffn_supported(P) && tc_ffn_preferred(P)) return launch_ffn_tc(P, stream);
  init_kernel_attrs();
  if (P.format == MOE_FORMAT_SIGN) launch_ffn_fmt<MOE_FORMAT_SIGN>(P, stream);
  else if (P.format == MOE_FORMAT_E16) launch_ffn_fmt<MOE_FORMAT_E16>(P, stream);
  else launch_ffn_fmt<MOE_FORMAT_TERNARY>(P, stream);
  return check_launch("expert_ffn");
}

int launch_debug_matvec(const moe_tmat* m, int ntok, const int8_t* xq, const float* xd, float* out,
                        int32_t* isum, cudaStream_t stream) {
  init_kernel_attrs();
  const size_t s = ActSmem<1>::bytes(m->k) + kGateUpWarps * 32 * 4;
  const dim3 grid(m->rows / kPanel, ntok);
  if (m->format == MOE_FORMAT_SIGN)
    k_debug_matvec<1><<<grid, kGateUpWarps * 32, s, stream>>>(m->trits, m->scales, nullptr, m->rows, m->k, xq, xd,
                                                             out, isum);
  else if (m->format == MOE_FORMAT_E16)
    k_debug_matvec<2><<<grid, kGateUpWarps * 32, s, stream>>>(m->trits, m->scales, m->codes, m->rows, m->k, xq, xd,
                                                             out, isum);
  else
    k_debug_matvec<0><<<grid, kGateUpWarps * 32, s, stream>>>(m->trits, m->scales, nullptr, m->rows, m->k, xq, xd,
                                                             out, isum);
  note_launch(MOE_K_DEBUG_MATVEC, stream);
  return check_launch("debug_matvec");
}

}  // namespace bitmoe
