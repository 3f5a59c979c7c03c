// decode2.cu -- decode step kernels (sm_100a): a fused route kernel and
// persistent gate/up and down mat-vec kernels whose warps stream their own
// weight blocks into shared-memory rings with cp.async.
//
// Parakon Runtime README, "How it works": decode uses fused mat-vec kernels
// that read the quantized blocks directly from VRAM and accumulate against
// int8-quantized activations via dp4a.  pxq_llama README, "Updates --
// 2026-07-28": gate and up are computed together with the SiLU unary; "What's
// PXQ?": gate/up fusion and a K-split decode.  llama-modchip page, "Key
// highlights": all top-k experts are evaluated.
//
// Each warp keeps kRing items in flight: an item is one 256-weight block of a
// 32-row panel (1728 bytes per matrix: 13x32 packed words and 32 fp16
// scales); all 32 lanes issue its 16-byte asynchronous copies, so the copy
// issue cost is spread over every lane of every warp (a single issuing thread
// per SM cannot keep up with HBM).  With one token the activation vector is
// staged once per CTA; with several tokens each item also carries the
// activation block of each of its pairs.
//
// Numerics are those of the mat-vec core of decode.cu: per 32-weight
// sub-block an exact int32 sum, scaled by the activation scale in fp32
// (sub-blocks in order), the fp16 weight scale applied per 256-block; gate/up
// blocks b = w, w + 8, ... of a row are accumulated by warp w and the eight
// warp partials summed in warp order; down rows are accumulated block by block
// in order.
#include <atomic>
#include "bitmoe.h"
#include "common.cuh"
#include "decode2.cuh"
#include "matvec.cuh"
#include "ptx.cuh"

namespace bitmoe {

// ---------------------------------------------------------------------------
// S3 + S4: gate/up.  Units are (group, 32-row panel of ffn); a CTA owns a
// contiguous range of units; its warps split each unit's hidden blocks (block
// b -> warp b % 8), reduce through shared memory in warp order, and warp n
// finishes pair n: a = g/(1+exp(-g))*u, int8 requant per 32 rows.
// ---------------------------------------------------------------------------
template <int NTMAX, bool kStaged>
__global__ void __launch_bounds__(kNC * 32) k_gateup3(Decode2Params D) {
  extern __shared__ __align__(1024) unsigned char smem[];
  constexpr int SW = ring_depth<NTMAX>();
  using S = Slot<2, NTMAX, kStaged>;
  const DecodeParams& P = D.P;
  const int H = P.hidden, F = P.ffn, nb = H / kBlock, panels = F / kPanel;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* myring = smem + static_cast<size_t>(warp) * SW * S::bytes;
  float* red = reinterpret_cast<float*>(smem + static_cast<size_t>(kNC) * SW * S::bytes);
  int* sq4 = reinterpret_cast<int*>(red + 2 * 2 * kNC * NTMAX * 32);
  float* sd = reinterpret_cast<float*>(sq4 + H / 4);
  int* sas = reinterpret_cast<int*>(sd + H / kQBlock);
  pdl_wait();
  pdl_launch_dependents();
  int64_t u0, u1;
  cta_range(static_cast<int64_t>(n_groups(P)) * panels, blockIdx.x, gridDim.x, u0, u1);
  if constexpr (kStaged) {
    stage_vector(P.xq, P.xd, H, sq4, sd, sas);
    __syncthreads();
  }
  // issue cursor: the next (unit, block) of this warp to copy
  int64_t iu = u0;
  int ib = warp;
  int ig = -1;
  Group iG{};
  ActSrc<NTMAX> iA;
  auto issue_next = [&](int slot) {
    while (iu < u1 && ib >= nb) { ++iu; ib = warp; }
    if (iu < u1) {
      const int g = static_cast<int>(iu / panels);
      if (g != ig) { iG = get_group(P, g); act_sources<2, NTMAX>(P, iG, iA); ig = g; }
      issue_item<2, NTMAX, kStaged>(myring + slot * S::bytes, P, iG, iA, static_cast<int>(iu % panels), ib, lane);
      ib += kNC;
    }
    cp_commit();
  };
#pragma unroll
  for (int k = 0; k < SW; ++k) issue_next(k);

  int s = 0, ui = 0, cg = -1;
  Group G{};
  for (int64_t u = u0; u < u1; ++u, ++ui) {
    const int g = static_cast<int>(u / panels);
    if (g != cg) { G = get_group(P, g); cg = g; }
    const int p = static_cast<int>(u % panels);
    float part[2][NTMAX];
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int n = 0; n < NTMAX; ++n) part[m][n] = 0.f;
    for (int b = warp; b < nb; b += kNC, ++s) {
      cp_wait<SW - 1>();
      __syncwarp();
      const unsigned char* src = myring + (s % SW) * S::bytes;
      if (G.expert >= 0) {
        if constexpr (kStaged)
          block_dot_n<2, NTMAX>(G.count, src, sq4 + b * (kBlock / 4), 0, sd + b * kSubPerBlock,
                                sas + b * kSubPerBlock, 0, lane, part);
        else
          block_dot_n<2, NTMAX>(G.count, src, reinterpret_cast<const int*>(src + S::act), kBlock / 4,
                                reinterpret_cast<const float*>(src + S::act_d), nullptr, kSubPerBlock, lane,
                                part);
      }
      __syncwarp();
      issue_next(s % SW);
    }
    float* rb = red + (ui & 1) * (2 * kNC * NTMAX * 32);
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int n = 0; n < NTMAX; ++n) rb[((m * kNC + warp) * NTMAX + n) * 32 + lane] = part[m][n];
    __syncthreads();
    if (warp < G.count) {
      const int n = warp;
      float gg = 0.f, uu = 0.f;
      const int nw = nb < kNC ? nb : kNC;
      for (int v = 0; v < nw; ++v) {
        gg = __fadd_rn(gg, rb[((0 * kNC + v) * NTMAX + n) * 32 + lane]);
        uu = __fadd_rn(uu, rb[((1 * kNC + v) * NTMAX + n) * 32 + lane]);
      }
      const float a = __fmul_rn(__fdiv_rn(gg, __fadd_rn(1.f, expf(-gg))), uu);
      const float amax = warp_max(fabsf(a));
      const float dd = __fdiv_rn(amax, 127.f);
      int q = 0;
      if (dd != 0.f) q = max(-127, min(127, __float2int_rn(__fdiv_rn(a, dd))));
      const int pair = group_pair(P, G, n);
      P.aq[static_cast<size_t>(pair) * F + p * kPanel + lane] = static_cast<int8_t>(q);
      if (lane == 0) P.ad[static_cast<size_t>(pair) * (F / kQBlock) + p] = dd;
      if (G.expert < 0 && lane == 0) record_status(P.status, MOE_ERR_BAD_INDEX);
    }
  }
  cp_wait<0>();
}

// ---------------------------------------------------------------------------
// S5: down.  Units are (group, 32-row panel of hidden); warp w of a CTA takes
// the CTA's units w, w+8, ... and accumulates all ffn blocks of a unit in
// order, writes the per-pair rows to ye, then the CTA completing the last of
// a token's top_k slots for that panel combines y = sum_j wts[j] * ye[j] over
// the slots in order.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void down_arrive(const DecodeParams& P, int pair, int panel, int lane) {
  const int K = P.top_k, H = P.hidden;
  const int t = pair / K;
  int32_t* c = P.cnt + static_cast<size_t>(t) * (H / kPanel) + panel;
  int old = 0;
  if (lane == 0) old = atomicAdd(c, 1);
  old = __shfl_sync(0xffffffffu, old, 0);
  if (old == K - 1) {
    __threadfence();
    float y = 0.f;
    const float* ye = P.ye + static_cast<size_t>(t) * K * H + panel * kPanel + lane;
    for (int j = 0; j < K; ++j)
      y = __fmaf_rn(__ldcg(P.wts + static_cast<size_t>(t) * K + j), __ldcg(ye + static_cast<size_t>(j) * H), y);
    P.y[static_cast<size_t>(t) * H + panel * kPanel + lane] = y;
    if (lane == 0) atomicExch(c, 0);
  }
}

template <int NTMAX, bool kStaged>
__global__ void __launch_bounds__(kNC * 32) k_down3(Decode2Params D) {
  extern __shared__ __align__(1024) unsigned char smem[];
  constexpr int SW = ring_depth<NTMAX>();
  using S = Slot<1, NTMAX, kStaged>;
  const DecodeParams& P = D.P;
  const int H = P.hidden, F = P.ffn, K = P.top_k, nb = F / kBlock, panels = H / kPanel;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* myring = smem + static_cast<size_t>(warp) * SW * S::bytes;
  int* sq4 = reinterpret_cast<int*>(smem + static_cast<size_t>(kNC) * SW * S::bytes);  // [K][F/4]
  float* sd = reinterpret_cast<float*>(sq4 + K * (F / 4));                              // [K][F/32]
  int* sas = reinterpret_cast<int*>(sd + K * (F / kQBlock));                            // [K][F/32]
  // The routing is complete when this grid starts (the gate/up grid lets it
  // launch only after its own wait on the router), so weight copies can start
  // before the wait on the gate/up results.
  int64_t u0, u1;
  cta_range(static_cast<int64_t>(n_groups(P)) * panels, blockIdx.x, gridDim.x, u0, u1);
  int64_t iu = u0 + warp;
  int ib = 0;
  int ig = -1;
  Group iG{};
  ActSrc<NTMAX> iA;
  auto issue_next = [&](int slot) {
    if (iu < u1) {
      const int g = static_cast<int>(iu / panels);
      if (g != ig) { iG = get_group(P, g); act_sources<1, NTMAX>(P, iG, iA); ig = g; }
      issue_item<1, NTMAX, kStaged>(myring + slot * S::bytes, P, iG, iA, static_cast<int>(iu % panels), ib, lane);
      if (++ib == nb) { ib = 0; iu += kNC; }
    }
    cp_commit();
  };
  if constexpr (kStaged) {
#pragma unroll
    for (int k = 0; k < SW; ++k) issue_next(k);
    pdl_wait();
    for (int j = 0; j < K; ++j)
      stage_vector(P.aq + static_cast<size_t>(j) * F, P.ad + static_cast<size_t>(j) * (F / kQBlock), F,
                   sq4 + j * (F / 4), sd + j * (F / kQBlock), sas + j * (F / kQBlock));
    __syncthreads();
  } else {
    pdl_wait();
#pragma unroll
    for (int k = 0; k < SW; ++k) issue_next(k);
  }
  int s = 0;
  for (int64_t u = u0 + warp; u < u1; u += kNC) {
    const int g = static_cast<int>(u / panels);
    const Group G = get_group(P, g);
    const int p = static_cast<int>(u % panels);
    float part[1][NTMAX];
#pragma unroll
    for (int n = 0; n < NTMAX; ++n) part[0][n] = 0.f;
    for (int b = 0; b < nb; ++b, ++s) {
      cp_wait<SW - 1>();
      __syncwarp();
      const unsigned char* src = myring + (s % SW) * S::bytes;
      if (G.expert >= 0) {
        if constexpr (kStaged)
          block_dot_n<1, NTMAX>(G.count, src, sq4 + g * (F / 4) + b * (kBlock / 4), 0,
                                sd + g * (F / kQBlock) + b * kSubPerBlock,
                                sas + g * (F / kQBlock) + b * kSubPerBlock, 0, lane, part);
        else
          block_dot_n<1, NTMAX>(G.count, src, reinterpret_cast<const int*>(src + S::act), kBlock / 4,
                                reinterpret_cast<const float*>(src + S::act_d), nullptr, kSubPerBlock, lane,
                                part);
      }
      __syncwarp();
      issue_next(s % SW);
    }
#pragma unroll
    for (int n = 0; n < NTMAX; ++n)
      if (n < G.count) P.ye[static_cast<size_t>(group_pair(P, G, n)) * H + p * kPanel + lane] = part[0][n];
    if (G.expert < 0 && lane == 0) record_status(P.status, MOE_ERR_BAD_INDEX);
    __threadfence();
    __syncwarp();
    for (int n = 0; n < G.count; ++n) down_arrive(P, group_pair(P, G, n), p, lane);
  }
  cp_wait<0>();
}

// ---------------------------------------------------------------------------
// S1 + S2 (+ S6): k_route.  CTA (i, c) copies router rows [i*W, (i+1)*W) and
// tokens [c*TC, (c+1)*TC) into shared memory, computes those logits in the
// fixed order (lane l: fma over k = l mod 32 ascending; xor-butterfly adds),
// and CTAs with i == 0 quantize their tokens to int8 32-blocks.  The last CTA
// to finish takes the top-k of every token (logit descending, ties to the
// lower id), the softmax over the selected logits, and with more than one
// token groups the (token, slot) pairs by expert.
// ---------------------------------------------------------------------------
constexpr int kRouteMaxWarps = 8;

__device__ void route_topk_token(const Decode2Params& D, int t, int lane, float* lsm, float* sel_v,
                                 int* sel_e) {
  const DecodeParams& P = D.P;
  const int E = P.n_experts, K = P.top_k;
  const float* lg = D.logits + static_cast<size_t>(t) * E;
  for (int e = lane; e < E; e += 32) lsm[e] = __ldcg(lg + e);
  __syncwarp();
  uint32_t used = 0;
  for (int r = 0; r < K; ++r) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
    for (int i = 0; i * 32 + lane < E; ++i) {
      if (used & (1u << i)) continue;
      const int e = i * 32 + lane;
      const float v = lsm[e];
      if (v > bv || (v == bv && e < be)) { bv = v; be = e; }
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, m);
      const int oe = __shfl_xor_sync(0xffffffffu, be, m);
      if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
    }
    if ((be & 31) == lane) used |= 1u << (be >> 5);
    if (lane == 0) { sel_v[r] = bv; sel_e[r] = be; }
  }
  __syncwarp();
  if (lane == 0) {
    const float l0 = sel_v[0];
    float den = 0.f;
    for (int r = 0; r < K; ++r) {
      sel_v[r] = expf(__fsub_rn(sel_v[r], l0));
      den = __fadd_rn(den, sel_v[r]);
    }
    int32_t* idx = const_cast<int32_t*>(P.idx);
    float* wts = const_cast<float*>(P.wts);
    for (int r = 0; r < K; ++r) {
      idx[static_cast<size_t>(t) * K + r] = sel_e[r];
      wts[static_cast<size_t>(t) * K + r] = __fdiv_rn(sel_v[r], den);
    }
  }
  __syncwarp();
}

// Group the pairs by expert (cnt/off/fill: shared arrays of E + 1 ints).
__device__ void route_group(const Decode2Params& D, int* cnt, int* off, int* fill, int* wsum) {
  const DecodeParams& P = D.P;
  const int E = P.n_experts, npairs = P.ntok * P.top_k;
  const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e <= E; e += nthr) { cnt[e] = 0; fill[e] = 0; }
  __syncthreads();
  for (int p = tid; p < npairs; p += nthr) {
    int e = P.idx[p];
    if (e < 0 || e >= E) e = E;
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  // exclusive scans of the pair counts and the item counts over groups 0..E:
  // thread tid owns groups [tid*per, (tid+1)*per)
  const int per = (E + 1 + nthr - 1) / nthr;
  int c_loc = 0, i_loc = 0;
  for (int q = 0; q < per; ++q) {
    const int e = tid * per + q;
    if (e <= E) { c_loc += cnt[e]; i_loc += (cnt[e] + kChunk - 1) / kChunk; }
  }
  int c_inc = c_loc, i_inc = i_loc;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const int c2 = __shfl_up_sync(0xffffffffu, c_inc, m);
    const int i2 = __shfl_up_sync(0xffffffffu, i_inc, m);
    if (lane >= m) { c_inc += c2; i_inc += i2; }
  }
  if (lane == 31) { wsum[2 * warp] = c_inc; wsum[2 * warp + 1] = i_inc; }
  __syncthreads();
  int c_base = 0, i_base = 0;
  for (int v = 0; v < warp; ++v) { c_base += wsum[2 * v]; i_base += wsum[2 * v + 1]; }
  int c_off = c_base + c_inc - c_loc, i_off = i_base + i_inc - i_loc;
  Item* items = const_cast<Item*>(P.items);
  for (int q = 0; q < per; ++q) {
    const int e = tid * per + q;
    if (e > E) break;
    off[e] = c_off;
    const int ce = cnt[e];
    for (int i = 0; i * kChunk < ce; ++i) {
      Item it;
      it.expert = e == E ? -1 : e;
      it.start = c_off + i * kChunk;
      it.count = min(kChunk, ce - i * kChunk);
      it.pad = 0;
      items[i_off++] = it;
    }
    c_off += ce;
  }
  if (tid == nthr - 1) *const_cast<int32_t*>(P.n_items) = i_base + i_inc;
  __syncthreads();
  int32_t* pairs = const_cast<int32_t*>(P.pairs);
  for (int p = tid; p < npairs; p += nthr) {
    int e = P.idx[p];
    if (e < 0 || e >= E) { record_status(P.status, MOE_ERR_BAD_INDEX); e = E; }
    pairs[off[e] + atomicAdd(&fill[e], 1)] = p;
  }
}

__global__ void __launch_bounds__(kRouteMaxWarps * 32) k_route(Decode2Params D) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const DecodeParams& P = D.P;
  const int H = P.hidden, E = P.n_experts, T = P.ntok;
  const int W = blockDim.x >> 5, TC = D.route_tc;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  int* flag = reinterpret_cast<int*>(smem + 8);
  float* wsm = reinterpret_cast<float*>(smem + 128);
  float* xsm = wsm + static_cast<size_t>(W) * H;
  const int e0 = blockIdx.x * W, ne = min(W, E - e0);
  const int t0 = blockIdx.y * TC, nt = min(TC, T - t0);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(ne + nt) * H * 4);
    bulk_g2s(wsm, D.wr + static_cast<size_t>(e0) * H, static_cast<uint32_t>(ne) * H * 4, bar,
             policy_evict_first());
  }
  pdl_wait();  // x and every output belong to the kernels before this one
  if (tid == 0)
    bulk_g2s(xsm, D.x + static_cast<size_t>(t0) * H, static_cast<uint32_t>(nt) * H * 4, bar,
             policy_evict_last());
  pdl_launch_dependents();
  if (!mbar_wait(bar, 0)) {
    record_status(P.status, MOE_ERR_TIMEOUT);
    mbar_wait(bar, 0);
    return;
  }
  if (warp < ne) {
    const float* wrow = wsm + static_cast<size_t>(warp) * H;
    for (int t = 0; t < nt; ++t) {
      const float* xr = xsm + static_cast<size_t>(t) * H;
      float p = 0.f;
      for (int k = lane; k < H; k += 32) p = __fmaf_rn(wrow[k], xr[k], p);
#pragma unroll
      for (int m = 16; m >= 1; m >>= 1) p = __fadd_rn(p, __shfl_xor_sync(0xffffffffu, p, m));
      if (lane == 0) D.logits[static_cast<size_t>(t0 + t) * E + e0 + warp] = p;
    }
  }
  {
    const int nblk = nt * (H / kQBlock);
    int8_t* xq = const_cast<int8_t*>(P.xq);
    float* xd = const_cast<float*>(P.xd);
    for (int blk = blockIdx.x * W + warp; blk < nblk; blk += gridDim.x * W) {
      const int t = blk / (H / kQBlock), j = blk % (H / kQBlock);
      const float v = xsm[static_cast<size_t>(t) * H + j * kQBlock + lane];
      const float amax = warp_max(fabsf(v));
      const float d = __fdiv_rn(amax, 127.f);
      int q = 0;
      if (d != 0.f) q = max(-127, min(127, __float2int_rn(__fdiv_rn(v, d))));
      xq[static_cast<size_t>(t0 + t) * H + j * kQBlock + lane] = static_cast<int8_t>(q);
      if (lane == 0) xd[static_cast<size_t>(t0 + t) * (H / kQBlock) + j] = d;
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const uint32_t total = gridDim.x * gridDim.y;
    *flag = (atomicAdd(D.route_cnt, 1u) == total - 1) ? 1 : 0;
  }
  __syncthreads();
  if (!*flag) return;
  __threadfence();
  // the last CTA: top-k of every token, then grouping
  float* sel_v = wsm;                                   // reuse: [W][32]
  int* sel_e = reinterpret_cast<int*>(wsm + W * kMaxTopK);
  float* lsm = wsm + 2 * W * kMaxTopK;                  // [W][E]
  for (int t = warp; t < T; t += W)
    route_topk_token(D, t, lane, lsm + static_cast<size_t>(warp) * E, sel_v + warp * kMaxTopK,
                     sel_e + warp * kMaxTopK);
  if (T > 1) {
    __threadfence();
    __syncthreads();
    int* cnt = reinterpret_cast<int*>(wsm + 2 * W * kMaxTopK);
    route_group(D, cnt, cnt + (E + 1), cnt + 2 * (E + 1), cnt + 3 * (E + 1));
  }
  if (tid == 0) atomicExch(D.route_cnt, 0u);
}

// ---------------------------------------------------------------------------
// launch
// ---------------------------------------------------------------------------
template <typename Kern>
static cudaError_t launch_pdl(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              const Decode2Params& D) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, D);
}

template <int NTMAX, bool kStaged>
static size_t gateup_smem(int H) {
  return static_cast<size_t>(kNC) * ring_depth<NTMAX>() * Slot<2, NTMAX, kStaged>::bytes +
         2 * 2 * kNC * NTMAX * 32 * 4 + (kStaged ? static_cast<size_t>(H / 4 + 2 * (H / kQBlock)) * 4 : 0);
}
template <int NTMAX, bool kStaged>
static size_t down_smem(int F, int K) {
  return static_cast<size_t>(kNC) * ring_depth<NTMAX>() * Slot<1, NTMAX, kStaged>::bytes +
         (kStaged ? static_cast<size_t>(K) * (F / 4 + 2 * (F / kQBlock)) * 4 : 0);
}

static void init_attrs2() {
  constexpr int kMaxDev = 64;
  static std::atomic<bool> done[kMaxDev];  // the attribute calls are idempotent
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < kMaxDev && done[dev].load(std::memory_order_relaxed)) return;
  const void* ks[] = {reinterpret_cast<const void*>(&k_gateup3<1, true>),
                      reinterpret_cast<const void*>(&k_gateup3<kChunk, false>),
                      reinterpret_cast<const void*>(&k_down3<1, true>),
                      reinterpret_cast<const void*>(&k_down3<kChunk, false>),
                      reinterpret_cast<const void*>(&k_route)};
  for (const void* k : ks) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
  if (dev >= 0 && dev < kMaxDev) done[dev].store(true, std::memory_order_relaxed);
}

// CTAs per SM the occupancy calculator allows, at most 2.
template <typename Kern>
static int ctas_per_sm(Kern kernel, size_t smem) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kNC * 32, smem) != cudaSuccess || n < 1) n = 1;
  return n > 2 ? 2 : n;
}

// Route CTA shape: W experts and TC tokens per CTA, with the router rows and
// the tokens of a CTA held in shared memory.
static void route_shape(int H, int E, int T, int* W, int* TC) {
  const int row = H * 4;
  int w = 2;
  while (w > 1 && w * row > 96 * 1024) --w;
  int tc = T;
  while (tc > 1 && (w + tc) * row > 192 * 1024) tc = (tc + 1) / 2;
  *W = w;
  *TC = tc;
}

static size_t route_smem_bytes(int H, int E, int W, int TC) {
  size_t a = 128 + static_cast<size_t>(W + TC) * H * 4;
  const size_t b = 128 + static_cast<size_t>(2 * W * kMaxTopK) * 4 +
                   (static_cast<size_t>(W) * E + 3 * static_cast<size_t>(E + 1) + 2 * kRouteMaxWarps) * 4;
  return a > b ? a : b;
}

int launch_route_only(Decode2Params& D, cudaStream_t stream) {
  init_attrs2();
  const DecodeParams& P = D.P;
  int W, TC;
  route_shape(P.hidden, P.n_experts, P.ntok, &W, &TC);
  D.route_warps = W;
  D.route_tc = TC;
  dim3 grid((P.n_experts + W - 1) / W, (P.ntok + TC - 1) / TC);
  cudaError_t err = launch_pdl(k_route, grid, dim3(W * 32), route_smem_bytes(P.hidden, P.n_experts, W, TC), stream, D);
  if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "route: %s", cudaGetErrorString(err));
  note_launch(MOE_K_ROUTE, stream);
  return MOE_OK;
}

int launch_decode2(Decode2Params& D, bool with_route, cudaStream_t stream) {
  init_attrs2();
  const DecodeParams& P = D.P;
  cudaError_t err = cudaSuccess;
  if (with_route) {
    int W, TC;
    route_shape(P.hidden, P.n_experts, P.ntok, &W, &TC);
    D.route_warps = W;
    D.route_tc = TC;
    dim3 grid((P.n_experts + W - 1) / W, (P.ntok + TC - 1) / TC);
    err = launch_pdl(k_route, grid, dim3(W * 32), route_smem_bytes(P.hidden, P.n_experts, W, TC), stream, D);
    if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "route: %s", cudaGetErrorString(err));
    note_launch(MOE_K_ROUTE, stream);
  }
  const dim3 block(kNC * 32);
  if (P.direct) {
    const size_t s1 = gateup_smem<1, true>(P.hidden), s2 = down_smem<1, true>(P.ffn, P.top_k);
    const int c1 = ctas_per_sm(k_gateup3<1, true>, s1), c2 = ctas_per_sm(k_down3<1, true>, s2);
    err = launch_pdl(k_gateup3<1, true>, dim3(D.n_sm * c1), block, s1, stream, D);
    if (err == cudaSuccess) note_launch(MOE_K_GATEUP, stream);
    if (err == cudaSuccess) err = launch_pdl(k_down3<1, true>, dim3(D.n_sm * c2), block, s2, stream, D);
  } else {
    const size_t s1 = gateup_smem<kChunk, false>(P.hidden), s2 = down_smem<kChunk, false>(P.ffn, P.top_k);
    const int c1 = ctas_per_sm(k_gateup3<kChunk, false>, s1), c2 = ctas_per_sm(k_down3<kChunk, false>, s2);
    err = launch_pdl(k_gateup3<kChunk, false>, dim3(D.n_sm * c1), block, s1, stream, D);
    if (err == cudaSuccess) note_launch(MOE_K_GATEUP, stream);
    if (err == cudaSuccess) err = launch_pdl(k_down3<kChunk, false>, dim3(D.n_sm * c2), block, s2, stream, D);
  }
  if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "expert_ffn: %s", cudaGetErrorString(err));
  note_launch(MOE_K_DOWN, stream);
  return check_launch("expert_ffn");
}

}  // namespace bitmoe
