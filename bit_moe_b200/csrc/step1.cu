// step1.cu -- the whole one-token decode step in one persistent kernel
// (sm_100a), for layers with hidden <= 4096, ffn <= 2048, top_k <= 8 and at
// least as many CTAs as 32-row panels of hidden.
//
// A one-token step moves a few megabytes: it is bound by latency, not by
// bandwidth, so the step's three dependent phases run inside one cooperative
// launch (every CTA resident) separated by two grid barriers:
//   A. every CTA quantizes x to int8 32-blocks in its shared memory (the same
//      result everywhere) and computes the fixed-order router logits of its
//      share of the experts;                                     -- barrier --
//   B. every CTA takes the top-k of the E logits itself (ties to the lower
//      id, so every CTA agrees), starts the bulk copies of the down-projection
//      weights it will need (its 32-row panel of hidden for each selected
//      expert) into shared memory, and computes its share of the gate/up
//      units (32-row panels of ffn, hidden blocks split over the warps),
//      writing the requantized SwiGLU codes;                    -- barrier --
//   C. each CTA with a panel of hidden finishes it: warp j multiplies slot j's
//      codes with the prefetched down weights, and the slots are summed in
//      order (no atomics).
// Parakon Runtime README, "How it works" (fused decode mat-vecs on the packed
// blocks, int8 activations); llama-modchip page, "Key highlights" (all top-k
// experts evaluated); pxq_llama README, "Updates -- 2026-07-28" (gate/up with
// the SiLU unary).  The numerics are those of the decode kernels.
#include "bitmoe.h"
#include "common.cuh"
#include "decode2.cuh"
#include "matvec.cuh"
#include "ptx.cuh"

namespace bitmoe {

constexpr int kS1MaxH = 4096, kS1MaxF = 2048, kS1MaxK = 8;
constexpr uint32_t kSpinLimit = 1u << 24;

struct Step1Params {
  Decode2Params D;
  uint32_t* bar_count;  // 64-bit grid barrier ticket counter (only grows)
  uint32_t* bar_gen;    // unused
};

struct Step1Layout {
  size_t ring, pref, xq4, xd, xas, lg, sel, red, flag, xf, act, total;
};

// Shared-memory plan of one CTA (x fp32 and the down activations alias the
// gate/up ring; the router rows alias the down prefetch area).
__host__ __device__ inline Step1Layout step1_layout(int H, int F, int E, int K) {
  Step1Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = (off + bytes + 127) / 128 * 128;
    return o;
  };
  const size_t ring = static_cast<size_t>(kNC) * ring_depth<1>() * Slot<2, 1, true>::bytes;
  const size_t xf = static_cast<size_t>(H) * 4;
  const size_t act = static_cast<size_t>(K) * (F + 2 * (F / kQBlock) * 4);
  L.ring = take(ring > xf ? (ring > act ? ring : act) : (xf > act ? xf : act));
  L.xf = L.ring;
  L.act = L.ring;
  const size_t pref = static_cast<size_t>(K) * (F / kBlock) * kMatBytes;
  const size_t rows = static_cast<size_t>(2) * H * 4;  // at most two router rows per CTA
  L.pref = take(pref > rows ? pref : rows);
  L.xq4 = take(static_cast<size_t>(H));
  L.xd = take(static_cast<size_t>(H / kQBlock) * 4);
  L.xas = take(static_cast<size_t>(H / kQBlock) * 4);
  L.lg = take(static_cast<size_t>(E) * 4);
  L.sel = take(2 * kMaxTopK * 4);
  L.red = take(2 * 2 * kNC * 32 * 4);
  L.flag = take(64);
  L.total = off;
  return L;
}

// Grid barrier in two halves (all CTAs are resident: cooperative launch), so
// that a CTA can work between announcing its arrival and waiting for the
// others.  grid_arrive returns the generation to wait on; grid_wait is
// bounded and returns false, with MOE_ERR_TIMEOUT recorded, if the other CTAs
// did not arrive.
__device__ __forceinline__ uint64_t grid_arrive(const Step1Params& S) {
  __syncthreads();
  uint64_t target = 0;
  if (threadIdx.x == 0) {
    __threadfence();
    // tickets of one barrier round are consecutive: every CTA arrives at round
    // r before any CTA leaves it, so round r owns tickets [r*C, (r+1)*C)
    const unsigned long long t = atomicAdd(reinterpret_cast<unsigned long long*>(S.bar_count), 1ull);
    target = (t / gridDim.x + 1) * gridDim.x;
  }
  return target;
}

__device__ __forceinline__ bool grid_wait(const Step1Params& S, uint64_t target, volatile int* abort) {
  if (threadIdx.x == 0 && !*abort) {
    uint32_t polls = 0;
    for (;;) {
      uint64_t v;
      asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(S.bar_count) : "memory");
      if (v >= target) break;
      if (++polls > kSpinLimit) {
        record_status(S.D.P.status, MOE_ERR_TIMEOUT);
        *abort = 1;
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();
  return !*abort;
}

__device__ __forceinline__ bool grid_sync(const Step1Params& S, volatile int* abort) {
  return grid_wait(S, grid_arrive(S), abort);
}

// Order-preserving map of an fp32 value to uint32 (larger value, larger key).
__device__ __forceinline__ uint32_t f32_key(float v) {
  const uint32_t b = __float_as_uint(v == 0.f ? 0.f : v);  // -0 ranks as +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__global__ void __launch_bounds__(kNC * 32, 1) k_step1(Step1Params S1) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const Decode2Params& D = S1.D;
  const DecodeParams& P = D.P;
  const int H = P.hidden, F = P.ffn, E = P.n_experts, K = P.top_k;
  const int nbH = H / kBlock, nbF = F / kBlock;
  const int C = gridDim.x, c = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Step1Layout L = step1_layout(H, F, E, K);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L.flag);
  uint64_t* pbar = reinterpret_cast<uint64_t*>(smem + L.flag + 16);
  int* sq4 = reinterpret_cast<int*>(smem + L.xq4);
  float* sxd = reinterpret_cast<float*>(smem + L.xd);
  int* sxas = reinterpret_cast<int*>(smem + L.xas);
  float* lg = reinterpret_cast<float*>(smem + L.lg);
  int* sel_e = reinterpret_cast<int*>(smem + L.sel);
  float* sel_w = reinterpret_cast<float*>(smem + L.sel + kMaxTopK * 4);
  float* xf = reinterpret_cast<float*>(smem + L.xf);
  float* rows = reinterpret_cast<float*>(smem + L.pref);
  if (tid == 0) {
    *abort = 0;
    mbar_init(pbar, K);
    fence_mbar_init();
  }

  // ---------------- phase A: x, int8 x^, logits of this CTA's experts
  const int e0 = static_cast<int>(static_cast<int64_t>(E) * c / C);
  const int e1 = static_cast<int>(static_cast<int64_t>(E) * (c + 1) / C);
  for (int q = tid; q < H * 4 / 16; q += blockDim.x)
    cp16(reinterpret_cast<unsigned char*>(xf) + q * 16, reinterpret_cast<const unsigned char*>(D.x) + q * 16);
  for (int q = tid; q < (e1 - e0) * H * 4 / 16; q += blockDim.x)
    cp16(reinterpret_cast<unsigned char*>(rows) + q * 16,
         reinterpret_cast<const unsigned char*>(D.wr + static_cast<size_t>(e0) * H) + q * 16);
  cp_commit();
  cp_wait<0>();
  __syncthreads();
  if (warp < e1 - e0) {
    const float* wrow = rows + static_cast<size_t>(warp) * H;
    float p = 0.f;
#pragma unroll 16
    for (int k = lane; k < H; k += 32) p = __fmaf_rn(wrow[k], xf[k], p);
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) p = __fadd_rn(p, __shfl_xor_sync(0xffffffffu, p, m));
    if (lane == 0) D.logits[e0 + warp] = p;
  }
  const uint64_t gen1 = grid_arrive(S1);
  for (int blk = warp; blk < H / kQBlock; blk += kNC) {
    const float v = xf[blk * kQBlock + lane];
    const float amax = warp_max(fabsf(v));
    const float d = __fdiv_rn(amax, 127.f);
    int q = 0;
    if (d != 0.f) q = max(-127, min(127, __float2int_rn(__fdiv_rn(v, d))));
    reinterpret_cast<int8_t*>(sq4)[blk * kQBlock + lane] = static_cast<int8_t>(q);
    if (lane == 0) sxd[blk] = d;
    if (c == 0) {
      const_cast<int8_t*>(P.xq)[blk * kQBlock + lane] = static_cast<int8_t>(q);
      if (lane == 0) const_cast<float*>(P.xd)[blk] = d;
    }
  }
  __syncthreads();
  for (int i = tid; i < H / kQBlock; i += blockDim.x) {
    int sum = 0;
#pragma unroll
    for (int j = 0; j < kQBlock / 4; ++j) sum = __dp4a(sq4[i * 8 + j], 0x01010101, sum);
    sxas[i] = sum;
  }
  if (!grid_wait(S1, gen1, abort)) return;

  // ---------------- phase B: top-k (every CTA), down prefetch, gate/up
  if (warp == 0) {
    for (int e = lane; e < E; e += 32) lg[e] = __ldcg(D.logits + e);
    __syncwarp();
    // the K largest logits, larger first, equal logits by lower id: per round
    // the largest key over the warp, then the lowest id holding it
    uint32_t used = 0;
    for (int r = 0; r < K; ++r) {
      uint32_t bk = 0;
      int be = 0x7fffffff;
      for (int i = 0; i * 32 + lane < E; ++i) {
        if (used & (1u << i)) continue;
        const uint32_t k = f32_key(lg[i * 32 + lane]);
        if (k > bk) { bk = k; be = i * 32 + lane; }  // ascending ids: keep the first
      }
      const uint32_t wk = __reduce_max_sync(0xffffffffu, bk);
      const int we = static_cast<int>(__reduce_min_sync(0xffffffffu, bk == wk ? static_cast<uint32_t>(be) : 0xffffffffu));
      if ((we & 31) == lane) used |= 1u << (we >> 5);
      if (lane == 0) { sel_e[r] = we; sel_w[r] = lg[we]; }
    }
    __syncwarp();
    if (lane == 0) {
      const float l0 = sel_w[0];
      float den = 0.f;
      for (int r = 0; r < K; ++r) {
        sel_w[r] = expf(__fsub_rn(sel_w[r], l0));
        den = __fadd_rn(den, sel_w[r]);
      }
      for (int r = 0; r < K; ++r) {
        sel_w[r] = __fdiv_rn(sel_w[r], den);
        if (c == 0) {
          const_cast<int32_t*>(P.idx)[r] = sel_e[r];
          const_cast<float*>(P.wts)[r] = sel_w[r];
        }
      }
    }
  }
  __syncthreads();
  // down prefetch: this CTA's panel of hidden for every slot (one issuing
  // thread per slot: the panel's blocks are contiguous, one copy for the
  // digits and one for the scales)
  const int panelH = c;  // C >= hidden/32: at most one panel per CTA
  const bool has_panel = panelH < H / kPanel;
  unsigned char* pref = smem + L.pref;
  const size_t pref_slot = static_cast<size_t>(nbF) * kMatBytes;
  if (has_panel && tid < K) {
    const int j = tid;
    const size_t pb0 = (static_cast<size_t>(sel_e[j]) * (H / kPanel) + panelH) * nbF;
    unsigned char* dst = pref + j * pref_slot;
    const uint32_t tb = static_cast<uint32_t>(nbF) * kBlockWords * kPanel * 4;
    const uint32_t sb = static_cast<uint32_t>(nbF) * kPanel * 2;
    mbar_arrive_expect_tx(pbar, tb + sb);
    bulk_g2s(dst, P.down_trits + pb0 * kBlockWords * kPanel, tb, pbar, policy_evict_first());
    bulk_g2s(dst + tb, P.down_scales + pb0 * kPanel, sb, pbar, policy_evict_first());
  }
  // gate/up: units (slot, 32-row panel of ffn); blocks of hidden split by warp
  {
    using SL = Slot<2, 1, true>;
    constexpr int SW = ring_depth<1>();
    const int panels = F / kPanel;
    const int64_t U = static_cast<int64_t>(K) * panels;
    int64_t u0, u1;
    cta_range(U, c, C, u0, u1);
    unsigned char* myring = smem + L.ring + static_cast<size_t>(warp) * SW * SL::bytes;
    float* red = reinterpret_cast<float*>(smem + L.red);
    int64_t iu = u0;
    int ib = warp;
    auto issue_next = [&](int slot) {
      while (iu < u1 && ib >= nbH) { ++iu; ib = warp; }
      if (iu < u1) {
        Group G;
        G.expert = sel_e[iu / panels];
        G.count = 1;
        G.start = static_cast<int>(iu / panels);
        ActSrc<1> A{};
        issue_item<2, 1, true>(myring + slot * SL::bytes, P, G, A, static_cast<int>(iu % panels), ib, lane);
        ib += kNC;
      }
      cp_commit();
    };
#pragma unroll
    for (int k = 0; k < SW; ++k) issue_next(k);
    int s = 0, ui = 0;
    for (int64_t u = u0; u < u1; ++u, ++ui) {
      const int j = static_cast<int>(u / panels), p = static_cast<int>(u % panels);
      float part[2][1] = {{0.f}, {0.f}};
      for (int b = warp; b < nbH; b += kNC, ++s) {
        cp_wait<SW - 1>();
        __syncwarp();
        block_dot<2, 1, 1>(myring + (s % SW) * SL::bytes, sq4 + b * (kBlock / 4), 0, sxd + b * kSubPerBlock,
                           sxas + b * kSubPerBlock, 0, lane, part);
        __syncwarp();
        issue_next(s % SW);
      }
      float* rb = red + (ui & 1) * (2 * kNC * 32);
      rb[(0 * kNC + warp) * 32 + lane] = part[0][0];
      rb[(1 * kNC + warp) * 32 + lane] = part[1][0];
      __syncthreads();
      if (warp == 0) {
        float g = 0.f, uu = 0.f;
        const int nw = nbH < kNC ? nbH : kNC;
        for (int v = 0; v < nw; ++v) {
          g = __fadd_rn(g, rb[(0 * kNC + v) * 32 + lane]);
          uu = __fadd_rn(uu, rb[(1 * kNC + v) * 32 + lane]);
        }
        const float a = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.f, expf(-g))), uu);
        const float amax = warp_max(fabsf(a));
        const float dd = __fdiv_rn(amax, 127.f);
        int q = 0;
        if (dd != 0.f) q = max(-127, min(127, __float2int_rn(__fdiv_rn(a, dd))));
        P.aq[static_cast<size_t>(j) * F + p * kPanel + lane] = static_cast<int8_t>(q);
        if (lane == 0) P.ad[static_cast<size_t>(j) * (F / kQBlock) + p] = dd;
      }
    }
    cp_wait<0>();
  }
  const bool synced = grid_sync(S1, abort);

  // ---------------- phase C: this CTA's panel of hidden, all slots
  if (has_panel) {
    // the prefetch must land before this CTA reads it or exits
    bool ok = mbar_wait(pbar, 0);
    if (!ok) record_status(P.status, MOE_ERR_TIMEOUT);
    if (synced && ok) {
      int* aq4 = reinterpret_cast<int*>(smem + L.act);                       // [K][F/4]
      float* ad = reinterpret_cast<float*>(aq4 + K * (F / 4));                 // [K][F/32]
      int* aas = reinterpret_cast<int*>(ad + K * (F / kQBlock));              // [K][F/32]
      float* part = reinterpret_cast<float*>(smem + L.red);                  // [K][32]
      for (int q = tid; q < K * (F / 4); q += blockDim.x)
        aq4[q] = __ldcg(reinterpret_cast<const int*>(P.aq) + q);
      for (int q = tid; q < K * (F / kQBlock); q += blockDim.x) ad[q] = __ldcg(P.ad + q);
      __syncthreads();
      for (int q = tid; q < K * (F / kQBlock); q += blockDim.x) {
        int sum = 0;
#pragma unroll
        for (int j = 0; j < kQBlock / 4; ++j) sum = __dp4a(aq4[q * 8 + j], 0x01010101, sum);
        aas[q] = sum;
      }
      __syncthreads();
      for (int j = warp; j < K; j += kNC) {
        float acc[1][1] = {{0.f}};
        const unsigned char* wj = pref + j * pref_slot;
        for (int b = 0; b < nbF; ++b) {
          const int scale_off = nbF * kBlockWords * kPanel * 4 + b * kPanel * 2 - b * kBlockWords * kPanel * 4;
          block_dot<1, 1, 1>(wj + static_cast<size_t>(b) * kBlockWords * kPanel * 4,
                             aq4 + j * (F / 4) + b * (kBlock / 4), 0,
                             ad + j * (F / kQBlock) + b * kSubPerBlock, aas + j * (F / kQBlock) + b * kSubPerBlock,
                             0, lane, acc, scale_off);
        }
        part[j * 32 + lane] = acc[0][0];
      }
      __syncthreads();
      if (warp == 0) {
        float y = 0.f;
        for (int j = 0; j < K; ++j) y = __fmaf_rn(sel_w[j], part[j * 32 + lane], y);
        P.y[panelH * kPanel + lane] = y;
      }
    }
  }
}

bool step1_supported(const DecodeParams& P, int n_sm, size_t* smem) {
  if (P.ntok != 1 || P.hidden > kS1MaxH || P.ffn > kS1MaxF || P.top_k > kS1MaxK) return false;
  if (P.hidden / kPanel > n_sm) return false;
  if (P.n_experts > 2 * n_sm) return false;  // at most two router rows per CTA
  const Step1Layout L = step1_layout(P.hidden, P.ffn, P.n_experts, P.top_k);
  *smem = L.total;
  return L.total <= static_cast<size_t>(kMaxDynSmem);
}

int launch_step1(const Decode2Params& D, uint32_t* bar_count, uint32_t* bar_gen, cudaStream_t stream) {
  static bool done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !done[dev]) {
    cudaFuncSetAttribute(k_step1, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
    done[dev] = true;
  }
  size_t smem = 0;
  if (!step1_supported(D.P, D.n_sm, &smem)) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "step1: unsupported shape");
  Step1Params S{D, bar_count, bar_gen};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(D.n_sm);
  cfg.blockDim = dim3(kNC * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(&cfg, k_step1, S);
  if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "step1: %s", cudaGetErrorString(err));
  note_launch(MOE_K_STEP1, stream);
  return check_launch("step1");
}

}  // namespace bitmoe
