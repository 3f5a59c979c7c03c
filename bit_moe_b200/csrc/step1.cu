// step1.cu -- the whole one-token decode step in one persistent kernel
// (sm_100a), for layers with hidden <= 4096, ffn <= 2048, top_k <= 8 and at
// least as many CTAs as 32-row panels of hidden.
//
// A one-token step moves a few megabytes: it is bound by latency, not by
// bandwidth, so the step's three dependent phases run inside one cooperative
// launch (every CTA resident), handing data over through L2 as values tagged
// with the launch's generation instead of grid-wide barriers:
//   A. every CTA quantizes x to int8 32-blocks in its shared memory (the same
//      result everywhere) and publishes the fixed-order router logits of its
//      share of the experts, each tagged;
//   B. every CTA polls the E tagged logits until all carry this launch's tag,
//      takes the top-k itself (ties to the lower id, so every CTA agrees),
//      starts the bulk copies of the down-projection weights it will need (its
//      32-row panel of hidden for each selected expert) into shared memory,
//      and computes its share of the gate/up units (32-row panels of ffn) in
//      two streams of 8 warps, the hidden blocks of a unit split over a
//      stream's warps; each finished unit publishes its requantized SwiGLU
//      codes, scale and code sum as tagged words;
//   C. each CTA with a panel of hidden splits every slot's ffn blocks over two
//      warps, which start as soon as the units of their blocks carry this
//      launch's tag, multiply them with the prefetched down weights, and one
//      warp applies the block scales and sums the slots in order (no atomics
//      on data).
// Parakon Runtime README, "How it works" (fused decode mat-vecs on the packed
// blocks, int8 activations); llama-modchip page, "Key highlights" (all top-k
// experts evaluated); pxq_llama README, "Updates -- 2026-07-28" (gate/up with
// the SiLU unary).  The numerics are those of the decode kernels.  The same
// kernel takes 1-bit sign codes (pxq_llama README, "What's PXQ?", the PXQ1
// tier) with their block decode, and two-level scales (an fp16 anchor per row,
// a 4-bit sub-scale per 16 weights): their down rows keep one fp32 chain over
// every sub-block, so phase C's items leave the blocks' exact integer sums
// and one warp per slot chains them in order.
#include <atomic>
#include "bitmoe.h"
#include "common.cuh"
#include "decode2.cuh"
#include "matvec.cuh"
#include "ptx.cuh"
#include "shared.cuh"
#include "topk.cuh"

namespace bitmoe {

constexpr int kS1MaxH = 4096, kS1MaxF = 2048, kS1MaxK = 8;
constexpr uint32_t kSpinLimit = 1u << 22;  // polls before a wait gives up (seconds)
// Two gate/up streams of kNC warps per CTA: each stream computes one unit at a
// time with the block split and summation order of the grouped decode kernels,
// and the two streams of an SM run different units side by side.
constexpr int kS1Streams = 2;
constexpr int kS1Warps = kS1Streams * kNC;
constexpr int kS1MaxE = kNC * 32;          // experts: one per lane of the polling warp's kPer rounds
// One 128-byte line per tagged logit, so that the CTAs polling the logits
// spread their loads over many L2 lines instead of queueing on a few.
constexpr int kTagStride = 16;
static_assert(kS1MaxK <= kNC, "phase C: one warp per slot");

// One finished gate/up unit (slot j, 32-row panel p of ffn) is published as
// kUnitWords tagged words: its 32 int8 codes four to a word, the fp32 scale
// and the int32 code sum.
constexpr int kUnitWords = kPanel / 4 + 2;

// Bytes of one 256-weight block of a 32-row panel: packed words, then the
// 32 fp16 scales (base-3 digits, or 1-bit sign codes), or for two-level
// scales the rows' 4-bit sub-scale code words (their per-row fp16 anchors
// come once per panel).
__host__ __device__ constexpr int s1_word_bytes(int fmt) {
  return (fmt == MOE_FORMAT_SIGN ? kSignWords : kBlockWords) * kPanel * 4;
}
__host__ __device__ constexpr int s1_tail_bytes(int fmt) {
  return fmt == MOE_FORMAT_E16 ? kE16Words * kPanel * 4 : kPanel * 2;
}
__host__ __device__ constexpr int s1_mat_bytes(int fmt) { return s1_word_bytes(fmt) + s1_tail_bytes(fmt); }
// Per-block results phase C keeps in shared memory: the inner sum and the
// weight scale, or for two-level scales the 8 sub-blocks' integer sums.
__host__ __device__ constexpr int s1_item_words(int fmt) { return fmt == MOE_FORMAT_E16 ? kSubPerBlock : 2; }

struct Step1Params {
  Decode2Params D;
  unsigned long long* ticket;  // launch ticket counter (only grows): generation = ticket / CTAs
  unsigned long long* tagged;  // [E][kTagStride] logits as (generation + 1) << 32 | fp32 bits
  unsigned long long* units;   // [top_k][ffn/32][kUnitWords] unit outputs, tagged the same way
  // the shared expert (kShared): its 32-row blocks of the shared ffn are
  // units after the routed ones, published to sunits [ffn_s/32][kUnitWords]
  SharedParams S;
  unsigned long long* sunits;
};

struct Step1Layout {
  size_t ring, pref, xq4, xd, xas, sel, red, flag, rbar, shr, xf, act, inner, total;
  int sw;  // ring slots per warp
};

// Shared-memory plan of one CTA.  x in fp32, the logits and the down
// activations alias the gate/up ring (which is used only between them); the
// router rows alias the down prefetch area.  Three ring slots per warp where
// they fit, else two, else one (two-level scales at the largest shapes).
__host__ __device__ inline Step1Layout step1_layout(int H, int F, int E, int K, int fmt) {
  Step1Layout L{};
  for (int sw = 3; sw >= 1; --sw) {
    L = Step1Layout{};
    L.sw = sw;
    size_t off = 0;
    auto take = [&](size_t bytes) {
      const size_t o = off;
      off = (off + bytes + 127) / 128 * 128;
      return o;
    };
    size_t ring = static_cast<size_t>(kS1Warps) * sw * 2 * s1_mat_bytes(fmt);
    const size_t xf = static_cast<size_t>(H) * 4;
    const size_t act = static_cast<size_t>(K) * (F + 2 * (F / kQBlock) * 4);
    const size_t inner = static_cast<size_t>(s1_item_words(fmt)) * K * (F / kBlock) * kPanel * 4;
    if (ring < xf) ring = xf;
    // phase C also keeps a shared expert's block codes and scales after the
    // inner sums
    const size_t scodes = static_cast<size_t>(kMaxSharedUnits) * (kPanel / 4 + 1) * 4;
    if (ring < act + inner + scodes) ring = act + inner + scodes;
    L.ring = take(ring);
    L.act = L.ring;
    L.inner = L.ring + act;
    L.xf = L.ring;
    const size_t pref = static_cast<size_t>(K) * ((F / kBlock) * s1_mat_bytes(fmt) + (fmt == MOE_FORMAT_E16 ? kPanel * 2 : 0));
    const size_t rows = static_cast<size_t>(2) * H * 4;  // at most two router rows per CTA
    L.pref = take(pref > rows ? pref : rows);
    L.xq4 = take(static_cast<size_t>(H));
    L.xd = take(static_cast<size_t>(H / kQBlock) * 4);
    L.xas = take(static_cast<size_t>(H / kQBlock) * 4);
    L.sel = take(2 * kMaxTopK * 4);
    L.red = take(static_cast<size_t>(kS1Streams) * 2 * kNC * 32 * 4);
    L.flag = take(64);
    L.rbar = take(static_cast<size_t>(kS1Warps) * 3 * 8);
    L.shr = take(static_cast<size_t>(kS1Streams + 1) * 32 * 4);  // shared expert: a of a block per stream, down rows
    L.total = off;
    if (L.total <= static_cast<size_t>(kMaxDynSmem)) break;
  }
  return L;
}

// Named barriers of gate/up stream h (kNC warps each): the unit's partial
// sums are written (the unit's epilogue warp syncs, the others arrive), and
// read by the epilogue warp (it arrives, the other warps sync before they
// overwrite them).
__device__ __forceinline__ void stream_bar_sync(int id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(kNC * 32) : "memory");
}
__device__ __forceinline__ void stream_bar_arrive(int id) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "n"(kNC * 32) : "memory");
}

// Bring a range of global memory into L2 (16-byte aligned, a multiple of 16
// bytes), without waiting for it.
__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Bounded polls of values another CTA publishes.
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// kFmt: the weights' format (base-3 digits, 1-bit sign codes or two-level
// scales).  kSlotOrder:
// the down items go to the warps in slot order (at most two items per warp),
// else by halves of a slot.  kShared: the layer's shared expert (8-bit
// blocks) is computed in the same launch: its 32-row blocks of the shared
// ffn are gate/up units after the routed ones (on the streams the routed
// units leave idle), and the CTAs with a panel of hidden add the panel's
// rows of its down projection to y after the routed combine, with the
// arithmetic of the shared expert's own kernels.
template <int kFmt, bool kSlotOrder, bool kShared>
__global__ void __launch_bounds__(kS1Warps * 32, 1) k_step1(Step1Params S1) {
  constexpr bool kSign = kFmt == MOE_FORMAT_SIGN, kE16 = kFmt == MOE_FORMAT_E16;
  static_assert(!kE16 || kSlotOrder, "two-level scales take the down items in slot order");
  constexpr int kWBytes = s1_word_bytes(kFmt), kMat = s1_mat_bytes(kFmt);
  constexpr int kWords = kSign ? kSignWords : kBlockWords;
  extern __shared__ __align__(1024) unsigned char smem[];
  const Decode2Params& D = S1.D;
  const DecodeParams& P = D.P;
  const int H = P.hidden, F = P.ffn, E = P.n_experts, K = P.top_k;
  const int nbH = H / kBlock, nbF = F / kBlock;
  const int C = gridDim.x, c = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Step1Layout L = step1_layout(H, F, E, K, kFmt);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L.flag);
  uint64_t* pbar = reinterpret_cast<uint64_t*>(smem + L.flag + 16);
  int* sq4 = reinterpret_cast<int*>(smem + L.xq4);
  float* sxd = reinterpret_cast<float*>(smem + L.xd);
  int* sxas = reinterpret_cast<int*>(smem + L.xas);
  int* sel_e = reinterpret_cast<int*>(smem + L.sel);
  float* sel_w = reinterpret_cast<float*>(smem + L.sel + kMaxTopK * 4);
  float* xf = reinterpret_cast<float*>(smem + L.xf);
  float* rows = reinterpret_cast<float*>(smem + L.pref);
  uint32_t* sgen = reinterpret_cast<uint32_t*>(smem + L.flag + 32);
  uint64_t* rbar = reinterpret_cast<uint64_t*>(smem + L.rbar);  // [warp][ring slot]
  if (tid == 0) {
    *abort = 0;
    mbar_init(pbar, K);
    for (int i = 0; i < kS1Warps * L.sw; ++i) mbar_init(rbar + i, 1);
    fence_mbar_init();
    // every CTA takes one ticket per launch, so the tickets of a launch are
    // [g*C, (g+1)*C) and ticket / C is the same generation g in every CTA;
    // the logits of this launch carry the tag g + 1
    const uint32_t g = static_cast<uint32_t>(atomicAdd(S1.ticket, 1ull) / static_cast<unsigned long long>(C));
    *sgen = g + 1u;
  }

  // ---------------- phase A: x, int8 x^, logits of this CTA's experts
  // The router rows are caller data that no kernel of this library writes,
  // so their copy starts before the dependency wait below.
  const int e0 = static_cast<int>(static_cast<int64_t>(E) * c / C);
  const int e1 = static_cast<int>(static_cast<int64_t>(E) * (c + 1) / C);
  for (int q = tid; q < (e1 - e0) * H * 4 / 16; q += blockDim.x)
    cp16(reinterpret_cast<unsigned char*>(rows) + q * 16,
         reinterpret_cast<const unsigned char*>(D.wr + static_cast<size_t>(e0) * H) + q * 16);
  cp_commit();
  if constexpr (kShared) {
    // the shared expert's gate/up blocks this CTA will compute: into L2 now
    // (caller data, like the router rows)
    if (tid == 0) {
      const int64_t U = static_cast<int64_t>(K) * (F / kPanel), Us = S1.S.ffn / kQBlock;
      for (int64_t q = 0;; ++q) {
        const int64_t u = q == 0 ? static_cast<int64_t>(c) : q * C + (C - 1 - c);
        if (u >= U + Us) break;
        if (u < U) continue;
        const int64_t f0 = (u - U) * kQBlock;
        bulk_prefetch_l2(S1.S.gate_q + f0 * H, static_cast<uint32_t>(kQBlock * H));
        bulk_prefetch_l2(S1.S.up_q + f0 * H, static_cast<uint32_t>(kQBlock * H));
        bulk_prefetch_l2(S1.S.gate_d + f0 * (H / kQBlock), static_cast<uint32_t>(2 * H));
        bulk_prefetch_l2(S1.S.up_d + f0 * (H / kQBlock), static_cast<uint32_t>(2 * H));
      }
    }
  }

  // launched as a programmatic dependent: everything the kernels before it
  // wrote (x among them) is visible only past this wait
  pdl_wait();

  for (int q = tid; q < H * 4 / 16; q += blockDim.x)
    cp16(reinterpret_cast<unsigned char*>(xf) + q * 16, reinterpret_cast<const unsigned char*>(D.x) + q * 16);
  cp_commit();
  cp_wait<0>();
  __syncthreads();
  // the next kernel may start launching (its CTAs become resident as this
  // launch's CTAs leave their SMs, then wait in pdl_wait for this launch to
  // complete); every CTA of this launch holds its ticket by now
  pdl_launch_dependents();
  const int nrows = e1 - e0;
  const uint32_t tag = *sgen;
  if (warp < nrows) {
    const float* wrow = rows + static_cast<size_t>(warp) * H;
    float p = 0.f;
#pragma unroll 16
    for (int k = lane; k < H; k += 32) p = __fmaf_rn(wrow[k], xf[k], p);
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) p = __fadd_rn(p, __shfl_xor_sync(0xffffffffu, p, m));
    // the tagged value is all a reader needs: no ordering with other data
    if (lane == 0) st_relaxed_u64(S1.tagged + static_cast<size_t>(e0 + warp) * kTagStride, (static_cast<unsigned long long>(tag) << 32) | __float_as_uint(p));
  }
  if (warp == 0) {
    // ---------------- phase B: poll the E logits of this launch (all loads of
    // a round in flight at once), then the top-k, while the other warps
    // quantize x.  (The wait test knob makes this poll wait for the next
    // generation's tag, which no CTA of this launch publishes, with its own
    // poll budget.)
    const int32_t* knob = reinterpret_cast<const int32_t*>(P.status);
    const uint32_t want = tag + (knob[kWsKnobMode] == kKnobStep1Tag ? 1u : 0u);
    const uint32_t limit = knob[kWsKnobPolls] ? static_cast<uint32_t>(knob[kWsKnobPolls]) : kSpinLimit;
    constexpr int kPer = kS1MaxE / 32;
    unsigned long long v[kPer];
    uint32_t ready = 0, need = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (lane + 32 * i < E) need |= 1u << i;
    for (uint32_t polls = 0; ready != need; ++polls) {
      if (polls > limit) break;
#pragma unroll
      for (int i = 0; i < kPer; ++i)
        if ((need & ~ready) & (1u << i)) v[i] = ld_relaxed_u64(S1.tagged + static_cast<size_t>(lane + 32 * i) * kTagStride);
#pragma unroll
      for (int i = 0; i < kPer; ++i)
        if (((need & ~ready) & (1u << i)) && static_cast<uint32_t>(v[i] >> 32) == want) ready |= 1u << i;
    }
    if (!__all_sync(0xffffffffu, ready == need)) {
      if (lane == 0) {
        record_status(P.status, MOE_ERR_TIMEOUT);
        *abort = 1;
      }
    } else {
      // the top-k and the renormalised softmax over it
      uint32_t key[kPer];
#pragma unroll
      for (int i = 0; i < kPer; ++i) key[i] = f32_key(__uint_as_float(static_cast<uint32_t>(v[i])));
      int my_e;
      float w;
      warp_topk_softmax<kPer>(key, need, K, lane, my_e, w);
      if (lane < K) {
        sel_e[lane] = my_e;
        sel_w[lane] = w;
        if (c == 0) {
          const_cast<int32_t*>(P.idx)[lane] = my_e;
          const_cast<float*>(P.wts)[lane] = w;
        }
      }
    }
  } else {
    // x -> int8 32-blocks, kU blocks per warp at a time so that the
    // reductions and divisions of independent blocks overlap
    constexpr int kU = 8;
    const int nblk = H / kQBlock, nqw = kS1Warps - 1;
    for (int b0 = warp - 1; b0 < nblk; b0 += nqw * kU) {
      float xv[kU], am[kU];
#pragma unroll
      for (int i = 0; i < kU; ++i) {
        const int blk = b0 + i * nqw;
        xv[i] = blk < nblk ? xf[blk * kQBlock + lane] : 0.f;
        am[i] = fabsf(xv[i]);
      }
#pragma unroll
      for (int m = 16; m >= 1; m >>= 1)
#pragma unroll
        for (int i = 0; i < kU; ++i) am[i] = fmaxf(am[i], __shfl_xor_sync(0xffffffffu, am[i], m));
#pragma unroll
      for (int i = 0; i < kU; ++i) {
        const int blk = b0 + i * nqw;
        if (blk < nblk) {
          const float d = __fdiv_rn(am[i], 127.f);
          int q = 0;
          if (d != 0.f) q = max(-127, min(127, __float2int_rn(__fdiv_rn(xv[i], d))));
          reinterpret_cast<int8_t*>(sq4)[blk * kQBlock + lane] = static_cast<int8_t>(q);
          const int qs = __reduce_add_sync(0xffffffffu, q);
          if (lane == 0) {
            sxd[blk] = d;
            sxas[blk] = qs;
          }
          if (c == 0) {
            const_cast<int8_t*>(P.xq)[blk * kQBlock + lane] = static_cast<int8_t>(q);
            if (lane == 0) const_cast<float*>(P.xd)[blk] = d;
          }
        }
      }
    }
  }
  __syncthreads();
  if (*abort) return;
  // down prefetch (issued after the first gate/up copies): this CTA's panel
  // of hidden for every slot, one issuing thread per slot (the panel's blocks
  // are contiguous: one copy for the digits and one for the scales)
  const int panelH = c;  // C >= hidden/32: at most one panel per CTA
  const bool has_panel = panelH < H / kPanel;
  unsigned char* pref = smem + L.pref;
  const size_t pref_slot = static_cast<size_t>(nbF) * kMat + (kE16 ? kPanel * 2 : 0);  // E16: + the rows' anchors
  // gate/up: units (slot, 32-row panel of ffn); stream h of this CTA takes
  // every other unit of the CTA's list, the blocks of hidden of a unit split
  // over the stream's warps
  {
    constexpr int kSlotBytes = 2 * kMat;  // gate, then up: words and scales each
    const int SW = L.sw;
    const int panels = F / kPanel;
    const int64_t U = static_cast<int64_t>(K) * panels;
    const int h = warp / kNC, w8 = warp % kNC;
    // this CTA's units: unit c first, then in each later round the unit
    // counted from the round's end, so that the extra units fall on the
    // highest CTA ids (those without a panel of hidden) and the slots of the
    // first round are complete first; stream h takes rounds h, h+2, ...
    auto unit_of = [&](int q) -> int64_t {
      return q == 0 ? static_cast<int64_t>(c) : static_cast<int64_t>(q) * C + (C - 1 - c);
    };
    int nmine = 0;  // routed units; the shared expert's units come after them
    while (unit_of(kS1Streams * nmine + h) < U) ++nmine;
    int nshared = 0;
    if constexpr (kShared)
      while (unit_of(kS1Streams * (nmine + nshared) + h) < U + S1.S.ffn / kQBlock) ++nshared;
    auto my_unit = [&](int i) { return unit_of(kS1Streams * i + h); };
    unsigned char* myring = smem + L.ring + static_cast<size_t>(warp) * SW * kSlotBytes;
    float* rb = reinterpret_cast<float*>(smem + L.red) + h * (2 * kNC * 32);
    const int bar_done = 1 + h, bar_free = 1 + kS1Streams + h;
    const unsigned long long tag64 = static_cast<unsigned long long>(*sgen) << 32;
    int im = 0;
    int ib = w8;
    // ring slot k of a warp is filled by bulk copies issued by its lane 0
    // and completes on the slot's mbarrier
    const uint64_t pol = policy_evict_first();
    uint64_t* mybar = rbar + warp * SW;
    auto issue_next = [&](int slot) {
      while (im < nmine && ib >= nbH) { ++im; ib = w8; }
      if (im < nmine) {
        if (lane == 0) {
          const int64_t iu = my_unit(im);
          const int e = sel_e[iu / panels];
          unsigned char* dst = myring + slot * kSlotBytes;
          if (e >= 0 && e < E) {
            const size_t pb = (static_cast<size_t>(e) * panels + static_cast<size_t>(iu % panels)) * nbH + ib;
            const uint32_t tb = kWBytes, sb = kMat - kWBytes;
            // after the words: the block scales, or the sub-scale code words
            const void* gtail = kE16 ? static_cast<const void*>(P.gate_codes + pb * kE16Words * kPanel)
                                     : static_cast<const void*>(P.gate_scales + pb * kPanel);
            const void* utail = kE16 ? static_cast<const void*>(P.up_codes + pb * kE16Words * kPanel)
                                     : static_cast<const void*>(P.up_scales + pb * kPanel);
            mbar_arrive_expect_tx(mybar + slot, 2 * (tb + sb));
            bulk_g2s(dst, P.gate_trits + pb * kWords * kPanel, tb, mybar + slot, pol);
            bulk_g2s(dst + tb, gtail, sb, mybar + slot, pol);
            bulk_g2s(dst + kMat, P.up_trits + pb * kWords * kPanel, tb, mybar + slot, pol);
            bulk_g2s(dst + kMat + tb, utail, sb, mybar + slot, pol);
          } else {
            mbar_arrive(mybar + slot);
          }
        }
        ib += kNC;
      }
    };
#pragma unroll 1
    for (int k = 0; k < SW; ++k) issue_next(k);
    // then the down panels, which are needed only after the gate/up phase:
    // lane 0 of warp j issues slot j's
    if (has_panel && lane == 0 && warp < K) {
      const int j = warp;
      const size_t pb0 = (static_cast<size_t>(sel_e[j]) * (H / kPanel) + panelH) * nbF;
      unsigned char* dst = pref + j * pref_slot;
      const uint32_t tb = static_cast<uint32_t>(nbF) * kWBytes;
      const uint32_t sb = static_cast<uint32_t>(nbF) * (kMat - kWBytes);
      if constexpr (kE16) {
        // words, sub-scale codes, then the panel rows' fp16 anchors
        mbar_arrive_expect_tx(pbar, tb + sb + kPanel * 2);
        bulk_g2s(dst, P.down_trits + pb0 * kWords * kPanel, tb, pbar, policy_evict_first());
        bulk_g2s(dst + tb, P.down_codes + pb0 * kE16Words * kPanel, sb, pbar, policy_evict_first());
        bulk_g2s(dst + tb + sb, P.down_scales + static_cast<size_t>(sel_e[j]) * H + static_cast<size_t>(panelH) * kPanel,
                 kPanel * 2, pbar, policy_evict_first());
      } else {
        mbar_arrive_expect_tx(pbar, tb + sb);
        bulk_g2s(dst, P.down_trits + pb0 * kWords * kPanel, tb, pbar, policy_evict_first());
        bulk_g2s(dst + tb, P.down_scales + pb0 * kPanel, sb, pbar, policy_evict_first());
      }
    }
    if constexpr (kShared) {
      // this panel's rows of the shared expert's down projection, for phase C
      if (has_panel && tid == 0) {
        const int Fs = S1.S.ffn;
        bulk_prefetch_l2(S1.S.down_q + static_cast<size_t>(panelH) * kPanel * Fs, static_cast<uint32_t>(kPanel * Fs));
        bulk_prefetch_l2(S1.S.down_d + static_cast<size_t>(panelH) * kPanel * (Fs / kQBlock),
                         static_cast<uint32_t>(2 * Fs));
      }
    }
    int s = 0;
    for (int ui = 0; ui < nmine; ++ui) {
      const int64_t u = my_unit(ui);
      const int j = static_cast<int>(u / panels), p = static_cast<int>(u % panels);
      float part[2][1] = {{0.f}, {0.f}};
      // two-level scales: the rows' anchors / 16 (loaded now, used at the
      // unit's end) and one fp32 chain over the warp's blocks, as the grouped
      // E16 gate/up kernel keeps
      float a16[2] = {0.f, 0.f}, tot[2] = {0.f, 0.f};
      if constexpr (kE16) {
        const int e = sel_e[j];
        if (e >= 0 && e < E) {
          const size_t row = static_cast<size_t>(e) * F + static_cast<size_t>(p) * kPanel + lane;
          a16[0] = f16_bits_to_f32(P.gate_scales[row]) * 0.0625f;
          a16[1] = f16_bits_to_f32(P.up_scales[row]) * 0.0625f;
        }
      }
      for (int b = w8; b < nbH; b += kNC, ++s) {
        const int slot = s % SW;
        if (!mbar_wait_sleep(mybar + slot, static_cast<uint32_t>(s / SW) & 1u) && lane == 0) {
          record_status(P.status, MOE_ERR_TIMEOUT);
          *abort = 1;
        }
        if constexpr (kE16) {
          int isum[2][kSubPerBlock];
          block_isums_e16<2>(myring + slot * kSlotBytes, kMat, kWBytes, sq4 + b * (kBlock / 4), lane, isum);
#pragma unroll
          for (int sb = 0; sb < kSubPerBlock; ++sb) {
            const float dn = sxd[b * kSubPerBlock + sb];
#pragma unroll
            for (int m = 0; m < 2; ++m) tot[m] = __fmaf_rn(dn, static_cast<float>(isum[m][sb]), tot[m]);
          }
        } else if constexpr (kSign) {
          block_dot_sign<2>(myring + slot * kSlotBytes, kMat, kWBytes, sq4 + b * (kBlock / 4), sxd + b * kSubPerBlock,
                            sxas + b * kSubPerBlock, lane, part);
        } else {
          block_dot<2, 1, 1>(myring + slot * kSlotBytes, sq4 + b * (kBlock / 4), 0, sxd + b * kSubPerBlock,
                             sxas + b * kSubPerBlock, 0, lane, part);
        }
        __syncwarp();
        issue_next(slot);
      }
      if constexpr (kE16) {
#pragma unroll
        for (int m = 0; m < 2; ++m) part[m][0] = __fmaf_rn(a16[m], tot[m], 0.f);
      }
      // unit ui's epilogue runs on warp ui % kNC of the stream, which waits
      // for the stream's sums; the other warps leave theirs and go on with
      // the next unit (before they overwrite the sums, the previous unit's
      // epilogue warp has read them)
      const int ep = ui % kNC, ep_prev = (ui + kNC - 1) % kNC;
      if (ui > 0 && w8 != ep_prev) stream_bar_sync(bar_free);
      rb[(0 * kNC + w8) * 32 + lane] = part[0][0];
      rb[(1 * kNC + w8) * 32 + lane] = part[1][0];
      if (w8 != ep) {
        stream_bar_arrive(bar_done);
      } else {
        stream_bar_sync(bar_done);
        float g = 0.f, uu = 0.f;
        const int nw = nbH < kNC ? nbH : kNC;
        for (int v = 0; v < nw; ++v) {
          g = __fadd_rn(g, rb[(0 * kNC + v) * 32 + lane]);
          uu = __fadd_rn(uu, rb[(1 * kNC + v) * 32 + lane]);
        }
        if (ui + 1 < nmine) stream_bar_arrive(bar_free);
        const float a = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.f, expf(-g))), uu);
        const float amax = warp_max(fabsf(a));
        const float dd = __fdiv_rn(amax, 127.f);
        int q = 0;
        if (dd != 0.f) q = max(-127, min(127, __float2int_rn(__fdiv_rn(a, dd))));
        const int qs = __reduce_add_sync(0xffffffffu, q);
        // publish the unit: lane i < 8 the codes of rows 4i..4i+3, lane 8
        // the scale, lane 9 the code sum, each word tagged with the launch
        const uint32_t qb = static_cast<uint32_t>(q) & 0xffu;
        const uint32_t w4 = qb | (__shfl_down_sync(0xffffffffu, qb, 1) << 8) |
                            (__shfl_down_sync(0xffffffffu, qb, 2) << 16) |
                            (__shfl_down_sync(0xffffffffu, qb, 3) << 24);
        const uint32_t cw = __shfl_sync(0xffffffffu, w4, (4 * lane) & 31);
        const uint32_t payload = lane < kPanel / 4 ? cw
                                 : lane == kPanel / 4 ? __float_as_uint(dd) : static_cast<uint32_t>(qs);
        if (lane < kUnitWords)
          st_relaxed_u64(S1.units + (static_cast<size_t>(j) * panels + p) * kUnitWords + lane, tag64 | payload);
      }
    }
    if constexpr (kShared) {
      // the shared expert's units of this stream: warp w8 takes rows w8,
      // w8 + 8, ... of the 32-row block (one row per warp, as the shared
      // expert's own gate/up kernel), then warp 0 of the stream requantizes
      // the block and publishes it like a routed unit
      float* ssa = reinterpret_cast<float*>(smem + L.shr) + h * kQBlock;
      const int8_t* xq8 = reinterpret_cast<const int8_t*>(sq4);
      const int bar_sh = 1 + 2 * kS1Streams + h;
      for (int si = 0; si < nshared; ++si) {
        const int64_t su = my_unit(nmine + si) - U;
        for (int r = w8; r < kQBlock; r += kNC) {
          const int64_t f = su * kQBlock + r;
          float g, u;
          q8_row_dot2(S1.S.gate_q + f * H, S1.S.gate_d + f * (H / kQBlock), S1.S.up_q + f * H,
                      S1.S.up_d + f * (H / kQBlock), H, xq8, sxd, lane, g, u);
          if (lane == 0) ssa[r] = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.f, expf(-g))), u);
        }
        stream_bar_sync(bar_sh);
        if (w8 == 0) {
          const float a = ssa[lane];
          const float amax = warp_max(fabsf(a));
          const float dd = __fdiv_rn(amax, 127.f);
          int q = 0;
          if (dd != 0.f) q = max(-127, min(127, __float2int_rn(__fdiv_rn(a, dd))));
          const int qs = __reduce_add_sync(0xffffffffu, q);
          const uint32_t qb = static_cast<uint32_t>(q) & 0xffu;
          const uint32_t w4 = qb | (__shfl_down_sync(0xffffffffu, qb, 1) << 8) |
                              (__shfl_down_sync(0xffffffffu, qb, 2) << 16) |
                              (__shfl_down_sync(0xffffffffu, qb, 3) << 24);
          const uint32_t cw = __shfl_sync(0xffffffffu, w4, (4 * lane) & 31);
          const uint32_t payload = lane < kPanel / 4 ? cw
                                   : lane == kPanel / 4 ? __float_as_uint(dd) : static_cast<uint32_t>(qs);
          if (lane < kUnitWords) st_relaxed_u64(S1.sunits + su * kUnitWords + lane, tag64 | payload);
        }
        stream_bar_sync(bar_sh);
      }
    }
    // every copy issued was consumed above: none is in flight here
    __syncthreads();
  }

  // ---------------- phase C: this CTA's panel of hidden, all slots
  if (has_panel) {
    // the prefetch must land before this CTA reads it or exits
    bool ok = mbar_wait_sleep(pbar, 0);
    if (!ok) record_status(P.status, MOE_ERR_TIMEOUT);
    // the items (slot j, block b of ffn): each polls the tagged words of its
    // 8 units, multiplies them with the prefetched down weights and leaves
    // its inner sums and weight scales in shared memory; one warp per slot
    // then applies the scales and warp 0 combines the slots, in the order of
    // the grouped down kernel.  With at most two items per warp they go to
    // the warps in slot order (item i to warp i % kS1Warps: the units of the
    // lower slots are published first, so every warp starts at once);
    // otherwise warp w takes slot w % kNC, the first (w < kNC) or second half
    // of its blocks, so that the warps of the early slots finish early.
    const int panels = F / kPanel;
    int* aq4 = reinterpret_cast<int*>(smem + L.act);                       // [K][F/4]
    float* ad = reinterpret_cast<float*>(aq4 + K * (F / 4));                 // [K][F/32]
    int* aas = reinterpret_cast<int*>(ad + K * (F / kQBlock));              // [K][F/32]
    float* sinner = reinterpret_cast<float*>(smem + L.inner);               // [K][nbF][32]
    float* sscale = sinner + K * nbF * kPanel;                              // [K][nbF][32]
    if constexpr (kSlotOrder) {
      const uint32_t tag = *sgen;
      const unsigned char* wbase = pref;
      constexpr int kItemWords = (kBlock / kPanel) * kUnitWords;  // the 8 units of one block of ffn
      constexpr int kPerI = (kItemWords + 31) / 32;
      uint32_t need = 0;
#pragma unroll
      for (int i = 0; i < kPerI; ++i)
        if (lane + 32 * i < kItemWords) need |= 1u << i;
      auto item_src = [&](int it) {
        const int j = it / nbF, b = it % nbF;
        return S1.units + (static_cast<size_t>(j) * panels + b * (kBlock / kPanel)) * kUnitWords;
      };
      const int nitems = warp < K * nbF ? (K * nbF - 1 - warp) / kS1Warps + 1 : 0;
      auto item_at = [&](int q) { return warp + q * kS1Warps; };
      // the loads of a warp's next item are in flight while it computes the
      // current one
      unsigned long long vn[kPerI];
      if (nitems > 0) {
        const unsigned long long* src = item_src(item_at(0));
#pragma unroll
        for (int i = 0; i < kPerI; ++i)
          if (need & (1u << i)) vn[i] = ld_relaxed_u64(src + lane + 32 * i);
      }
      for (int q = 0; ok && q < nitems; ++q) {
        if (*abort) break;
        const int it = item_at(q);
        const int j = it / nbF, b = it % nbF;
        const unsigned long long* src = item_src(it);
        unsigned long long v[kPerI];
        uint32_t ready = 0;
#pragma unroll
        for (int i = 0; i < kPerI; ++i) {
          v[i] = vn[i];
          if ((need & (1u << i)) && static_cast<uint32_t>(v[i] >> 32) == tag) ready |= 1u << i;
        }
        if (q + 1 < nitems) {
          const unsigned long long* nsrc = item_src(item_at(q + 1));
#pragma unroll
          for (int i = 0; i < kPerI; ++i)
            if (need & (1u << i)) vn[i] = ld_relaxed_u64(nsrc + lane + 32 * i);
        }
        for (uint32_t polls = 0; ready != need; ++polls) {
          if (polls > kSpinLimit) break;
#pragma unroll
          for (int i = 0; i < kPerI; ++i)
            if ((need & ~ready) & (1u << i)) v[i] = ld_relaxed_u64(src + lane + 32 * i);
#pragma unroll
          for (int i = 0; i < kPerI; ++i)
            if (((need & ~ready) & (1u << i)) && static_cast<uint32_t>(v[i] >> 32) == tag) ready |= 1u << i;
        }
        if (!__all_sync(0xffffffffu, ready == need)) {
          if (lane == 0) {
            record_status(P.status, MOE_ERR_TIMEOUT);
            *abort = 1;
          }
          break;
        }
#pragma unroll
        for (int i = 0; i < kPerI; ++i) {
          const int w = lane + 32 * i;
          if (w < kItemWords) {
            const int pl = b * (kBlock / kPanel) + w / kUnitWords, k = w % kUnitWords;
            const uint32_t x32 = static_cast<uint32_t>(v[i]);
            if (k < kPanel / 4) aq4[j * (F / 4) + pl * (kPanel / 4) + k] = static_cast<int>(x32);
            else if (k == kPanel / 4) ad[j * (F / kQBlock) + pl] = __uint_as_float(x32);
            else aas[j * (F / kQBlock) + pl] = static_cast<int>(x32);
          }
        }
        __syncwarp();
        const unsigned char* wj = wbase + j * pref_slot;
        // block b's words, then (after every block's words) its scales or
        // sub-scale code words
        const int tail_off = nbF * kWBytes + b * (kMat - kWBytes) - b * kWBytes;
        if constexpr (kE16) {
          // the block's 8 integer sums; warp j chains them with the scales
          int isum[1][kSubPerBlock];
          block_isums_e16<1>(wj + static_cast<size_t>(b) * kWBytes, kMat, tail_off,
                             aq4 + j * (F / 4) + b * (kBlock / 4), lane, isum);
          int* sacc = reinterpret_cast<int*>(sinner);  // [K][nbF][8][32]
#pragma unroll
          for (int sb = 0; sb < kSubPerBlock; ++sb) sacc[((j * nbF + b) * kSubPerBlock + sb) * kPanel + lane] = isum[0][sb];
        } else {
          float inner[1][1];
          float sc[1];
          if constexpr (kSign)
            block_dot_sign<1, true>(wj + static_cast<size_t>(b) * kWBytes, kMat, tail_off,
                                    aq4 + j * (F / 4) + b * (kBlock / 4), ad + j * (F / kQBlock) + b * kSubPerBlock,
                                    aas + j * (F / kQBlock) + b * kSubPerBlock, lane, inner, sc);
          else
            block_dot<1, 1, 1, true>(wj + static_cast<size_t>(b) * kWBytes, aq4 + j * (F / 4) + b * (kBlock / 4), 0,
                                     ad + j * (F / kQBlock) + b * kSubPerBlock,
                                     aas + j * (F / kQBlock) + b * kSubPerBlock, 0, lane, inner, tail_off, sc);
          sinner[(j * nbF + b) * kPanel + lane] = inner[0][0];
          sscale[(j * nbF + b) * kPanel + lane] = sc[0];
        }
      }
    } else {
      const int j = warp % kNC, half = warp / kNC;
      const int nb0 = (nbF + 1) / 2;
      const int bb = half ? nb0 : 0, be = half ? nbF : nb0;
      if (j < K && ok && bb < be) {
        // the tagged words of panels [8*bb, 8*be) of slot j, all loads of a
        // round in flight at once
        constexpr int kPerC = (kS1MaxF / kBlock + 1) / 2 * (kBlock / kPanel) * kUnitWords / 32;
        const int nw = (be - bb) * (kBlock / kPanel) * kUnitWords;
        const unsigned long long* src =
            S1.units + (static_cast<size_t>(j) * panels + bb * (kBlock / kPanel)) * kUnitWords;
        const uint32_t tag = *sgen;
        unsigned long long v[kPerC];
        uint32_t ready = 0, need = 0;
#pragma unroll
        for (int i = 0; i < kPerC; ++i)
          if (lane + 32 * i < nw) need |= 1u << i;
        for (uint32_t polls = 0; ready != need; ++polls) {
          if (polls > kSpinLimit) break;
#pragma unroll
          for (int i = 0; i < kPerC; ++i)
            if ((need & ~ready) & (1u << i)) v[i] = ld_relaxed_u64(src + lane + 32 * i);
#pragma unroll
          for (int i = 0; i < kPerC; ++i)
            if (((need & ~ready) & (1u << i)) && static_cast<uint32_t>(v[i] >> 32) == tag) ready |= 1u << i;
        }
        if (!__all_sync(0xffffffffu, ready == need)) {
          if (lane == 0) {
            record_status(P.status, MOE_ERR_TIMEOUT);
            *abort = 1;
          }
        } else {
#pragma unroll
          for (int i = 0; i < kPerC; ++i) {
            const int w = lane + 32 * i;
            if (w < nw) {
              const int pl = bb * (kBlock / kPanel) + w / kUnitWords, k = w % kUnitWords;
              const uint32_t x32 = static_cast<uint32_t>(v[i]);
              if (k < kPanel / 4) aq4[j * (F / 4) + pl * (kPanel / 4) + k] = static_cast<int>(x32);
              else if (k == kPanel / 4) ad[j * (F / kQBlock) + pl] = __uint_as_float(x32);
              else aas[j * (F / kQBlock) + pl] = static_cast<int>(x32);
            }
          }
          __syncwarp();
          const unsigned char* wj = pref + j * pref_slot;
          for (int b = bb; b < be; ++b) {
            // block b's words, then (after every block's words) its scales
            const int scale_off = nbF * kWBytes + b * kPanel * 2 - b * kWBytes;
            float inner[1][1];
            float sc[1];
            if constexpr (kSign)
              block_dot_sign<1, true>(wj + static_cast<size_t>(b) * kWBytes, kMat, scale_off,
                                      aq4 + j * (F / 4) + b * (kBlock / 4), ad + j * (F / kQBlock) + b * kSubPerBlock,
                                      aas + j * (F / kQBlock) + b * kSubPerBlock, lane, inner, sc);
            else
              block_dot<1, 1, 1, true>(wj + static_cast<size_t>(b) * kWBytes, aq4 + j * (F / 4) + b * (kBlock / 4), 0,
                                       ad + j * (F / kQBlock) + b * kSubPerBlock,
                                       aas + j * (F / kQBlock) + b * kSubPerBlock, 0, lane, inner, scale_off, sc);
            sinner[(j * nbF + b) * kPanel + lane] = inner[0][0];
            sscale[(j * nbF + b) * kPanel + lane] = sc[0];
          }
        }
      }
    }
    float* ssv = reinterpret_cast<float*>(smem + L.shr) + kS1Streams * kQBlock;  // [32] shared down rows
    if constexpr (kShared) {
      // the panel's 32 rows of the shared expert's down projection on warps
      // kNC.. (four rows each), lane j taking the shared ffn's 32-blocks j,
      // j + 32, ... as the shared expert's own down kernel does.  Block j's
      // codes and scale are the tagged words of shared unit j; one warp polls
      // them (a warp per CTA, not eight: the units are few lines of L2 that
      // every CTA reads) into the ring area past the inner sums.  Warps kNC..
      // start as soon as their down items are done (in slot order they hold
      // fewer), before the CTA-wide barrier.
      if (ok && warp >= kNC) {
        const int Fs = S1.S.ffn, nbs = Fs / kQBlock;
        int* saq = reinterpret_cast<int*>(smem + L.inner + static_cast<size_t>(s1_item_words(kFmt)) * K * nbF * kPanel * 4);  // [nbs][8]
        float* sad = reinterpret_cast<float*>(saq + kMaxSharedUnits * (kPanel / 4));                      // [nbs]
        if (warp == kNC && !*abort) {
          const uint32_t tag = *sgen;
          for (int j0 = 0; j0 < nbs; j0 += 32) {
            const int jb = j0 + lane;
            const uint32_t need = jb < nbs ? (1u << (kPanel / 4 + 1)) - 1u : 0u;  // 8 code words and the scale
            const unsigned long long* src = S1.sunits + static_cast<size_t>(jb) * kUnitWords;
            unsigned long long wv[kPanel / 4 + 1];
            uint32_t ready = 0;
            for (uint32_t polls = 0;; ++polls) {
#pragma unroll
              for (int i = 0; i <= kPanel / 4; ++i)
                if ((need & ~ready) & (1u << i)) wv[i] = ld_relaxed_u64(src + i);
#pragma unroll
              for (int i = 0; i <= kPanel / 4; ++i)
                if (((need & ~ready) & (1u << i)) && static_cast<uint32_t>(wv[i] >> 32) == tag) ready |= 1u << i;
              if (__all_sync(0xffffffffu, ready == need) || polls > kSpinLimit) break;
            }
            if (!__all_sync(0xffffffffu, ready == need)) {
              if (lane == 0) {
                record_status(P.status, MOE_ERR_TIMEOUT);
                *abort = 1;
              }
              break;
            }
            if (jb < nbs) {
#pragma unroll
              for (int i = 0; i < kPanel / 4; ++i) saq[jb * (kPanel / 4) + i] = static_cast<int>(wv[i]);
              sad[jb] = __uint_as_float(static_cast<uint32_t>(wv[kPanel / 4]));
            }
          }
        }
        stream_bar_sync(1 + 3 * kS1Streams);  // warps kNC.. (the shared codes are in place)
        if (!*abort) {
          constexpr int kRows = kPanel / (kS1Warps - kNC);
          float acc[kRows];
#pragma unroll
          for (int i = 0; i < kRows; ++i) acc[i] = 0.f;
          for (int jb = lane; jb < nbs; jb += 32) {
            const int4 a0 = reinterpret_cast<const int4*>(saq + jb * (kPanel / 4))[0];
            const int4 a1 = reinterpret_cast<const int4*>(saq + jb * (kPanel / 4))[1];
            const float ad = sad[jb];
#pragma unroll
            for (int i = 0; i < kRows; ++i) {
              const size_t hrow = static_cast<size_t>(panelH) * kPanel + (warp - kNC) + (kS1Warps - kNC) * i;
              const int4* wq = reinterpret_cast<const int4*>(S1.S.down_q + hrow * Fs + static_cast<size_t>(jb) * kQBlock);
              const int4 w0 = wq[0], w1 = wq[1];
              int sd = __dp4a(w0.x, a0.x, 0);
              sd = __dp4a(w0.y, a0.y, sd);
              sd = __dp4a(w0.z, a0.z, sd);
              sd = __dp4a(w0.w, a0.w, sd);
              sd = __dp4a(w1.x, a1.x, sd);
              sd = __dp4a(w1.y, a1.y, sd);
              sd = __dp4a(w1.z, a1.z, sd);
              sd = __dp4a(w1.w, a1.w, sd);
              const float sc = __fmul_rn(f16_bits_to_f32(S1.S.down_d[hrow * nbs + jb]), ad);
              acc[i] = __fmaf_rn(sc, static_cast<float>(sd), acc[i]);
            }
          }
#pragma unroll
          for (int i = 0; i < kRows; ++i) {
            float v = acc[i];
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, m));
            if (lane == 0) ssv[(warp - kNC) + (kS1Warps - kNC) * i] = v;
          }
        }
      }
    }
    __syncthreads();
    // warp j applies slot j's block scales in order, then warp 0 combines
    // the slots in order (the summation order of the grouped down kernel)
    float* spart = reinterpret_cast<float*>(smem + L.red);  // [K][32]; the gate/up sums are done with it
    if (!*abort && ok && warp < K) {
      float part = 0.f;
      if constexpr (kE16) {
        // one fp32 chain over every sub-block of the row, then the row's
        // anchor / 16 (the grouped E16 down kernel's order)
        const int* sacc = reinterpret_cast<const int*>(sinner);
        float tot = 0.f;
        for (int b = 0; b < nbF; ++b)
#pragma unroll
          for (int sb = 0; sb < kSubPerBlock; ++sb)
            tot = __fmaf_rn(ad[warp * (F / kQBlock) + b * kSubPerBlock + sb],
                            static_cast<float>(sacc[((warp * nbF + b) * kSubPerBlock + sb) * kPanel + lane]), tot);
        const uint16_t* anc = reinterpret_cast<const uint16_t*>(pref + warp * pref_slot + static_cast<size_t>(nbF) * kMat);
        part = __fmaf_rn(f16_bits_to_f32(anc[lane]) * 0.0625f, tot, 0.f);
      } else {
        for (int b = 0; b < nbF; ++b)
          part = __fmaf_rn(sscale[(warp * nbF + b) * kPanel + lane], sinner[(warp * nbF + b) * kPanel + lane], part);
      }
      spart[warp * kPanel + lane] = part;
    }
    __syncthreads();
    if (!*abort && ok && warp == 0) {
      float y = 0.f;
      for (int jj = 0; jj < K; ++jj) y = __fmaf_rn(sel_w[jj], spart[jj * kPanel + lane], y);
      if constexpr (kShared) y = __fadd_rn(y, ssv[lane]);  // after the routed combine, as the shared kernel adds it
      P.y[panelH * kPanel + lane] = y;
    }
  }
}

bool step1_supported(const DecodeParams& P, int n_sm, size_t* smem) {
  if (P.ntok != 1 || P.hidden > kS1MaxH || P.ffn > kS1MaxF || P.top_k > kS1MaxK) return false;
  if (P.hidden / kPanel > n_sm) return false;
  if (P.n_experts > 2 * n_sm) return false;  // at most two router rows per CTA
  if (P.n_experts > kS1MaxE) return false;
  if (P.format != MOE_FORMAT_TERNARY && P.format != MOE_FORMAT_SIGN && P.format != MOE_FORMAT_E16) return false;
  const Step1Layout L = step1_layout(P.hidden, P.ffn, P.n_experts, P.top_k, P.format);
  *smem = L.total;
  return L.total <= static_cast<size_t>(kMaxDynSmem);
}

int launch_step1(const Decode2Params& D, unsigned long long* ticket, unsigned long long* units,
                 cudaStream_t stream, const SharedParams* shared, unsigned long long* sunits) {
  static std::atomic<bool> done[64];  // the attribute call is idempotent
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !done[dev].load(std::memory_order_relaxed)) {
    constexpr int T = MOE_FORMAT_TERNARY, Sg = MOE_FORMAT_SIGN, E6 = MOE_FORMAT_E16;
    const void* ks[] = {reinterpret_cast<const void*>(&k_step1<T, false, false>),
                        reinterpret_cast<const void*>(&k_step1<Sg, false, false>),
                        reinterpret_cast<const void*>(&k_step1<T, true, false>),
                        reinterpret_cast<const void*>(&k_step1<Sg, true, false>),
                        reinterpret_cast<const void*>(&k_step1<E6, true, false>),
                        reinterpret_cast<const void*>(&k_step1<T, false, true>),
                        reinterpret_cast<const void*>(&k_step1<Sg, false, true>),
                        reinterpret_cast<const void*>(&k_step1<T, true, true>),
                        reinterpret_cast<const void*>(&k_step1<Sg, true, true>),
                        reinterpret_cast<const void*>(&k_step1<E6, true, true>)};
    for (const void* k : ks) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
    done[dev].store(true, std::memory_order_relaxed);
  }
  size_t smem = 0;
  if (!step1_supported(D.P, D.n_sm, &smem)) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "step1: unsupported shape");
  if (shared && (shared->hidden != D.P.hidden || shared->ffn <= 0 || shared->ffn % kQBlock ||
                 shared->ffn / kQBlock > kMaxSharedUnits || !sunits))
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "step1: unsupported shared expert");
  Step1Params S{D, ticket, reinterpret_cast<unsigned long long*>(D.logits), units, SharedParams{}, sunits};
  if (shared) S.S = *shared;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(D.n_sm);
  cfg.blockDim = dim3(kS1Warps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  // cooperative (every CTA resident), and a programmatic dependent launch so
  // that consecutive steps overlap (phase A of one step with the tail of the
  // previous); without the latter where the runtime refuses the combination
  static std::atomic<int> pdl_ok[64];  // 0 unknown, 1 yes, -1 no (any thread may settle it)
  const int di = dev >= 0 && dev < 64 ? dev : 0;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_ok[di] >= 0 ? 2 : 1;
  // two-level scales always take the down items in slot order (their
  // per-block results are integer sums that one warp per slot chains)
  const int fmt = D.P.format;
  const bool slot_order = fmt == MOE_FORMAT_E16 || D.P.top_k * (D.P.ffn / kBlock) <= 2 * kS1Warps;
  constexpr int T = MOE_FORMAT_TERNARY, Sg = MOE_FORMAT_SIGN, E6 = MOE_FORMAT_E16;
  void (*kern)(Step1Params) = nullptr;
  if (fmt == E6) kern = shared ? k_step1<E6, true, true> : k_step1<E6, true, false>;
  else if (fmt == Sg)
    kern = shared ? (slot_order ? k_step1<Sg, true, true> : k_step1<Sg, false, true>)
                  : (slot_order ? k_step1<Sg, true, false> : k_step1<Sg, false, false>);
  else
    kern = shared ? (slot_order ? k_step1<T, true, true> : k_step1<T, false, true>)
                  : (slot_order ? k_step1<T, true, false> : k_step1<T, false, false>);
  cudaError_t err = cudaLaunchKernelEx(&cfg, kern, S);
  if (err != cudaSuccess && cfg.numAttrs == 2 && pdl_ok[di] == 0) {
    cudaGetLastError();
    pdl_ok[di] = -1;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, kern, S);
  } else if (err == cudaSuccess && cfg.numAttrs == 2) {
    pdl_ok[di] = 1;
  }
  if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "step1: %s", cudaGetErrorString(err));
  note_launch(MOE_K_STEP1, stream);
  return check_launch("step1");
}

}  // namespace bitmoe
