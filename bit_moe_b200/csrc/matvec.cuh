// matvec.cuh -- shared device code of the persistent decode kernels: work
// groups, cp.async item copies, and the in-register base-3 decode with dp4a
// accumulation of one 256-weight block of a 32-row panel (sm_100a).
#pragma once

#include "common.cuh"
#include "decode2.cuh"
#include "ptx.cuh"

namespace bitmoe {

constexpr int kNC = kConsumerWarps;

template <int NTMAX>
constexpr int ring_depth() { return NTMAX == 1 ? 3 : 3; }

// Ring slot of one item: NM matrix blocks of a 32-row panel, then (without
// staged activations) the activation block of each of the item's pairs.
template <int NM, int NTMAX, bool kStaged>
struct Slot {
  static constexpr int act = NM * kMatBytes;                     // codes [NTMAX][256]
  static constexpr int act_d = NM * kMatBytes + NTMAX * kBlock;  // scales [NTMAX][8]
  static constexpr int bytes = kStaged ? NM * kMatBytes : NM * kMatBytes + NTMAX * kActBytes;
};

// Group g of the mat-vec work: the (token, slot) pairs routed to one expert.
struct Group {
  int expert;  // -1: out-of-range id
  int count;
  int start;   // grouped mode: first entry of the pair list
};

__device__ __forceinline__ Group get_group(const DecodeParams& P, int g) {
  Group G;
  if (P.direct) {
    const int e = P.idx[g];
    G.expert = (e >= 0 && e < P.n_experts) ? e : -1;
    G.count = 1;
    G.start = g;
  } else {
    const Item it = P.items[g];
    G.expert = it.expert;
    G.count = it.count;
    G.start = it.start;
  }
  return G;
}

__device__ __forceinline__ int group_pair(const DecodeParams& P, const Group& G, int n) {
  return P.direct ? G.start + n : P.pairs[G.start + n];
}

__device__ __forceinline__ int n_groups(const DecodeParams& P) {
  return P.direct ? P.ntok * P.top_k : *P.n_items;
}

// Balanced contiguous range [lo, hi) of n units for CTA c of C.
__device__ __forceinline__ void cta_range(int64_t n, int c, int C, int64_t& lo, int64_t& hi) {
  lo = n * c / C;
  hi = n * (c + 1) / C;
}

// ---- asynchronous copies: 16 bytes per lane, completion per commit group
__device__ __forceinline__ void cp16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global.L2::128B [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Copy n16 16-byte chunks from src to dst, spread over the 32 lanes.
__device__ __forceinline__ void warp_copy(unsigned char* dst, const void* src, int n16, int lane) {
  const unsigned char* s = static_cast<const unsigned char*>(src);
  for (int c = lane; c < n16; c += 32) cp16(dst + c * 16, s + c * 16);
}

// The activation rows of a group's pairs: token rows of x^ (gate/up) or pair
// rows of a^ (down).
template <int NTMAX>
struct ActSrc {
  const int8_t* codes[NTMAX];
  const float* scales[NTMAX];
};

template <int NM, int NTMAX>
__device__ __forceinline__ void act_sources(const DecodeParams& P, const Group& G, ActSrc<NTMAX>& A) {
  const bool gu = (NM == 2);
  const int k = gu ? P.hidden : P.ffn;
#pragma unroll
  for (int n = 0; n < NTMAX; ++n) {
    A.codes[n] = nullptr;
    A.scales[n] = nullptr;
    if (n < G.count) {
      const int pair = group_pair(P, G, n);
      const int row = gu ? pair / P.top_k : pair;
      A.codes[n] = (gu ? P.xq : P.aq) + static_cast<size_t>(row) * k;
      A.scales[n] = (gu ? P.xd : P.ad) + static_cast<size_t>(row) * (k / kQBlock);
    }
  }
}

// Issue the copies of one item (block b of panel p of group G) into dst.
template <int NM, int NTMAX, bool kStaged>
__device__ __forceinline__ void issue_item(unsigned char* dst, const DecodeParams& P, const Group& G,
                                           const ActSrc<NTMAX>& A, int p, int b, int lane) {
  using S = Slot<NM, NTMAX, kStaged>;
  const bool gu = (NM == 2);
  const int nb = (gu ? P.hidden : P.ffn) / kBlock;
  const int panels = (gu ? P.ffn : P.hidden) / kPanel;
  if (G.expert >= 0) {
    const size_t pb = (static_cast<size_t>(G.expert) * panels + p) * nb + b;
    const uint32_t* tr[2] = {gu ? P.gate_trits : P.down_trits, P.up_trits};
    const uint16_t* sc[2] = {gu ? P.gate_scales : P.down_scales, P.up_scales};
#pragma unroll
    for (int m = 0; m < NM; ++m) {
      warp_copy(dst + m * kMatBytes, tr[m] + pb * kBlockWords * kPanel, kBlockWords * kPanel * 4 / 16, lane);
      warp_copy(dst + m * kMatBytes + kBlockWords * kPanel * 4, sc[m] + pb * kPanel, kPanel * 2 / 16, lane);
    }
  }
  if constexpr (!kStaged) {
#pragma unroll
    for (int n = 0; n < NTMAX; ++n) {
      if (n < G.count) {
        warp_copy(dst + S::act + n * kBlock, A.codes[n] + b * kBlock, kBlock / 16, lane);
        warp_copy(dst + S::act_d + n * kSubPerBlock * 4, A.scales[n] + b * kSubPerBlock,
                  kSubPerBlock * 4 / 16, lane);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Decode of one block: NM matrices (words and scales at wsrc) against NT
// activation vectors (codes q4[n*qs + g], scales ds[n*dsn + s], block sums
// as[n*dsn + s], or computed here from the codes when as is null).
// part[m][n] += s_w[m] * sum_s d[n][s] * isum[m][n][s]; with kInner, part
// receives the block's inner sum sum_s d[n][s] * isum[m][n][s] itself and
// sc_out[m] the weight scale s_w[m], so that a caller can apply the scales of
// blocks computed by different warps in the same order.
// ---------------------------------------------------------------------------
template <int NM, int NT, int NTMAX, bool kInner = false>
__device__ __forceinline__ void block_dot(const unsigned char* __restrict__ wsrc, const int* __restrict__ q4,
                                          int qs, const float* __restrict__ ds, const int* __restrict__ as,
                                          int dsn, int lane, float (&part)[NM][NTMAX],
                                          int scale_off = kBlockWords * kPanel * 4, float* sc_out = nullptr) {
  int s2[NT];
  if (as == nullptr) {
    // sums of the codes per 32-block: lane l adds words 2l, 2l+1 (sub-block
    // l/4), then the four lanes of a sub-block are summed
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int2 v = reinterpret_cast<const int2*>(q4 + n * qs)[lane];
      int sum = __dp4a(v.x, 0x01010101, 0);
      sum = __dp4a(v.y, 0x01010101, sum);
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      s2[n] = sum;
    }
  }
  uint32_t w[NM][kBlockWords];
  float sc[NM];
#pragma unroll
  for (int m = 0; m < NM; ++m) {
    const uint32_t* tw = reinterpret_cast<const uint32_t*>(wsrc + m * kMatBytes);
#pragma unroll
    for (int j = 0; j < kBlockWords; ++j) w[m][j] = tw[j * kPanel + lane];
    sc[m] = f16_bits_to_f32(reinterpret_cast<const uint16_t*>(wsrc + m * kMatBytes + scale_off)[lane]);
  }
  int acc[NM][NT];
  float inner[NM][NT];
#pragma unroll
  for (int m = 0; m < NM; ++m)
#pragma unroll
    for (int n = 0; n < NT; ++n) { acc[m][n] = 0; inner[m][n] = 0.f; }
#pragma unroll
  for (int j = 0; j < kBlockWords; ++j) {
    uint32_t lo[NM], hi[NM], hp[NM];
#pragma unroll
    for (int m = 0; m < NM; ++m) {
      lo[m] = w[m][j] & 0x00FF00FFu;
      hi[m] = __byte_perm(w[m][j], 0u, 0x4341);  // bytes 1, 3 into 16-bit lanes
      hp[m] = 0u;
    }
#pragma unroll
    for (int i = 0; i < 5; ++i) {
      if (j == kBlockWords - 1 && i == 4) break;  // pad digit of the last word
      const int g = 5 * j + i;
      int a[NT];
#pragma unroll
      for (int n = 0; n < NT; ++n) a[n] = q4[n * qs + g];
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        lo[m] *= 3u;
        hi[m] *= 3u;
        const uint32_t hn = __byte_perm(lo[m], hi[m], 0x7351);
        const int t = static_cast<int>(hn - 3u * hp[m]);
        hp[m] = hn;
#pragma unroll
        for (int n = 0; n < NT; ++n) acc[m][n] = __dp4a(t, a[n], acc[m][n]);
      }
      if ((g & 7) == 7) {
        const int s = g >> 3;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const int an = as ? as[n * dsn + s] : __shfl_sync(0xffffffffu, s2[n], 4 * s);
          const float dn = ds[n * dsn + s];
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            inner[m][n] = __fmaf_rn(dn, static_cast<float>(acc[m][n] - an), inner[m][n]);
            acc[m][n] = 0;
          }
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < NM; ++m) {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      if constexpr (kInner) part[m][n] = inner[m][n];
      else part[m][n] = __fmaf_rn(sc[m], inner[m][n], part[m][n]);
    }
    if constexpr (kInner) sc_out[m] = sc[m];
  }
}

// Two-level scales (E16) of one block for one vector: NM matrices' base-3
// words at wsrc + m * mat_stride and their 4-bit sub-scale code words
// (kE16Words per row) code_off bytes after each matrix's words.  accw[m][s]
// receives, per 32-weight sub-block s, the exact integer sum over its two
// 16-weight halves h of (c_h + 1) * (sum(t * a) - sum(a)) -- the integer the
// grouped E16 kernels multiply by the activation scale of sub-block s; the
// caller chains those products in the kernels' order.
template <int NM>
__device__ __forceinline__ void block_isums_e16(const unsigned char* __restrict__ wsrc, int mat_stride,
                                                int code_off, const int* __restrict__ q4, int lane,
                                                int (&accw_out)[NM][kSubPerBlock]) {
  uint32_t w[NM][kBlockWords];
  uint32_t cw[NM][kE16Words];
#pragma unroll
  for (int m = 0; m < NM; ++m) {
    const uint32_t* tw = reinterpret_cast<const uint32_t*>(wsrc + m * mat_stride);
    const uint32_t* tc = reinterpret_cast<const uint32_t*>(wsrc + m * mat_stride + code_off);
#pragma unroll
    for (int j = 0; j < kBlockWords; ++j) w[m][j] = tw[j * kPanel + lane];
#pragma unroll
    for (int u = 0; u < kE16Words; ++u) cw[m][u] = tc[u * kPanel + lane];
  }
  int acc[NM], accw[NM];
  int as16 = 0;
#pragma unroll
  for (int m = 0; m < NM; ++m) { acc[m] = 0; accw[m] = 0; }
#pragma unroll
  for (int j = 0; j < kBlockWords; ++j) {
    uint32_t lo[NM], hi[NM], hp[NM];
#pragma unroll
    for (int m = 0; m < NM; ++m) {
      lo[m] = w[m][j] & 0x00FF00FFu;
      hi[m] = __byte_perm(w[m][j], 0u, 0x4341);  // bytes 1, 3 into 16-bit lanes
      hp[m] = 0u;
    }
#pragma unroll
    for (int i = 0; i < 5; ++i) {
      if (j == kBlockWords - 1 && i == 4) break;  // pad digit of the last word
      const int g = 5 * j + i;                    // group of 4 weights, 0..63
      const int a = q4[g];
      as16 = __dp4a(a, 0x01010101, as16);
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        lo[m] *= 3u;
        hi[m] *= 3u;
        const uint32_t hn = __byte_perm(lo[m], hi[m], 0x7351);
        const int t = static_cast<int>(hn - 3u * hp[m]);
        hp[m] = hn;
        acc[m] = __dp4a(t, a, acc[m]);
      }
      if ((g & 3) == 3) {  // a 16-weight half is complete
        const int h = g >> 2;
#pragma unroll
        for (int m = 0; m < NM; ++m) {
          const int cm = static_cast<int>((cw[m][h >> 3] >> (4 * (h & 7))) & 15u) + 1;
          accw[m] += cm * (acc[m] - as16);
          acc[m] = 0;
        }
        as16 = 0;
      }
      if ((g & 7) == 7) {  // a 32-weight sub-block is complete
#pragma unroll
        for (int m = 0; m < NM; ++m) {
          accw_out[m][g >> 3] = accw[m];
          accw[m] = 0;
        }
      }
    }
  }
}

// The same for one vector over 1-bit sign codes (kSignWords words per
// block, word j = activation block j, weight 32j + 4i + l in bit 8l + i):
// per sub-block the exact sum(q * a) = 2 * sum(t * a) - sum(a), scaled and
// accumulated in the order of the grouped sign-code kernels.  Matrix m's
// words are at wsrc + m * mat_stride, its fp16 scales scale_off bytes further.
template <int NM, bool kInner = false>
__device__ __forceinline__ void block_dot_sign(const unsigned char* __restrict__ wsrc, int mat_stride, int scale_off,
                                               const int* __restrict__ q4, const float* __restrict__ ds,
                                               const int* __restrict__ as, int lane, float (&part)[NM][1],
                                               float* sc_out = nullptr) {
  uint32_t w[NM][kSignWords];
  float sc[NM];
#pragma unroll
  for (int m = 0; m < NM; ++m) {
    const uint32_t* tw = reinterpret_cast<const uint32_t*>(wsrc + m * mat_stride);
#pragma unroll
    for (int j = 0; j < kSignWords; ++j) w[m][j] = tw[j * kPanel + lane];
    sc[m] = f16_bits_to_f32(reinterpret_cast<const uint16_t*>(wsrc + m * mat_stride + scale_off)[lane]);
  }
  float inner[NM];
#pragma unroll
  for (int m = 0; m < NM; ++m) inner[m] = 0.f;
#pragma unroll
  for (int j = 0; j < kSignWords; ++j) {
    int acc[NM];
#pragma unroll
    for (int m = 0; m < NM; ++m) acc[m] = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int a = q4[8 * j + i];
#pragma unroll
      for (int m = 0; m < NM; ++m) acc[m] = __dp4a(static_cast<int>((w[m][j] >> i) & 0x01010101u), a, acc[m]);
    }
    const int an = as[j];
    const float dn = ds[j];
#pragma unroll
    for (int m = 0; m < NM; ++m) inner[m] = __fmaf_rn(dn, static_cast<float>(2 * acc[m] - an), inner[m]);
  }
#pragma unroll
  for (int m = 0; m < NM; ++m) {
    if constexpr (kInner) {
      part[m][0] = inner[m];
      sc_out[m] = sc[m];
    } else {
      part[m][0] = __fmaf_rn(sc[m], inner[m], part[m][0]);
    }
  }
}

// Dispatch on the number of pairs of the item (1, 2, 4 or 8 vectors).
template <int NM, int NTMAX>
__device__ __forceinline__ void block_dot_n(int count, const unsigned char* wsrc, const int* q4, int qs,
                                            const float* ds, const int* as, int dsn, int lane,
                                            float (&part)[NM][NTMAX]) {
  if constexpr (NTMAX == 1) {
    block_dot<NM, 1, 1>(wsrc, q4, qs, ds, as, dsn, lane, part);
  } else {
    if (count <= 1) block_dot<NM, 1, NTMAX>(wsrc, q4, qs, ds, as, dsn, lane, part);
    else if (count <= 2) block_dot<NM, 2, NTMAX>(wsrc, q4, qs, ds, as, dsn, lane, part);
    else if (count <= 4) block_dot<NM, 4, NTMAX>(wsrc, q4, qs, ds, as, dsn, lane, part);
    else block_dot<NM, 8, NTMAX>(wsrc, q4, qs, ds, as, dsn, lane, part);
  }
}

// Stage one activation vector (k codes, k/32 scales) and its block sums in
// shared memory; all threads of the CTA take part.
__device__ __forceinline__ void stage_vector(const int8_t* __restrict__ codes, const float* __restrict__ scales,
                                             int k, int* q4, float* d, int* as) {
  const int* src = reinterpret_cast<const int*>(codes);
  for (int i = threadIdx.x; i < k / 4; i += blockDim.x) q4[i] = src[i];
  for (int i = threadIdx.x; i < k / kQBlock; i += blockDim.x) {
    d[i] = scales[i];
    int sum = 0;
#pragma unroll
    for (int j = 0; j < kQBlock / 4; ++j) sum = __dp4a(src[i * 8 + j], 0x01010101, sum);
    as[i] = sum;
  }
}


}  // namespace bitmoe
