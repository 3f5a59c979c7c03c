// ternary_dot.cuh -- in-register base-3 decode and int8 dot products of
// 32-row panels of ternary blocks against NT int8 activation vectors (sm_100a).
//
// Weights stay packed in HBM and are decoded in registers only (Parakon
// Runtime README, "How it works": fused mat-vec over the quantized blocks,
// int8 activations, dp4a).  One thread owns one row of a 32-row panel; the 13
// packed words of a block are loaded per lane (32 lanes read 128 contiguous
// bytes per word).  Each decoded digit word is used for NT activation vectors
// (tokens routed to the same expert), so the decode cost is paid once per
// weight whatever the number of tokens.
//
// Decode of one packed byte u = ceil(v * 256 / 243): with P_i = u * 3^i (it
// fits 16 bits for i <= 5), the high byte H_i = floor(P_i / 256) equals
// floor(v / 3^(5-i)), so base-3 digit i is t_i = H_(i+1) - 3 * H_i.  The four
// bytes of a word are split into two registers of two 16-bit lanes
// (bytes 0,2 and bytes 1,3), multiplied by 3 per level, and the four high
// bytes are gathered back with one byte permute; the digit word
// H_(i+1) - 3*H_i is then one 32-bit multiply-add (each byte of 3*H_i is at
// most 240 and each byte difference is in {0,1,2}, so no carry or borrow
// crosses a byte).  The digits t = q + 1 are unsigned; dp4a against the
// activation word gives sum t*a, and sum q*a = sum t*a - sum a, where sum a is
// the precomputed sum of the 32-value activation block.
//
// Scales (pxq_llama README, "PXQ vs MXFP4": one fixup per 32-value block):
// per 32-block the exact int32 sum is scaled by the activation scale and
// accumulated in fp32 (sub-blocks in order), and the fp16 weight scale is
// applied once per 256-block.
//
// 1-bit sign codes (kSign; pxq_llama README, "What's PXQ?": the PXQ1 tier of
// sign codes times scales): 8 words per block, word j covering activation
// block j, weight 32j + 4i + l in bit 8l + i.  For group i of a word the
// digit word t = (w >> i) & 0x01010101 holds the bits of weights 4i..4i+3 in
// its four bytes, dp4a gives sum t*a, and with q = 2t - 1 the block sum is
// sum q*a = 2 * sum t*a - sum a.
//
// Shared-memory activation layout for NT vectors over a k-long dimension:
//   q4  [k/4][NT]  int32, four int8 codes each (token-minor, so the NT words
//                  of one group load as NT/4 128-bit broadcasts)
//   d   [k/32][NT] fp32 scales
//   as  [k/32][NT] int32 block sums of the codes
#pragma once

#include "common.cuh"

namespace bitmoe {

template <int NT>
struct ActSmem {
  static constexpr size_t bytes(int k) {
    return static_cast<size_t>(k / 4) * NT * 4 + 2 * static_cast<size_t>(k / kQBlock) * NT * 4;
  }
};

// Load the NT activation words of group g.
template <int NT>
__device__ __forceinline__ void load_group(const int* __restrict__ q4, int g, int (&a)[NT]) {
  if constexpr (NT % 4 == 0) {
#pragma unroll
    for (int n = 0; n < NT; n += 4) {
      const int4 v = *reinterpret_cast<const int4*>(q4 + g * NT + n);
      a[n] = v.x; a[n + 1] = v.y; a[n + 2] = v.z; a[n + 3] = v.w;
    }
  } else if constexpr (NT == 2) {
    const int2 v = *reinterpret_cast<const int2*>(q4 + g * NT);
    a[0] = v.x; a[1] = v.y;
  } else {
#pragma unroll
    for (int n = 0; n < NT; ++n) a[n] = q4[g * NT + n];
  }
}

// For NM matrices (same rows of different matrices, sharing the activations)
// and NT activation vectors: out[m][n] += sum over blocks b in
// [b_begin, b_end) step b_step of s[m][b] * sum_s d[s][n] * isum[m][n][s].
//   tw[m]: trits of matrix m at (panel, block 0), offset by lane
//   ts[m]: scales of matrix m at (panel, block 0), offset by lane
// If isum_out is not null (NM == 1), the exact block sums of the lane's row
// are stored at isum_out[n * isum_stride + s] for every global sub-block s.
template <int kSign>
struct WordsPerBlock {
  static constexpr int value = kSign ? kSignWords : kBlockWords;
};

template <int NM, int NT, bool kSign = false>
__device__ __forceinline__ void panel_dot(const uint32_t* const (&tw)[NM],
                                          const uint16_t* const (&ts)[NM], int b_begin, int b_end,
                                          int b_step, const int* __restrict__ q4,
                                          const float* __restrict__ d,
                                          const int* __restrict__ as, float (&out)[NM][NT],
                                          int32_t* isum_out = nullptr, size_t isum_stride = 0) {
  constexpr int kWords = WordsPerBlock<kSign>::value;
  // one matrix: the next block's words are loaded while this one decodes
  uint32_t wn[NM][WordsPerBlock<kSign>::value];
  uint16_t sn[NM];
  if (NM == 1 && b_begin < b_end) {
#pragma unroll
    for (int m = 0; m < NM; ++m) {
      const uint32_t* src = tw[m] + static_cast<size_t>(b_begin) * kWords * kPanel;
#pragma unroll
      for (int j = 0; j < kWords; ++j) wn[m][j] = ld_stream_u32(src + j * kPanel);
      sn[m] = ts[m][static_cast<size_t>(b_begin) * kPanel];
    }
  }
  for (int b = b_begin; b < b_end; b += b_step) {
    uint32_t w[NM][WordsPerBlock<kSign>::value];
    float sc[NM];
    if constexpr (NM == 1) {
#pragma unroll
      for (int m = 0; m < NM; ++m) {
#pragma unroll
        for (int j = 0; j < kWords; ++j) w[m][j] = wn[m][j];
        sc[m] = f16_bits_to_f32(sn[m]);
      }
      if (b + b_step < b_end) {
#pragma unroll
        for (int m = 0; m < NM; ++m) {
          const uint32_t* src = tw[m] + static_cast<size_t>(b + b_step) * kWords * kPanel;
#pragma unroll
          for (int j = 0; j < kWords; ++j) wn[m][j] = ld_stream_u32(src + j * kPanel);
          sn[m] = ts[m][static_cast<size_t>(b + b_step) * kPanel];
        }
      }
    } else {
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        const uint32_t* src = tw[m] + static_cast<size_t>(b) * kWords * kPanel;
#pragma unroll
        for (int j = 0; j < kWords; ++j) w[m][j] = ld_stream_u32(src + j * kPanel);
        sc[m] = f16_bits_to_f32(ts[m][static_cast<size_t>(b) * kPanel]);
      }
    }
    int acc[NM][NT];
    float inner[NM][NT];
#pragma unroll
    for (int m = 0; m < NM; ++m)
#pragma unroll
      for (int n = 0; n < NT; ++n) { acc[m][n] = 0; inner[m][n] = 0.f; }
    const int* qb = q4 + b * (kBlock / 4) * NT;
    if constexpr (kSign) {
#pragma unroll
      for (int j = 0; j < kSignWords; ++j) {  // word j = activation block j of the block
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          int a[NT];
          load_group<NT>(qb, 8 * j + i, a);
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            const int t = static_cast<int>((w[m][j] >> i) & 0x01010101u);
#pragma unroll
            for (int n = 0; n < NT; ++n) acc[m][n] = __dp4a(t, a[n], acc[m][n]);
          }
        }
        const int s = b * kSubPerBlock + j;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const float dn = d[s * NT + n];
          const int an = as[s * NT + n];
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            const int isum = 2 * acc[m][n] - an;
            inner[m][n] = __fmaf_rn(dn, static_cast<float>(isum), inner[m][n]);
            acc[m][n] = 0;
            if (NM == 1 && isum_out) isum_out[n * isum_stride + s] = isum;
          }
        }
      }
    } else {
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
          int a[NT];
          load_group<NT>(qb, g, a);
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
          if ((g & 7) == 7) {  // a 32-weight sub-block is complete
            const int s = b * kSubPerBlock + (g >> 3);
#pragma unroll
            for (int n = 0; n < NT; ++n) {
              const float dn = d[s * NT + n];
              const int an = as[s * NT + n];
#pragma unroll
              for (int m = 0; m < NM; ++m) {
                const int isum = acc[m][n] - an;
                inner[m][n] = __fmaf_rn(dn, static_cast<float>(isum), inner[m][n]);
                acc[m][n] = 0;
                if (NM == 1 && isum_out) isum_out[n * isum_stride + s] = isum;
              }
            }
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < NM; ++m)
#pragma unroll
      for (int n = 0; n < NT; ++n) out[m][n] = __fmaf_rn(sc[m], inner[m][n], out[m][n]);
  }
}

// Two-level (E16) scales (pxq_llama README, "What's PXQ?": a per-row fp16
// anchor A plus a 4-bit sub-scale per 16-element block): the ternary digits
// of panel_dot, and per 16-weight block h a code c_h with scale
// A * (c_h + 1) / 16.  Per 16-block the exact sum q.a = t.a - sum a is
// weighted by c_h + 1 (the activations' 16-sums come from dp4a against
// 0x01010101), per 32-block the weighted integer sum is scaled by the
// activation scale, and A / 16 (a16[m], exact) is applied once at the end.
//   tw[m]: digit words of matrix m at (panel, block 0), offset by lane
//   tc[m]: code words at (panel, block 0), offset by lane (kE16Words a block)
// If isum_out is not null (NM == 1), the weighted block sums
// sum_h (c_h + 1) * sum_{k in h} q * xq of every 32-block s are stored at
// isum_out[n * isum_stride + s].
template <int NM, int NT>
__device__ __forceinline__ void panel_dot_e16(const uint32_t* const (&tw)[NM], const uint32_t* const (&tc)[NM],
                                              const float (&a16)[NM], int b_begin, int b_end, int b_step,
                                              const int* __restrict__ q4, const float* __restrict__ d,
                                              float (&out)[NM][NT], int32_t* isum_out = nullptr,
                                              size_t isum_stride = 0) {
  float tot[NM][NT];
#pragma unroll
  for (int m = 0; m < NM; ++m)
#pragma unroll
    for (int n = 0; n < NT; ++n) tot[m][n] = 0.f;
  for (int b = b_begin; b < b_end; b += b_step) {
    uint32_t w[NM][kBlockWords];
    uint32_t cw[NM][kE16Words];
#pragma unroll
    for (int m = 0; m < NM; ++m) {
      const uint32_t* src = tw[m] + static_cast<size_t>(b) * kBlockWords * kPanel;
#pragma unroll
      for (int j = 0; j < kBlockWords; ++j) w[m][j] = ld_stream_u32(src + j * kPanel);
#pragma unroll
      for (int u = 0; u < kE16Words; ++u) cw[m][u] = ld_stream_u32(tc[m] + (static_cast<size_t>(b) * kE16Words + u) * kPanel);
    }
    int acc[NM][NT], accw[NM][NT], as16[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      as16[n] = 0;
#pragma unroll
      for (int m = 0; m < NM; ++m) { acc[m][n] = 0; accw[m][n] = 0; }
    }
    const int* qb = q4 + b * (kBlock / 4) * NT;
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
        int a[NT];
        load_group<NT>(qb, g, a);
#pragma unroll
        for (int n = 0; n < NT; ++n) as16[n] = __dp4a(a[n], 0x01010101, as16[n]);
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
        if ((g & 3) == 3) {  // a 16-weight block h = g / 4 is complete
          const int h = g >> 2;
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            const int cm = static_cast<int>((cw[m][h >> 3] >> (4 * (h & 7))) & 15u) + 1;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
              accw[m][n] += cm * (acc[m][n] - as16[n]);
              acc[m][n] = 0;
            }
          }
#pragma unroll
          for (int n = 0; n < NT; ++n) as16[n] = 0;
        }
        if ((g & 7) == 7) {  // a 32-weight activation block is complete
          const int s = b * kSubPerBlock + (g >> 3);
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            const float dn = d[s * NT + n];
#pragma unroll
            for (int m = 0; m < NM; ++m) {
              tot[m][n] = __fmaf_rn(dn, static_cast<float>(accw[m][n]), tot[m][n]);
              if (NM == 1 && isum_out) isum_out[n * isum_stride + s] = accw[m][n];
              accw[m][n] = 0;
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < NM; ++m)
#pragma unroll
    for (int n = 0; n < NT; ++n) out[m][n] = __fmaf_rn(a16[m], tot[m][n], out[m][n]);
}

// Stage activation vector n (k int8 codes with k/32 scales) into the
// token-minor shared layout; threads [tid0, tid0+nthr) take part.  The block
// sums are computed here from the codes.
template <int NT>
__device__ __forceinline__ void stage_act(const int8_t* __restrict__ xq,
                                          const float* __restrict__ xd, int k, int n, int* q4,
                                          float* d, int* as, int tid, int nthr) {
  const int* src = reinterpret_cast<const int*>(xq);
  for (int i = tid; i < k / 4; i += nthr) q4[i * NT + n] = src[i];
  for (int i = tid; i < k / kQBlock; i += nthr) {
    d[i * NT + n] = xd[i];
    int s = 0;
#pragma unroll
    for (int j = 0; j < kQBlock / 4; ++j) s = __dp4a(src[i * 8 + j], 0x01010101, s);
    as[i * NT + n] = s;
  }
}

// Fill vector slot n with zeros (an unused slot of a partly filled chunk).
template <int NT>
__device__ __forceinline__ void zero_act(int k, int n, int* q4, float* d, int* as, int tid,
                                         int nthr) {
  for (int i = tid; i < k / 4; i += nthr) q4[i * NT + n] = 0;
  for (int i = tid; i < k / kQBlock; i += nthr) { d[i * NT + n] = 0.f; as[i * NT + n] = 0; }
}

}  // namespace bitmoe
