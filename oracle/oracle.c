/*
 * oracle.c -- plain single-threaded CPU oracle for the ternary routed-expert
 * MoE hot path.  TEST INFRASTRUCTURE ONLY: used by the tests, the smoke check
 * and the benchmark's CPU-baseline leg, never by the product path.
 *
 * Written for clarity, not speed: each function follows its definition step
 * by step.  Compile with -O2 -ffp-contract=off (no fused multiply-adds other
 * than the explicit fmaf calls of the router).  See oracle.h for the sources
 * each definition follows.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ======================================================================== */
/* IEEE binary16                                                             */
/* ======================================================================== */

uint16_t orc_f16_from_f64(double x) {
  uint16_t sign = signbit(x) ? 0x8000u : 0u;
  double a = fabs(x);
  if (isnan(x)) return (uint16_t)(sign | 0x7E00u);
  /* 65520 is halfway between the largest finite half (65504) and 2^16; a tie
     there rounds to the even neighbour 2^16, which is out of range.        */
  if (a >= 65520.0) return (uint16_t)(sign | 0x7C00u);
  if (a < ldexp(1.0, -14)) {
    /* subnormal range: value = m * 2^-24 with integer m in [0, 1024]; m = 1024
       is the smallest normal, whose encoding 0x0400 continues the sequence. */
    double m = rint(ldexp(a, 24));  /* default rounding mode: ties to even */
    return (uint16_t)(sign | (uint16_t)m);
  }
  int e2;
  (void)frexp(a, &e2);              /* a = f * 2^e2, f in [0.5, 1)           */
  int E = e2 - 1;                   /* a = (2f) * 2^E, E in [-14, 15]        */
  double m = rint(ldexp(a, 10 - E)); /* in [1024, 2048]; 2048 carries into E */
  uint32_t bits = ((uint32_t)(E + 15) << 10) + (uint32_t)(m - 1024.0);
  return (uint16_t)(sign | bits);
}

float orc_f16_to_f32(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int m = h & 0x3FF;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24);
  } else if (e == 31) {
    v = m ? NAN : INFINITY;
  } else {
    v = ldexp((double)(1024 + m), e - 25);
  }
  return (float)(sign ? -v : v);
}

/* ======================================================================== */
/* base-3 bytes                                                              */
/* ======================================================================== */
/* Reading: five ternary digits per byte (243 <= 256).  The byte holds the
   base-3 number v = sum_i t_i 3^(4-i) as a fixed-point fraction of 243,
   u = ceil(v * 256 / 243), so that multiplying u by 3 and taking the high
   part peels off one digit at a time.  Decoding here does not use that
   property: it recovers v and divides.                                    */

uint8_t orc_trit_byte_encode(const int t[5]) {
  int v = 0;
  for (int i = 0; i < 5; ++i) v = 3 * v + t[i];
  int u = (v * 256 + 242) / 243;    /* ceil(v*256/243) */
  return (uint8_t)u;
}

int orc_trit_byte_decode(uint8_t u, int t[5]) {
  int v = ((int)u * 243) >> 8;      /* floor(u*243/256) */
  if (v > 242) return -1;
  /* u must be exactly the encoding of v */
  if ((v * 256 + 242) / 243 != (int)u) return -1;
  for (int i = 4; i >= 0; --i) {
    t[i] = v % 3;
    v /= 3;
  }
  return 0;
}

/* ======================================================================== */
/* weight storage                                                            */
/* ======================================================================== */
/* Reading (storage order; no page prints one):
     - a block is 256 consecutive weights of one row;
     - packed word w (0..12) of a block holds, in its byte lane l (0..3),
       the five digits (level i = 0..4) of weights k = 20w + 4i + l; the
       last word has four levels and a pad digit t = 1 (weight 0) at i = 4;
     - rows are grouped into panels of 32 and the words of a panel are
       interleaved row by row: word (b, w) of the 32 rows of a panel are 32
       consecutive uint32;
     - the fp16 scales are interleaved the same way: scale b of the 32 rows
       of a panel are 32 consecutive uint16.                                */

int64_t orc_trit_words(int64_t rows, int64_t k) {
  return rows * (k / ORC_BLOCK) * ORC_BLOCK_WORDS;
}
int64_t orc_scale_count(int64_t rows, int64_t k) {
  return rows * (k / ORC_BLOCK);
}
int64_t orc_word_index(int64_t k, int64_t r, int64_t b, int w) {
  int64_t nb = k / ORC_BLOCK;
  int64_t p = r / ORC_PANEL;
  return ((p * nb + b) * ORC_BLOCK_WORDS + w) * ORC_PANEL + (r % ORC_PANEL);
}
int64_t orc_scale_index(int64_t k, int64_t r, int64_t b) {
  int64_t nb = k / ORC_BLOCK;
  int64_t p = r / ORC_PANEL;
  return (p * nb + b) * ORC_PANEL + (r % ORC_PANEL);
}

/* Absmean ternarization of one 256-weight block (reading of "ternary"
   routed-expert weights: the BitNet b1.58 absmean rule, applied per block):
     s = fp16_RNE( (sum_k |w_k| in fp64, k ascending) / 256 )
     q_k = sign(w_k) if |w_k| >= 0.5 * s (compared in fp32), else 0,
   which is round-half-away(w/s) clipped to [-1, 1] without a division.   */
static void quantize_block(const float* w, uint16_t* s_out, int8_t q[256]) {
  double sum = 0.0;
  for (int k = 0; k < 256; ++k) sum += fabs((double)w[k]);
  uint16_t s = orc_f16_from_f64(sum / 256.0);
  float half = 0.5f * orc_f16_to_f32(s);
  for (int k = 0; k < 256; ++k) {
    float a = fabsf(w[k]);
    if (a >= half && w[k] != 0.0f) {
      q[k] = (int8_t)(w[k] > 0.0f ? 1 : -1);
    } else {
      q[k] = 0;
    }
  }
  *s_out = s;
}

int orc_quantize_weights(const float* w, int64_t rows, int64_t k,
                         uint32_t* trits, uint16_t* scales) {
  if (rows <= 0 || k <= 0 || rows % ORC_PANEL || k % ORC_BLOCK) return -1;
  int64_t nb = k / ORC_BLOCK;
  int8_t q[256];
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      uint16_t s;
      quantize_block(w + r * k + b * ORC_BLOCK, &s, q);
      scales[orc_scale_index(k, r, b)] = s;
      for (int wd = 0; wd < ORC_BLOCK_WORDS; ++wd) {
        uint32_t word = 0;
        for (int l = 0; l < 4; ++l) {
          int t[5];
          for (int i = 0; i < 5; ++i) {
            int kk = 20 * wd + 4 * i + l;
            t[i] = (kk < ORC_BLOCK) ? q[kk] + 1 : 1; /* pad digit: weight 0 */
          }
          word |= (uint32_t)orc_trit_byte_encode(t) << (8 * l);
        }
        trits[orc_word_index(k, r, b, wd)] = word;
      }
    }
  }
  return 0;
}

int orc_unpack_weights(const uint32_t* trits, const uint16_t* scales,
                       int64_t rows, int64_t k, int64_t row0, int64_t nrows,
                       int8_t* q, float* s) {
  if (rows <= 0 || k <= 0 || rows % ORC_PANEL || k % ORC_BLOCK) return -1;
  if (row0 < 0 || nrows < 0 || row0 + nrows > rows) return -1;
  int64_t nb = k / ORC_BLOCK;
  for (int64_t rr = 0; rr < nrows; ++rr) {
    int64_t r = row0 + rr;
    for (int64_t b = 0; b < nb; ++b) {
      if (s) s[rr * nb + b] = orc_f16_to_f32(scales[orc_scale_index(k, r, b)]);
      for (int wd = 0; wd < ORC_BLOCK_WORDS; ++wd) {
        uint32_t word = trits[orc_word_index(k, r, b, wd)];
        for (int l = 0; l < 4; ++l) {
          int t[5];
          if (orc_trit_byte_decode((uint8_t)(word >> (8 * l)), t)) return -1;
          for (int i = 0; i < 5; ++i) {
            int kk = 20 * wd + 4 * i + l;
            if (kk < ORC_BLOCK) q[rr * k + b * ORC_BLOCK + kk] = (int8_t)(t[i] - 1);
          }
        }
      }
    }
  }
  return 0;
}

/* ======================================================================== */
/* 1-bit sign codes                                                          */
/* ======================================================================== */
/* The PXQ1 tier of the pxq_llama README ("What's PXQ?": 1-bit sign codes
   times scales), read with this build's block and scale: per 256-weight
   block s = fp16_RNE(sum|w| / 256) as for the ternary format (for codes of
   +-1 this mean is also the scale of least squared error), q = -1 where
   w < 0 and +1 otherwise.  Storage: 8 words per block, word j holding the
   32 weights of activation block j, weight 32j + 4i + l in bit 8l + i (so
   that the bits of four consecutive weights sit in the four bytes of a word
   at the same position), a set bit meaning +1; words and scales interleaved
   over 32-row panels exactly as the ternary words and scales.            */
int64_t orc_sign_words(int64_t rows, int64_t k) {
  return rows * (k / ORC_BLOCK) * ORC_SIGN_WORDS;
}
int64_t orc_sign_word_index(int64_t k, int64_t r, int64_t b, int w) {
  int64_t nb = k / ORC_BLOCK;
  int64_t p = r / ORC_PANEL;
  return ((p * nb + b) * ORC_SIGN_WORDS + w) * ORC_PANEL + (r % ORC_PANEL);
}

int orc_quantize_weights_sign(const float* w, int64_t rows, int64_t k,
                              uint32_t* codes, uint16_t* scales) {
  if (rows <= 0 || k <= 0 || rows % ORC_PANEL || k % ORC_BLOCK) return -1;
  int64_t nb = k / ORC_BLOCK;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      const float* wb = w + r * k + b * ORC_BLOCK;
      double sum = 0.0;
      for (int kk = 0; kk < ORC_BLOCK; ++kk) sum += fabs((double)wb[kk]);
      scales[orc_scale_index(k, r, b)] = orc_f16_from_f64(sum / 256.0);
      for (int j = 0; j < ORC_SIGN_WORDS; ++j) {
        uint32_t word = 0;
        for (int i = 0; i < 8; ++i) {
          for (int l = 0; l < 4; ++l) {
            int kk = 32 * j + 4 * i + l;
            if (!(wb[kk] < 0.0f)) word |= 1u << (8 * l + i);
          }
        }
        codes[orc_sign_word_index(k, r, b, j)] = word;
      }
    }
  }
  return 0;
}

int orc_unpack_weights_sign(const uint32_t* codes, const uint16_t* scales,
                            int64_t rows, int64_t k, int64_t row0,
                            int64_t nrows, int8_t* q, float* s) {
  if (rows <= 0 || k <= 0 || rows % ORC_PANEL || k % ORC_BLOCK) return -1;
  if (row0 < 0 || nrows < 0 || row0 + nrows > rows) return -1;
  int64_t nb = k / ORC_BLOCK;
  for (int64_t rr = 0; rr < nrows; ++rr) {
    int64_t r = row0 + rr;
    for (int64_t b = 0; b < nb; ++b) {
      if (s) s[rr * nb + b] = orc_f16_to_f32(scales[orc_scale_index(k, r, b)]);
      for (int j = 0; j < ORC_SIGN_WORDS; ++j) {
        uint32_t word = codes[orc_sign_word_index(k, r, b, j)];
        for (int i = 0; i < 8; ++i) {
          for (int l = 0; l < 4; ++l) {
            int kk = 32 * j + 4 * i + l;
            q[rr * k + b * ORC_BLOCK + kk] = (int8_t)(((word >> (8 * l + i)) & 1u) ? 1 : -1);
          }
        }
      }
    }
  }
  return 0;
}

/* ======================================================================== */
/* two-level scales (E16)                                                    */
/* ======================================================================== */
/* The E16-row scales of the pxq_llama README ("What's PXQ?"), read onto the
   ternary digits (see oracle.h): one fp16 anchor per row, a 4-bit code per
   16-weight block, s_h = A * (c_h + 1) / 16.                              */
int64_t orc_e16_code_words(int64_t rows, int64_t k) {
  return rows * (k / ORC_BLOCK) * ORC_E16_WORDS;
}
int64_t orc_e16_code_index(int64_t k, int64_t r, int64_t b, int u) {
  int64_t nb = k / ORC_BLOCK;
  int64_t p = r / ORC_PANEL;
  return ((p * nb + b) * ORC_E16_WORDS + u) * ORC_PANEL + (r % ORC_PANEL);
}

static double mean_abs16(const float* w) {
  double sum = 0.0;
  for (int i = 0; i < 16; ++i) sum += fabs((double)w[i]);
  return sum / 16.0;
}

int orc_quantize_weights_e16(const float* w, int64_t rows, int64_t k,
                             uint32_t* trits, uint32_t* codes,
                             uint16_t* anchors) {
  if (rows <= 0 || k <= 0 || rows % ORC_PANEL || k % ORC_BLOCK) return -1;
  int64_t nb = k / ORC_BLOCK;
  int8_t q[256];
  for (int64_t r = 0; r < rows; ++r) {
    const float* wr = w + r * k;
    double mmax = 0.0;
    for (int64_t h = 0; h < k / 16; ++h) {
      double m = mean_abs16(wr + 16 * h);
      if (m > mmax) mmax = m;
    }
    uint16_t ah = orc_f16_from_f64(mmax);
    anchors[r] = ah;
    double a = (double)orc_f16_to_f32(ah);
    for (int64_t b = 0; b < nb; ++b) {
      uint32_t cw[ORC_E16_WORDS] = {0, 0};
      for (int h = 0; h < 16; ++h) {
        const float* wb = wr + b * ORC_BLOCK + 16 * h;
        int c = 0;
        if (a > 0.0) {
          double t = rint(16.0 * mean_abs16(wb) / a) - 1.0;
          c = t < 0.0 ? 0 : (t > 15.0 ? 15 : (int)t);
        }
        cw[h / 8] |= (uint32_t)c << (4 * (h % 8));
        float half = 0.5f * (float)(a * (c + 1) / 16.0);
        for (int i = 0; i < 16; ++i) {
          float x = wb[i];
          q[16 * h + i] = (fabsf(x) >= half && x != 0.0f) ? (int8_t)(x > 0.0f ? 1 : -1) : 0;
        }
      }
      for (int u = 0; u < ORC_E16_WORDS; ++u) codes[orc_e16_code_index(k, r, b, u)] = cw[u];
      for (int wd = 0; wd < ORC_BLOCK_WORDS; ++wd) {
        uint32_t word = 0;
        for (int l = 0; l < 4; ++l) {
          int t[5];
          for (int i = 0; i < 5; ++i) {
            int kk = 20 * wd + 4 * i + l;
            t[i] = (kk < ORC_BLOCK) ? q[kk] + 1 : 1;
          }
          word |= (uint32_t)orc_trit_byte_encode(t) << (8 * l);
        }
        trits[orc_word_index(k, r, b, wd)] = word;
      }
    }
  }
  return 0;
}

int orc_unpack_weights_e16(const uint32_t* trits, const uint32_t* codes,
                           const uint16_t* anchors, int64_t rows, int64_t k,
                           int64_t row0, int64_t nrows, int8_t* q,
                           float* s16) {
  if (rows <= 0 || k <= 0 || rows % ORC_PANEL || k % ORC_BLOCK) return -1;
  if (row0 < 0 || nrows < 0 || row0 + nrows > rows) return -1;
  int64_t nb = k / ORC_BLOCK;
  /* the digits are those of the ternary format; the scales come from the
     anchor and the codes */
  if (orc_unpack_weights(trits, NULL, rows, k, row0, nrows, q, NULL)) return -1;
  for (int64_t rr = 0; rr < nrows; ++rr) {
    int64_t r = row0 + rr;
    double a = (double)orc_f16_to_f32(anchors[r]);
    for (int64_t b = 0; b < nb; ++b) {
      for (int h = 0; h < 16; ++h) {
        uint32_t cw = codes[orc_e16_code_index(k, r, b, h / 8)];
        int c = (int)((cw >> (4 * (h % 8))) & 15u);
        s16[rr * (k / 16) + b * 16 + h] = (float)(a * (c + 1) / 16.0);
      }
    }
  }
  return 0;
}

void orc_matvec_e16(const int8_t* q, const float* s16, int64_t rows,
                    int64_t k, const int8_t* xq, const float* xd,
                    double* out) {
  for (int64_t r = 0; r < rows; ++r) {
    double acc = 0.0;
    for (int64_t j = 0; j < k / ORC_QBLOCK; ++j) {
      double inner = 0.0;
      for (int half = 0; half < 2; ++half) {
        int64_t h = 2 * j + half;
        int32_t isum = 0;
        for (int i = 0; i < 16; ++i) {
          int64_t kk = 16 * h + i;
          isum += (int32_t)q[r * k + kk] * (int32_t)xq[kk];
        }
        inner += (double)s16[r * (k / 16) + h] * (double)isum;
      }
      acc += (double)xd[j] * inner;
    }
    out[r] = acc;
  }
}

/* ======================================================================== */
/* activation quantization                                                   */
/* ======================================================================== */
/* int8 activations with one fp32 scale per 32 values (Parakon Runtime README
   "How it works"; pxq_llama README "PXQ vs MXFP4").  Reading of the rounding:
     amax = max |x| over the block, d = amax / 127 (IEEE fp32 division),
     q = clamp(rint(x / d), -127, 127) with IEEE fp32 division and ties to
     even; a block whose d is 0 (amax = 0, or amax/127 underflowing to 0)
     gets q = 0.                                                           */
int orc_quant_act_q8(const float* x, int64_t ntok, int64_t k, int8_t* xq,
                     float* xd) {
  if (k <= 0 || k % ORC_QBLOCK) return -1;
  int64_t nq = k / ORC_QBLOCK;
  for (int64_t t = 0; t < ntok; ++t) {
    for (int64_t j = 0; j < nq; ++j) {
      const float* xb = x + t * k + j * ORC_QBLOCK;
      int8_t* qb = xq + t * k + j * ORC_QBLOCK;
      float amax = 0.0f;
      for (int i = 0; i < ORC_QBLOCK; ++i) {
        float a = fabsf(xb[i]);
        if (a > amax) amax = a;
      }
      float d = amax / 127.0f;
      xd[t * nq + j] = d;
      for (int i = 0; i < ORC_QBLOCK; ++i) {
        if (d == 0.0f) { /* amax = 0, or amax/127 below the smallest subnormal */
          qb[i] = 0;
          continue;
        }
        float v = rintf(xb[i] / d);
        if (v > 127.0f) v = 127.0f;
        if (v < -127.0f) v = -127.0f;
        qb[i] = (int8_t)v;
      }
    }
  }
  return 0;
}

/* ======================================================================== */
/* block sums and mat-vec                                                    */
/* ======================================================================== */
/* Per 32-value block, the int8 x ternary dot product is exact in int32; the
   scales are applied once per block (pxq_llama README, "PXQ vs MXFP4": one
   scale fixup per 32-value block) and the weight scale once per 256 block. */
void orc_blocksums(const int8_t* q, int64_t rows, int64_t k, const int8_t* xq,
                   int32_t* isum) {
  int64_t nq = k / ORC_QBLOCK;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t j = 0; j < nq; ++j) {
      int32_t acc = 0;
      for (int i = 0; i < ORC_QBLOCK; ++i) {
        int64_t kk = j * ORC_QBLOCK + i;
        acc += (int32_t)q[r * k + kk] * (int32_t)xq[kk];
      }
      isum[r * nq + j] = acc;
    }
  }
}

void orc_matvec(const int8_t* q, const float* s, int64_t rows, int64_t k,
                const int8_t* xq, const float* xd, double* out) {
  int64_t nq = k / ORC_QBLOCK;
  int64_t nb = k / ORC_BLOCK;
  int32_t* isum = (int32_t*)malloc(sizeof(int32_t) * (size_t)nq);
  for (int64_t r = 0; r < rows; ++r) {
    orc_blocksums(q + r * k, 1, k, xq, isum);
    double acc = 0.0;
    for (int64_t b = 0; b < nb; ++b) {
      double inner = 0.0;
      for (int j = 0; j < ORC_BLOCK / ORC_QBLOCK; ++j) {
        int64_t jj = b * (ORC_BLOCK / ORC_QBLOCK) + j;
        inner += (double)xd[jj] * (double)isum[jj];
      }
      acc += (double)s[r * nb + b] * inner;
    }
    out[r] = acc;
  }
  free(isum);
}

/* ======================================================================== */
/* router                                                                    */
/* ======================================================================== */
/* Reading: the router is a dense fp32 matrix; its logits decide which experts
   run, so both implementations must take that decision on the same fp32
   numbers.  The order fixed here: 32 partial sums p_l, p_l accumulating
   fmaf(w[k], x[k], p_l) over k = l, l+32, l+64, ... ascending from 0, then
   five pairwise rounds p_l <- p_l + p_(l xor m) for m = 16, 8, 4, 2, 1; the
   logit is the final p_0.                                                 */
static float router_logit(const float* x, const float* wr_row, int64_t hidden) {
  float p[32], nx[32];
  for (int l = 0; l < 32; ++l) {
    p[l] = 0.0f;
    for (int64_t kk = l; kk < hidden; kk += 32) p[l] = fmaf(wr_row[kk], x[kk], p[l]);
  }
  for (int m = 16; m >= 1; m >>= 1) {
    for (int l = 0; l < 32; ++l) nx[l] = p[l] + p[l ^ m];
    for (int l = 0; l < 32; ++l) p[l] = nx[l];
  }
  return p[0];
}

int orc_router_logits(const float* x, const float* wr, int64_t ntok,
                      int64_t hidden, int64_t n_experts, float* logits) {
  if (hidden <= 0 || hidden % 32) return -1;
  for (int64_t t = 0; t < ntok; ++t)
    for (int64_t e = 0; e < n_experts; ++e)
      logits[t * n_experts + e] = router_logit(x + t * hidden, wr + e * hidden, hidden);
  return 0;
}

/* Top-k routing with every selected expert evaluated (llama-modchip page,
   "Key highlights": all Top-k experts, no dropping).  Reading: experts are
   ranked by logit, larger first, equal logits by lower id; the weights are
   the softmax over all experts renormalised over the k selected, i.e.
   w_i = exp(l_i - l_max) / sum_{j in top-k} exp(l_j - l_max), in fp64.   */
int orc_route_topk(const float* x, const float* wr, int64_t ntok,
                   int64_t hidden, int64_t n_experts, int64_t top_k,
                   int32_t* idx, double* wts) {
  if (hidden <= 0 || hidden % 32 || top_k < 1 || top_k > n_experts) return -1;
  float* lg = (float*)malloc(sizeof(float) * (size_t)n_experts);
  unsigned char* used = (unsigned char*)malloc((size_t)n_experts);
  for (int64_t t = 0; t < ntok; ++t) {
    orc_router_logits(x + t * hidden, wr, 1, hidden, n_experts, lg);
    memset(used, 0, (size_t)n_experts);
    for (int64_t j = 0; j < top_k; ++j) {
      int64_t best = -1;
      for (int64_t e = 0; e < n_experts; ++e) {
        if (used[e]) continue;
        if (best < 0 || lg[e] > lg[best]) best = e; /* strict: ties keep lower id */
      }
      used[best] = 1;
      idx[t * top_k + j] = (int32_t)best;
    }
    double lmax = (double)lg[idx[t * top_k]];
    double den = 0.0;
    for (int64_t j = 0; j < top_k; ++j) den += exp((double)lg[idx[t * top_k + j]] - lmax);
    for (int64_t j = 0; j < top_k; ++j)
      wts[t * top_k + j] = exp((double)lg[idx[t * top_k + j]] - lmax) / den;
  }
  free(lg);
  free(used);
  return 0;
}

/* ======================================================================== */
/* expert FFN                                                                */
/* ======================================================================== */
/* For each token t and slot j with expert e = idx[t][j] (reading of the
   gate/up SiLU unary followed by down, pxq_llama README "Updates --
   2026-07-28"; activations requantized to int8 between the two mat-vecs so
   that the down mat-vec is also int8 x ternary, Parakon Runtime README
   "How it works"):
     g = Wg_e . x^, u = Wu_e . x^                 (orc_matvec, fp64)
     a = g / (1 + exp(-g)) * u                    (fp64, rounded to fp32)
     (aq, ad) = q8(a)                             (orc_quant_act_q8)
     y_e = Wd_e . a^                              (orc_matvec, fp64)
     y_t = sum_j wts[t][j] * y_e                  (fp64, slots in order)
   Experts are visited one at a time (each expert's rows are expanded once
   per call); the per-slot results are kept and summed in slot order, so the
   visiting order does not change any value.                               */
int orc_expert_ffn(const orc_layer* L, int64_t ntok, const int8_t* xq,
                   const float* xd, const int32_t* idx, const float* wts,
                   double* y, double* g_out, double* u_out, int8_t* aq_out,
                   float* ad_out) {
  int64_t H = L->hidden, F = L->ffn, E = L->n_experts, K = L->top_k;
  if (H <= 0 || F <= 0 || E <= 0 || K < 1 || K > E) return -1;
  if (L->format != ORC_FORMAT_TERNARY && L->format != ORC_FORMAT_SIGN && L->format != ORC_FORMAT_E16)
    return -1;
  if (H % ORC_BLOCK || F % ORC_BLOCK || F % ORC_PANEL || H % ORC_PANEL) return -1;
  for (int64_t i = 0; i < ntok * K; ++i)
    if (idx[i] < 0 || idx[i] >= E) return -2;

  int64_t nbH = H / ORC_BLOCK, nbF = F / ORC_BLOCK;
  int8_t* qg = (int8_t*)malloc((size_t)(F * H));
  int8_t* qu = (int8_t*)malloc((size_t)(F * H));
  int8_t* qd = (int8_t*)malloc((size_t)(H * F));
  /* block scales: one per 256 weights, or one per 16 (ORC_FORMAT_E16) */
  const int64_t per = L->format == ORC_FORMAT_E16 ? ORC_BLOCK / 16 : 1;
  float* sg = (float*)malloc(sizeof(float) * (size_t)(F * nbH * per));
  float* su = (float*)malloc(sizeof(float) * (size_t)(F * nbH * per));
  float* sd = (float*)malloc(sizeof(float) * (size_t)(H * nbF * per));
  double* g = (double*)malloc(sizeof(double) * (size_t)F);
  double* u = (double*)malloc(sizeof(double) * (size_t)F);
  float* a = (float*)malloc(sizeof(float) * (size_t)F);
  int8_t* aq = (int8_t*)malloc((size_t)F);
  float* ad = (float*)malloc(sizeof(float) * (size_t)(F / ORC_QBLOCK));
  double* ye = (double*)malloc(sizeof(double) * (size_t)(ntok * K * H));
  int rc = 0;

  for (int64_t e = 0; e < E && rc == 0; ++e) {
    int used = 0;
    for (int64_t i = 0; i < ntok * K; ++i) used |= (idx[i] == e);
    if (!used) continue;
    int bad;
    if (L->format == ORC_FORMAT_E16) {
      bad = orc_unpack_weights_e16(L->gate_trits, L->gate_codes, L->gate_scales, E * F, H, e * F, F, qg, sg) ||
            orc_unpack_weights_e16(L->up_trits, L->up_codes, L->up_scales, E * F, H, e * F, F, qu, su) ||
            orc_unpack_weights_e16(L->down_trits, L->down_codes, L->down_scales, E * H, F, e * H, H, qd, sd);
    } else {
      int (*unpack)(const uint32_t*, const uint16_t*, int64_t, int64_t, int64_t, int64_t, int8_t*, float*) =
          L->format == ORC_FORMAT_SIGN ? orc_unpack_weights_sign : orc_unpack_weights;
      bad = unpack(L->gate_trits, L->gate_scales, E * F, H, e * F, F, qg, sg) ||
            unpack(L->up_trits, L->up_scales, E * F, H, e * F, F, qu, su) ||
            unpack(L->down_trits, L->down_scales, E * H, F, e * H, H, qd, sd);
    }
    if (bad) {
      rc = -1;
      break;
    }
    for (int64_t t = 0; t < ntok; ++t) {
      for (int64_t j = 0; j < K; ++j) {
        if (idx[t * K + j] != e) continue;
        const int8_t* xt = xq + t * H;
        const float* dt = xd + t * (H / ORC_QBLOCK);
        void (*matvec)(const int8_t*, const float*, int64_t, int64_t, const int8_t*, const float*, double*) =
            L->format == ORC_FORMAT_E16 ? orc_matvec_e16 : orc_matvec;
        matvec(qg, sg, F, H, xt, dt, g);
        matvec(qu, su, F, H, xt, dt, u);
        for (int64_t f = 0; f < F; ++f) a[f] = (float)(g[f] / (1.0 + exp(-g[f])) * u[f]);
        orc_quant_act_q8(a, 1, F, aq, ad);
        matvec(qd, sd, H, F, aq, ad, ye + (t * K + j) * H);
        int64_t o = t * K + j;
        if (g_out) memcpy(g_out + o * F, g, sizeof(double) * (size_t)F);
        if (u_out) memcpy(u_out + o * F, u, sizeof(double) * (size_t)F);
        if (aq_out) memcpy(aq_out + o * F, aq, (size_t)F);
        if (ad_out) memcpy(ad_out + o * (F / ORC_QBLOCK), ad, sizeof(float) * (size_t)(F / ORC_QBLOCK));
      }
    }
  }
  if (rc == 0) {
    for (int64_t t = 0; t < ntok; ++t) {
      for (int64_t h = 0; h < H; ++h) {
        double acc = 0.0;
        for (int64_t j = 0; j < K; ++j) acc += (double)wts[t * K + j] * ye[(t * K + j) * H + h];
        y[t * H + h] = acc;
      }
    }
  }
  free(qg); free(qu); free(qd); free(sg); free(su); free(sd);
  free(g); free(u); free(a); free(aq); free(ad); free(ye);
  return rc;
}

/* ======================================================================== */
/* shared expert (8-bit blocks)                                              */
/* ======================================================================== */
/* The shared expert beside the routed ones stays at higher precision
   (llama-modchip page, "The interesting bit"); read here as 8-bit blocks of
   32 weights with an fp16 scale (see oracle.h).                           */
int orc_quantize_weights_q8(const float* w, int64_t rows, int64_t k, int8_t* q,
                            uint16_t* d) {
  if (rows <= 0 || k <= 0 || k % ORC_QBLOCK) return -1;
  int64_t nq = k / ORC_QBLOCK;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t j = 0; j < nq; ++j) {
      const float* wb = w + r * k + j * ORC_QBLOCK;
      double amax = 0.0;
      for (int i = 0; i < ORC_QBLOCK; ++i) {
        double a = fabs((double)wb[i]);
        if (a > amax) amax = a;
      }
      uint16_t dh = orc_f16_from_f64(amax / 127.0);
      d[r * nq + j] = dh;
      float df = orc_f16_to_f32(dh);
      for (int i = 0; i < ORC_QBLOCK; ++i) {
        int8_t v = 0;
        if (df != 0.0f) {
          float t = rintf(wb[i] / df);
          if (t > 127.0f) t = 127.0f;
          if (t < -127.0f) t = -127.0f;
          v = (int8_t)t;
        }
        q[r * k + j * ORC_QBLOCK + i] = v;
      }
    }
  }
  return 0;
}

void orc_matvec_q8(const int8_t* q, const uint16_t* d, int64_t rows, int64_t k,
                   const int8_t* xq, const float* xd, double* out) {
  int64_t nq = k / ORC_QBLOCK;
  for (int64_t r = 0; r < rows; ++r) {
    double acc = 0.0;
    for (int64_t j = 0; j < nq; ++j) {
      int32_t isum = 0;
      for (int i = 0; i < ORC_QBLOCK; ++i)
        isum += (int32_t)q[r * k + j * ORC_QBLOCK + i] * (int32_t)xq[j * ORC_QBLOCK + i];
      acc += (double)orc_f16_to_f32(d[r * nq + j]) * (double)xd[j] * (double)isum;
    }
    out[r] = acc;
  }
}

int orc_shared_ffn(int64_t hidden, int64_t ffn, const int8_t* gq, const uint16_t* gd,
                   const int8_t* uq, const uint16_t* ud, const int8_t* dq,
                   const uint16_t* dd, int64_t ntok, const int8_t* xq,
                   const float* xd, double* y) {
  int64_t H = hidden, F = ffn;
  if (H <= 0 || F <= 0 || H % ORC_QBLOCK || F % ORC_QBLOCK) return -1;
  double* g = (double*)malloc(sizeof(double) * (size_t)F);
  double* u = (double*)malloc(sizeof(double) * (size_t)F);
  float* a = (float*)malloc(sizeof(float) * (size_t)F);
  int8_t* aq = (int8_t*)malloc((size_t)F);
  float* ad = (float*)malloc(sizeof(float) * (size_t)(F / ORC_QBLOCK));
  double* ys = (double*)malloc(sizeof(double) * (size_t)H);
  for (int64_t t = 0; t < ntok; ++t) {
    const int8_t* xt = xq + t * H;
    const float* dt = xd + t * (H / ORC_QBLOCK);
    orc_matvec_q8(gq, gd, F, H, xt, dt, g);
    orc_matvec_q8(uq, ud, F, H, xt, dt, u);
    for (int64_t f = 0; f < F; ++f) a[f] = (float)(g[f] / (1.0 + exp(-g[f])) * u[f]);
    orc_quant_act_q8(a, 1, F, aq, ad);
    orc_matvec_q8(dq, dd, H, F, aq, ad, ys);
    for (int64_t h = 0; h < H; ++h) y[t * H + h] += ys[h];
  }
  free(g); free(u); free(a); free(aq); free(ad); free(ys);
  return 0;
}
