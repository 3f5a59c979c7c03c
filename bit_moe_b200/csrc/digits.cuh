// digits.cuh -- base-3 digit words of a packed ternary block for the tensor
// cores (sm_100a): the digits t = q + 1 in {0, 1, 2}, four to a 32-bit word,
// in K order, as the A operand of the int8 MMAs.
//
// Packed word j of a block holds five levels of four bytes; level i of byte
// lane l is weight 20j + 4i + l, so digit word 5j + i (weights 4(5j+i) .. +3)
// is level i of packed word j.  Each byte u = ceil(v * 256 / 243) is peeled
// one base-3 digit per level: with P_i = u * 3^i in a 16-bit lane (it fits for
// i <= 5) and H_i its high byte, t_i = H_(i+1) - 3 * H_i.  The four bytes are
// split into two registers of two 16-bit lanes, multiplied by 3 per level,
// and the four high bytes gathered with one byte permute; the digit word is
// one multiply-add (no carry or borrow crosses a byte).  The last word's fifth
// level is the pad digit and is not produced.
#pragma once

#include "common.cuh"

namespace bitmoe {

// Digit words [32*kHalf, 32*kHalf + 32) of one block from packed words
// w[jj] = word 6*kHalf + jj, jj in [0, 7) (word 6 feeds both halves).
template <int kHalf>
__device__ __forceinline__ void digit_half(const uint32_t (&w)[7], uint32_t (&dg)[32]) {
  // level-major: the 7 words' chains advance side by side (7 independent
  // multiply chains per level), so one warp keeps its pipes busy
  uint32_t lo[7], hi[7], hp[7];
#pragma unroll
  for (int jj = 0; jj < 7; ++jj) {
    lo[jj] = w[jj] & 0x00FF00FFu;
    hi[jj] = __byte_perm(w[jj], 0u, 0x4341);
    hp[jj] = 0u;
  }
#pragma unroll
  for (int i = 0; i < 5; ++i) {
#pragma unroll
    for (int jj = 0; jj < 7; ++jj) {
      const int j = 6 * kHalf + jj;
      const int c = 5 * j + i - 32 * kHalf;
      if (j == kBlockWords - 1 && i == 4) continue;  // the last word's pad digit
      // levels past the half's last digit word are not needed
      if (c >= 32) continue;
      lo[jj] *= 3u;
      hi[jj] *= 3u;
      const uint32_t hn = __byte_perm(lo[jj], hi[jj], 0x7351);
      if (c >= 0) dg[c] = hn - 3u * hp[jj];
      hp[jj] = hn;
    }
  }
}

}  // namespace bitmoe
