// Value-side building block shared by the value pass and the fused attention
// kernel: fp16 reconstruction levels of eight packed coordinates
// ("TurboQuant explained", §Stage 1: the MSE stage codes the values).
#pragma once

#include "tq_internal.cuh"

namespace tqd {

// The MMA B operands of 32 tokens (the weights times the norms, scaled by
// 2^sc and split into fp16 hi + lo): row c = 2 q + (0: hi, 1: lo) for query
// slot q, one fp16 column per token, rows kBRow halves apart.  A fragment
// load reads word (c kBRow + tk) / 2 for c = g, tk = 2 t + const: rows of 20
// words put the 8 rows in different banks.
constexpr int kBRow = 40;

// fp16 level values of the 8 coordinates 8 kk .. 8 kk + 7 of a chunk, as four
// fp16 pairs (b <= 3: level selector and two byte permutes per 4 values; b =
// 4: sign-magnitude nibbles).  Tables: any struct with the byte-permute words
// tlo0, tlo1 (low bytes of the fp16 levels 0..7, or of the magnitudes for
// b = 4) and thi0, thi1 (high bytes).
template <int BITS, int E, class Tables>
__device__ __forceinline__ uint4 decode8(const uint32_t* cw, int kk, const Tables& p) {
  uint4 r;
  if constexpr (BITS <= 3) {
    uint32_t sel;
    if constexpr (BITS == 1) sel = (cw[kk / 4] >> (kk % 4)) & 0x11111111u;
    else if constexpr (BITS == 2) sel = (cw[kk / 2] >> (2 * (kk % 2))) & 0x33333333u;
    else {
      constexpr int full = E / 32;
      const int gg = kk / 4, j = kk % 4;
      if (gg < full) {
        sel = j < 3 ? cw[3 * gg + j] & 0x77777777u
                    : ((cw[3 * gg] >> 3) & 0x11111111u) | ((cw[3 * gg + 1] >> 2) & 0x22222222u) |
                          ((cw[3 * gg + 2] >> 1) & 0x44444444u);
      } else {
        sel = cw[3 * full + (kk - 4 * full)] & 0x77777777u;
      }
    }
    const uint32_t lo = prmt(p.tlo0, p.tlo1, sel), hi = prmt(p.thi0, p.thi1, sel);
    const uint32_t lo2 = prmt(p.tlo0, p.tlo1, sel >> 16), hi2 = prmt(p.thi0, p.thi1, sel >> 16);
    r.x = prmt(lo, hi, 0x5140u);
    r.y = prmt(lo, hi, 0x7362u);
    r.z = prmt(lo2, hi2, 0x5140u);
    r.w = prmt(lo2, hi2, 0x7362u);
  } else {
    // word kk: nibble a holds element 2a, nibble a + 4 element 2a + 1 (a < 4)
    const uint32_t x = cw[kk];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const uint32_t y = x >> (8 * half);           // elements 4 half .. 4 half + 3
      const uint32_t sel = (y & 0x77u) | ((y >> 8) & 0x7700u);
      const uint32_t lo = prmt(p.tlo0, p.tlo1, sel), hi = prmt(p.thi0, p.thi1, sel);
      const uint32_t h0 = prmt(lo, hi, 0x6240u) | ((y << 12) & 0x80008000u);
      const uint32_t h1 = prmt(lo, hi, 0x7351u) | ((y << 8) & 0x80008000u);
      if (half == 0) { r.x = h0; r.y = h1; } else { r.z = h0; r.w = h1; }
    }
  }
  return r;
}

}  // namespace tqd
