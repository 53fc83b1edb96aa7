// Packing of one chunk of a record (layout version 1) and the paged-slot
// address arithmetic, shared by the quantize kernels.
#pragma once

#include "tq_internal.cuh"

namespace tqd {

// Words of one chunk for BITS and E coordinates / F QJL rows per chunk.
template <int BITS, int E, int F>
struct ChunkWords {
  static constexpr int n_sign = BITS == 4 ? 0 : (E + 31) / 32;
  static constexpr int n_mag = BITS == 2 ? (E + 31) / 32 : BITS == 3 ? E / 16 : 0;
  static constexpr int n_nib = BITS == 4 ? E / 8 : 0;
  static constexpr int n_qjl = (F + 31) / 32;
  static constexpr int W = n_sign + n_mag + n_nib + n_qjl;
  static constexpr int q0 = n_sign + n_mag + n_nib;
};

// Adds element l with level index idx to the chunk words.  Callers unroll
// their element loops so that l, and every shift below, is a constant.
template <int BITS, int E, int F>
__device__ __forceinline__ void pack_index(uint32_t* w, int l, int idx) {
  using CW = ChunkWords<BITS, E, F>;
  constexpr int H = 1 << (BITS - 1);
  const uint32_t neg = idx < H ? 1u : 0u;
  const uint32_t mu = neg ? (uint32_t)(H - 1 - idx) : (uint32_t)(idx - H);
  if constexpr (BITS == 4) {
    w[l / 8] |= ((neg << 3) | mu) << nib_bit(l);
  } else {
    w[l / 32] |= neg << sign_bit(l);
    if constexpr (BITS == 2) w[CW::n_sign + l / 32] |= mu << mag1_bit(l);
    if constexpr (BITS == 3) w[CW::n_sign + l / 16] |= mu << mag2_bit(l);
  }
}

template <int BITS, int E, int F>
__device__ __forceinline__ void pack_qjl(uint32_t* w, int l, bool negative) {
  using CW = ChunkWords<BITS, E, F>;
  w[CW::q0 + l / 32] |= (negative ? 1u : 0u) << sign_bit(l);
}

// Byte offset of the head block holding token `pos` of sequence b, head h,
// or -1 (and an error bit) when the block-table entry is out of range.
__device__ __forceinline__ int64_t head_block_offset(const tq::CacheView& cv, int64_t b, int h,
                                                     int64_t pos) {
  if (pos < 0 || pos >= cv.max_pages * cv.page_tokens) {   // past the block table
    report(cv.err, TQ_DEV_ERR_PAGE);
    return -1;
  }
  const int64_t page = cv.block_table[b * cv.max_pages + pos / cv.page_tokens];
  if (page < 0 || page >= cv.n_pages) {
    report(cv.err, TQ_DEV_ERR_PAGE);
    return -1;
  }
  return page * cv.page_bytes + (int64_t)h * cv.head_block_bytes;
}

}  // namespace tqd
