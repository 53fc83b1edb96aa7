// Record-chunk word counts (layout version 3) and the paged-slot address
// arithmetic, shared by the quantize kernels.
#pragma once

#include "tq_internal.cuh"

namespace tqd {

// Words of one chunk for BITS and E coordinates / F QJL rows per chunk.
template <int BITS, int E, int F>
struct ChunkWords {
  static constexpr int n_idx = BITS == 1 ? (E + 31) / 32
                             : BITS == 2 ? E / 16
                             : BITS == 3 ? 3 * (E / 32) + 2 * ((E % 32) / 16)
                                         : E / 8;
  static constexpr int n_qjl = (F + 31) / 32;
  static constexpr int W = n_idx + n_qjl;
  static constexpr int q0 = n_idx;
};

// ORs the stored code of local element l (level index idx) into the chunk
// words w (shared memory; several threads may target one word).
template <int BITS, int E>
__device__ __forceinline__ void or_code_bits(uint32_t* w, int l, int idx) {
  const uint32_t code = stored_code<BITS>(idx);
  if (BITS == 3 && l / 32 < E / 32 && l % 32 >= 24) {
#pragma unroll
    for (int k = 0; k < 3; ++k)
      if ((code >> k) & 1u) atomicOr(w + code_word<BITS, E>(l, k), 1u << code_bit<BITS, E>(l, k));
  } else if (code) {
    atomicOr(w + code_word<BITS, E>(l, 0), code << code_bit<BITS, E>(l, 0));
  }
}

// Byte offset of the head block holding token `pos` of sequence b, head h,
// or -1 (and an error bit) when the position is past the block table or the
// block-table entry is out of range.
__device__ __forceinline__ int64_t head_block_offset(const tq::CacheView& cv, int64_t b, int h,
                                                     int64_t pos) {
  if (pos < 0 || pos >= cv.max_pages * cv.page_tokens) {
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
