// Internal declarations shared by the libtq kernels and the C-ABI layer.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <string>
#include <vector>

#include "../../include/tq.h"

namespace tq {

constexpr int kLayoutVersion = 3;

// Sizes of the packed record format (layout version 3).
struct Layout {
  int d, bits, m;
  int d_pad, m_pad;   // 64-multiples
  int E, F;           // coordinates / QJL rows per chunk
  int n_idx, n_qjl, W;   // words per chunk
  int code_bytes, norm_bytes;

  static int index_words(int bits, int E) {
    switch (bits) {
      case 1: return (E + 31) / 32;
      case 2: return E / 16;
      case 3: return 3 * (E / 32) + 2 * ((E % 32) / 16);
      default: return E / 8;
    }
  }
  static Layout make(int d, int bits, int m) {
    Layout L{};
    L.d = d;
    L.bits = bits;
    L.m = m;
    L.d_pad = 64 * ((d + 63) / 64);
    L.m_pad = m > 0 ? 64 * ((m + 63) / 64) : 0;
    L.E = L.d_pad / 4;
    L.F = L.m_pad / 4;
    L.n_idx = index_words(bits, L.E);
    L.n_qjl = (L.F + 31) / 32;
    L.W = L.n_idx + L.n_qjl;
    L.code_bytes = 16 * L.W;
    L.norm_bytes = m > 0 ? 4 : 2;
    return L;
  }
  int64_t head_block_bytes(int page_tokens) const {
    int64_t raw = (int64_t)page_tokens * (code_bytes + norm_bytes);
    return 16 * ((raw + 15) / 16);
  }
};

}  // namespace tq

// Opaque handle of the C ABI.
struct tq_codebook {
  tq::Layout lay;
  uint64_t seed_pi, seed_s;
  int device;
  // float64 host tables
  std::vector<double> pi, s, centroids, boundaries;
  double s_row_norm_max;        // max_i ||S_i|| (bounds |(S q)_i| <= this * ||q||)
  double qjl_scale;             // sqrt(pi/2) / m
  // device tables (one allocation, `dev_block`)
  void* dev_block;
  float* pi32;        // [d_pad][d]   Pi, rows >= d zero         (query rotation, v0 quantize)
  float* s32;         // [m_pad][d]   S, rows >= m zero           (query sketch)
  float* srott32;     // [d_pad][m_pad] (S Pi^T)^T, zero padded    (residual sketch, coalesced)
  float* pit32;       // [d][d_pad]   Pi^T, columns >= d zero     (query rotation, coalesced)
  float* st32;        // [d][m_pad]   S^T, columns >= m zero      (query sketch, coalesced)
  float* srot32;      // [m_pad][d_pad] S Pi^T row-major, zero padded (residual sketch, small appends)
  float* bound32;     // [2^b - 1]    boundaries (fp32)
  float* cent32;      // [2^b]        the reconstruction levels (fp32, exact)
  __nv_bfloat16* pi_bf;    // tensor-core operands: [2][d_pad][d_pad] hi, lo of Pi
  __nv_bfloat16* srot_bf;  // [2][m_pad][d_pad] hi, lo of S Pi^T
  // [Pi ; S] (R = d_pad + m_pad rows, d columns padded to d16 = ceil(d/16)
  // blocks of 16) as bf16 hi + lo in mma.m16n8k16 A-fragment order:
  // uint4 [R/16 row tiles][d16][2: hi, lo][32 lanes]
  uint4* qprep_frag;
  // reconstruction levels (float64 copies of what the kernels use): 8-bit
  // fixed point levels k_i 2^-table_exp for b <= 3, fp16 levels for b = 4
  std::vector<double> levels;
  // fp16 bit patterns of the levels (exact) and of the magnitudes
  // M[mu] = level[H + mu]
  uint16_t mag16[8];
  uint16_t cent16[16];
  // b <= 3: the integers k_i of levels 0..7 as int8 bytes (int8_levels[0] =
  // levels 0..3)
  int table_exp;
  uint32_t int8_levels[2];
};

namespace tq {

// The current device and its SM count (cached per device).
int current_device();
int device_sm_count();

// A flag per device (up to 64) for per-device set-up such as kernel
// attributes: need(dev) until mark(dev) (setting an attribute twice is harmless).
struct PerDeviceOnce {
  unsigned long long done = 0;
  bool need(int dev) const { return dev < 0 || dev >= 64 || !(done & (1ull << dev)); }
  void mark(int dev) {
    if (dev >= 0 && dev < 64) done |= 1ull << dev;
  }
};

// Error reporting (thread-local message for tq_last_error).
void set_error(const std::string& msg);
tq_status fail(tq_status st, const std::string& msg);
tq_status cuda_fail(cudaError_t e, const char* what);

// ---- kernel launchers (defined in the .cu files) --------------------------

struct CacheView {
  uint8_t* pages;
  int64_t n_pages;
  int page_tokens;
  int n_kv_heads;
  const int32_t* block_table;
  int64_t max_pages;
  uint32_t* err;
  int64_t head_block_bytes;
  int64_t page_bytes;
};

size_t logits_workspace(const tq_codebook* cb, int64_t groups, int G);
tq_status launch_logits(const tq_codebook* cb, const CacheView& cv, const void* q, tq_dtype dt,
                        int64_t batch, int n_q_heads, const int32_t* ctx_len, int64_t max_ctx,
                        float* out, int64_t out_stride, void* ws, size_t ws_bytes,
                        cudaStream_t st);

// The preparation kernel alone (query fragments for d <= 128, as the logits
// kernel reads them), a programmatic dependent of the previous kernel.
struct PreparedQueries {
  const uint2* frag;
  const uint2* qfrag;
  const float2* scal;
};
size_t query_prep_workspace(const tq_codebook* cb, int64_t batch, int n_kv_heads, int n_q_heads);
tq_status launch_query_prep(const tq_codebook* cb, const void* q, tq_dtype dt, int64_t batch, int n_kv_heads,
                            int n_q_heads, void* ws, PreparedQueries* pq, cudaStream_t st);

size_t search_workspace(const tq_codebook* cb, int64_t batch, int n_kv_heads, int n_q_heads, int64_t max_ctx,
                        int k);
tq_status launch_search(const tq_codebook* cb, const CacheView& cv, const void* q, tq_dtype dt, int64_t batch,
                        int n_q_heads, const int32_t* ctx_len, int64_t max_ctx, int k, float* out_score,
                        int32_t* out_idx, void* ws, size_t ws_bytes, cudaStream_t st);

tq_status polar_build(int d, int bits, int m, uint64_t seed_pi, uint64_t seed_s, tq_polar** out);
void polar_free(tq_polar* P);
tq_status polar_encode(const tq_polar* P, const void* x, tq_dtype dt, int64_t n, void* rec, uint32_t* err,
                       cudaStream_t st);
size_t polar_logits_workspace(const tq_polar* P, int nq);
tq_status polar_logits(const tq_polar* P, const void* rec, int64_t n, const void* q, tq_dtype dt, int nq, float* out,
                       int64_t out_stride, void* ws, size_t ws_bytes, cudaStream_t st);
int polar_record_bytes(const tq_polar* P);

size_t attend_workspace(const tq_codebook* kcb, const tq_codebook* vcb, int64_t batch, int n_kv_heads,
                        int n_q_heads, int64_t max_ctx);
tq_status launch_attend(const tq_codebook* kcb, const CacheView& kcv, const tq_codebook* vcb, const CacheView& vcv,
                        const void* q, tq_dtype dt, int64_t batch, int n_q_heads, const int32_t* ctx_len,
                        int64_t max_ctx, float scale, float* out, void* ws, size_t ws_bytes, cudaStream_t st);

size_t values_workspace(const tq_codebook* cb, int64_t batch, int n_kv_heads, int n_q_heads,
                        int64_t max_ctx);
tq_status launch_values(const tq_codebook* cb, const CacheView& cv, const float* w,
                        int64_t w_stride, int64_t batch, int n_q_heads, const int32_t* ctx_len,
                        int64_t max_ctx, void* out, tq_dtype odt, int64_t out_stride, void* ws,
                        size_t ws_bytes, cudaStream_t st);

}  // namespace tq

// ---- device helpers --------------------------------------------------------

namespace tqd {

// Division of 0 <= n < 2^31 by a divisor fixed at launch, without the
// software division routine: q = (umulhi(n, m) + n) >> s with
// m = floor(2^32 (2^s - d) / d) + 1, s = ceil(log2 d) (round-up reciprocal;
// exact for these n), or q = n when d = 1.
struct FastDiv {
  uint32_t d, m, s;
};
inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f{d, 0u, 0u};
  if (d > 1) {
    uint32_t l = 0;
    while ((1ull << l) < d) ++l;
    f.m = (uint32_t)((((uint64_t)1 << 32) * ((1ull << l) - d)) / d + 1);
    f.s = l;
  }
  return f;
}
__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return f.d == 1 ? n : (__umulhi(n, f.m) + n) >> f.s;
}

__device__ __forceinline__ void report(uint32_t* err, uint32_t bits) {
  if (err) atomicOr(err, bits);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ float load_elem(const void* p, int64_t i, tq_dtype dt) {
  if (dt == TQ_F32) return __ldg(reinterpret_cast<const float*>(p) + i);
  if (dt == TQ_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  return __half2float(reinterpret_cast<const __half*>(p)[i]);
}

// Layout version 3.  Bit k of the stored code of local element l of a chunk
// lives at index word code_word(l, k), bit code_bit(l, k).  The stored code is
// the level index for b <= 3 and the sign-magnitude nibble neg << 3 | mu for
// b = 4.  The b <= 3 positions make eight codes a byte-permute selector after
// one mask (b = 1: >> (l%32)/8 & 0x11111111; b = 2: >> 2((l%16)/8) &
// 0x33333333; b = 3: & 0x77777777, the last 8 of each group of 32 from the
// top bits of the group's three words).
template <int BITS, int E>
__host__ __device__ constexpr int code_word(int l, int k) {
  if (BITS == 1) return l / 32;
  if (BITS == 2) return l / 16;
  if (BITS == 3) {
    const int g = l / 32, lp = l % 32;
    if (g < E / 32) return lp < 24 ? 3 * g + lp / 8 : 3 * g + k;
    return 3 * (E / 32) + lp / 8;
  }
  return l / 8;
}
template <int BITS, int E>
__host__ __device__ constexpr int code_bit(int l, int k) {
  if (BITS == 1) return 4 * (l % 8) + (l % 32) / 8;
  if (BITS == 2) return 4 * (l % 8) + 2 * ((l % 16) / 8) + k;
  if (BITS == 3) {
    const int g = l / 32, lp = l % 32;
    if (g < E / 32 && lp >= 24) return 4 * (lp - 24) + 3;
    return 4 * (lp % 8) + k;
  }
  return 4 * ((l % 8) / 2 + 4 * (l % 2)) + k;
}
// Stored code of level index idx (b = 4: sign-magnitude nibble, H = 8).
template <int BITS>
__host__ __device__ constexpr uint32_t stored_code(int idx) {
  if (BITS < 4) return (uint32_t)idx;
  return idx < 8 ? (8u | (uint32_t)(7 - idx)) : (uint32_t)(idx - 8);
}
template <int BITS>
__host__ __device__ constexpr int level_index(uint32_t code) {
  if (BITS < 4) return (int)code;
  return (code & 8u) ? 7 - (int)(code & 7u) : 8 + (int)(code & 7u);
}
// QJL-word bit of local row l: word l/32, bit 8 (l%4) + (l%32)/4.
__host__ __device__ constexpr int qjl_bit(int l) { return 8 * (l % 4) + (l % 32) / 4; }

}  // namespace tqd
