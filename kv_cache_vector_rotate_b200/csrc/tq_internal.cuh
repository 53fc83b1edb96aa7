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

constexpr int kLayoutVersion = 1;

// Sizes of the packed record format (layout version 1).
struct Layout {
  int d, bits, m;
  int d_pad, m_pad;   // 64-multiples
  int E, F;           // coordinates / QJL rows per chunk
  int n_sign, n_mag, n_nib, n_qjl, W;   // words per chunk
  int code_bytes, norm_bytes;

  static Layout make(int d, int bits, int m) {
    Layout L{};
    L.d = d;
    L.bits = bits;
    L.m = m;
    L.d_pad = 64 * ((d + 63) / 64);
    L.m_pad = m > 0 ? 64 * ((m + 63) / 64) : 0;
    L.E = L.d_pad / 4;
    L.F = L.m_pad / 4;
    L.n_sign = bits == 4 ? 0 : (L.E + 31) / 32;
    L.n_mag = bits == 2 ? (L.E + 31) / 32 : bits == 3 ? L.E / 16 : 0;
    L.n_nib = bits == 4 ? L.E / 8 : 0;
    L.n_qjl = (L.F + 31) / 32;
    L.W = L.n_sign + L.n_mag + L.n_nib + L.n_qjl;
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
  float* srot32;      // [m_pad][d_pad] S Pi^T, zero padded        (residual sketch)
  float* bound32;     // [2^b - 1]    boundaries (fp32)
  float* cent32;      // [2^b]        float(fp16(c))
  __nv_bfloat16* pi_bf;    // tensor-core operands: [2][d_pad][d_pad] hi, lo of Pi
  __nv_bfloat16* srot_bf;  // [2][m_pad][d_pad] hi, lo of S Pi^T
  // fp16 bit patterns of the reconstruction magnitudes M[mu] = c16[H + mu]
  uint16_t mag16[8];
  uint16_t cent16[16];
};

namespace tq {

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

size_t values_workspace(const tq_codebook* cb, int64_t batch, int n_kv_heads, int n_q_heads,
                        int64_t max_ctx);
tq_status launch_values(const tq_codebook* cb, const CacheView& cv, const float* w,
                        int64_t w_stride, int64_t batch, int n_q_heads, const int32_t* ctx_len,
                        int64_t max_ctx, void* out, tq_dtype odt, int64_t out_stride, void* ws,
                        size_t ws_bytes, cudaStream_t st);

}  // namespace tq

// ---- device helpers --------------------------------------------------------

namespace tqd {

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

// Sign-word bit of local element l: word l/32, bit (l%32)/2 + 16 (l%2).
__host__ __device__ constexpr int sign_bit(int l) { return (l % 32) / 2 + 16 * (l % 2); }
// 1-bit magnitude (b = 2): word l/32, bit 8 (l%4) + (l%32)/4.
__host__ __device__ constexpr int mag1_bit(int l) { return 8 * (l % 4) + (l % 32) / 4; }
// 2-bit magnitude (b = 3): word l/16, bits p, p+1 with p = 8 (l%4) + 2 ((l%16)/4).
__host__ __device__ constexpr int mag2_bit(int l) { return 8 * (l % 4) + 2 * ((l % 16) / 4); }
// nibble (b = 4): word l/8, bits 4 ((l%8)/2 + 4 (l%2)).
__host__ __device__ constexpr int nib_bit(int l) { return 4 * ((l % 8) / 2 + 4 * (l % 2)); }

}  // namespace tqd
