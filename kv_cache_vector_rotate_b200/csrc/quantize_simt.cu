// Quantize-and-append on CUDA cores (fp32 projections).
//
// "TurboQuant explained" (a2a-mcp.org) §Stage 1: normalize, rotate by Pi,
// map each rotated coordinate to its Lloyd-Max cell; §Stage 2: signs of a
// Gaussian projection of the residual; §How to implement: quantize on every
// cache update.  This kernel is the plain variant used for small appends (a
// decode step's few new tokens) and for shapes the tensor-core kernel does not
// cover; it writes exactly the same records.
//
// One CTA handles TOK vectors (32, or 16 for d_pad > 128) with 4 threads per
// vector; thread (token, chunk) computes the E rotated coordinates and F
// projections of its chunk and packs them.

#include "pack.cuh"

namespace tqd {

struct QuantizeSimtParams {
  const void* x;
  tq_dtype dtype;
  int64_t rows;        // batch * n_kv_heads * n_new
  int64_t n_new;
  int n_kv_heads;
  int d;
  const int32_t* start_pos;
  tq::CacheView cv;
  const float* pi32;   // [d_pad][d]
  const float* srot32; // [m_pad][d_pad]
  const float* bound32;
  const float* cent32;
};

template <int E>
struct SimtTile {
  static constexpr int TOK = E <= 32 ? 32 : 16;
  static constexpr int THREADS = 4 * TOK;
};

template <int BITS, int E, int F>
__global__ void __launch_bounds__(SimtTile<E>::THREADS) quantize_simt_kernel(QuantizeSimtParams p) {
  constexpr int DP = 4 * E;
  constexpr int K = 1 << BITS;
  constexpr int TOK = SimtTile<E>::TOK;
  constexpr int NT = SimtTile<E>::THREADS;
  using CW = ChunkWords<BITS, E, F>;
  __shared__ float xs[TOK][DP + 1];
  __shared__ float rs[TOK][DP + 1];
  __shared__ float sb[K];
  __shared__ float sc[K];

  const int tid = threadIdx.x;
  const int tok = tid >> 2;     // 0..TOK-1
  const int t = tid & 3;        // chunk
  const int64_t row0 = (int64_t)blockIdx.x * TOK;
  const int d = p.d;

  if (tid < K) {
    sb[tid] = tid == 0 ? 0.0f : p.bound32[tid - 1];
    sc[tid] = p.cent32[tid];
  }
  for (int i = tid; i < TOK * DP; i += NT) {
    const int r = i / DP, k = i % DP;
    const int64_t row = row0 + r;
    xs[r][k] = (row < p.rows && k < d) ? load_elem(p.x, row * d + k, p.dtype) : 0.0f;
  }
  __syncthreads();

  const int64_t row = row0 + tok;
  const bool valid = row < p.rows;

  // ||x|| in fp32 from the input: each of the 4 chunk threads sums a quarter.
  float n2 = 0.0f;
  for (int k = t; k < d; k += 4) n2 = fmaf(xs[tok][k], xs[tok][k], n2);
  n2 += __shfl_xor_sync(0xffffffffu, n2, 1);
  n2 += __shfl_xor_sync(0xffffffffu, n2, 2);
  const float norm = sqrtf(n2);
  const float inv = norm > 0.0f ? 1.0f / norm : 0.0f;

  uint32_t w[CW::W];
#pragma unroll
  for (int i = 0; i < CW::W; ++i) w[i] = 0u;

  float r2 = 0.0f;
#pragma unroll
  for (int l = 0; l < E; ++l) {
    const int j = t * E + l;
    float u = 0.0f;
    if (j < d) {
      const float* pr = p.pi32 + (size_t)j * d;
      float y = 0.0f;
      for (int k = 0; k < d; ++k) y = fmaf(__ldg(pr + k), xs[tok][k], y);
      u = y * inv;
    }
    // threshold search: the largest idx with boundary t_idx <= u
    int idx = 0;
#pragma unroll
    for (int step = K / 2; step >= 1; step >>= 1)
      if (u >= sb[idx + step]) idx += step;
    pack_index<BITS, E, F>(w, l, idx);
    const float res = j < d ? u - sc[idx] : 0.0f;
    rs[tok][j] = res;
    r2 = fmaf(res, res, r2);
  }
  r2 += __shfl_xor_sync(0xffffffffu, r2, 1);
  r2 += __shfl_xor_sync(0xffffffffu, r2, 2);

  if constexpr (F > 0) {
    __syncthreads();
#pragma unroll
    for (int l = 0; l < F; ++l) {
      const int i = t * F + l;
      const float* ps = p.srot32 + (size_t)i * DP;
      float proj = 0.0f;
      for (int j = 0; j < DP; ++j) proj = fmaf(__ldg(ps + j), rs[tok][j], proj);
      pack_qjl<BITS, E, F>(w, l, proj < 0.0f);
    }
  }
  if (!valid) return;

  const int64_t per_seq = (int64_t)p.n_kv_heads * p.n_new;
  const int64_t b = row / per_seq;
  const int h = (int)((row / p.n_new) % p.n_kv_heads);
  const int64_t pos = p.start_pos[b] + row % p.n_new;
  const int64_t hb = head_block_offset(p.cv, b, h, pos);
  if (hb < 0) return;
  const int slot = (int)(pos % p.cv.page_tokens);
  uint32_t* rec = reinterpret_cast<uint32_t*>(p.cv.pages + hb + (int64_t)slot * 16 * CW::W) + t * CW::W;
#pragma unroll
  for (int i = 0; i < CW::W; ++i) rec[i] = w[i];
  if (t == 0) {
    const __half nh = __float2half_rn(norm);
    if (__hisinf(nh)) report(p.cv.err, TQ_DEV_ERR_RANGE);
    __half* nslot = reinterpret_cast<__half*>(p.cv.pages + hb + (int64_t)p.cv.page_tokens * 16 * CW::W +
                                              (int64_t)slot * (F > 0 ? 4 : 2));
    nslot[0] = nh;
    if constexpr (F > 0) nslot[1] = __float2half_rn(sqrtf(r2));
  }
}

}  // namespace tqd

namespace tq {

template <int BITS, int E, int F>
static void launch_simt(const tqd::QuantizeSimtParams& p, cudaStream_t st) {
  constexpr int TOK = tqd::SimtTile<E>::TOK;
  const unsigned blocks = (unsigned)((p.rows + TOK - 1) / TOK);
  tqd::quantize_simt_kernel<BITS, E, F><<<blocks, tqd::SimtTile<E>::THREADS, 0, st>>>(p);
}

template <int BITS>
static bool dispatch_simt_e(const Layout& L, const tqd::QuantizeSimtParams& p, cudaStream_t st) {
  if (L.E == 32 && L.F == 32) return launch_simt<BITS, 32, 32>(p, st), true;
  if (L.E == 32 && L.F == 0) return launch_simt<BITS, 32, 0>(p, st), true;
  if (L.E == 16 && L.F == 16) return launch_simt<BITS, 16, 16>(p, st), true;
  if (L.E == 16 && L.F == 0) return launch_simt<BITS, 16, 0>(p, st), true;
  if (L.E == 64 && L.F == 64) return launch_simt<BITS, 64, 64>(p, st), true;
  if (L.E == 64 && L.F == 0) return launch_simt<BITS, 64, 0>(p, st), true;
  if (L.E == 48 && L.F == 48) return launch_simt<BITS, 48, 48>(p, st), true;
  if (L.E == 48 && L.F == 0) return launch_simt<BITS, 48, 0>(p, st), true;
  return false;
}

tq_status launch_quantize_simt(const tq_codebook* cb, const void* x, tq_dtype dt, int64_t batch,
                               int n_kv_heads, int64_t n_new, const int32_t* start_pos,
                               const CacheView& cv, cudaStream_t st) {
  tqd::QuantizeSimtParams p;
  p.x = x;
  p.dtype = dt;
  p.rows = batch * n_kv_heads * n_new;
  p.n_new = n_new;
  p.n_kv_heads = n_kv_heads;
  p.d = cb->lay.d;
  p.start_pos = start_pos;
  p.cv = cv;
  p.pi32 = cb->pi32;
  p.srot32 = cb->srot32;
  p.bound32 = cb->bound32;
  p.cent32 = cb->cent32;
  bool ok = false;
  switch (cb->lay.bits) {
    case 1: ok = dispatch_simt_e<1>(cb->lay, p, st); break;
    case 2: ok = dispatch_simt_e<2>(cb->lay, p, st); break;
    case 3: ok = dispatch_simt_e<3>(cb->lay, p, st); break;
    case 4: ok = dispatch_simt_e<4>(cb->lay, p, st); break;
  }
  if (!ok) return fail(TQ_EUNSUPPORTED, "quantize: no kernel for this (d, m)");
  return cuda_fail(cudaGetLastError(), "quantize_simt launch");
}

}  // namespace tq
