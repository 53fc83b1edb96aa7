// The recursive polar form of stage 1 on the GPU: encode and logits.
//
// "TurboQuant explained" (a2a-mcp.org), §Stage 1, its PolarQuant paragraph:
// the normalized vector is rotated, its coordinates are paired recursively
// and every pair is turned into polar form; the angles' laws are known in
// advance, so they are quantized with fixed codebooks and no per-block scale
// is stored.  Readings (as the oracle's): the transform acts on u = Pi x /
// ||x|| (d a power of two); level 1 takes atan2(u[2i+1], u[2i]) in [-pi, pi],
// level l > 1 atan2(rho[2i+1], rho[2i]) in [0, pi/2] of the previous level's
// radii; each of the d - 1 angles gets b bits from the Lloyd-Max quantizer
// of its level's law (a tie to the upper cell); ||x|| is the fp16 side
// value; with a sketch (m > 0) the residual r = u - Pi^T u_hat (original
// space) keeps the signs of S r and fp16 ||r|| (§Stage 2).
//
// Record (one per vector, a multiple of 16 bytes): CW = ceil((d - 1) b / 32)
// code words -- angle a (level 1 first, then by index within the level) at
// bits a b .. a b + b - 1 of the little-endian word stream -- then m / 32
// sign words (bit i set where (S r)_i < 0), then one word holding fp16 ||x||
// (low half) and fp16 ||r|| (high half).
//
// The logit needs no reconstructed vector: with q~ = Pi q the pairs fold
// bottom-up, s_i = q~[2i] cos th_i + q~[2i+1] sin th_i at level 1, then
// s_i <- s_2i cos ph_i + s_2i+1 sin ph_i per level; the last s is
// <q~, u_hat>, and L = ||x|| (s + sqrt(pi/2)/m ||r|| <S q, sign>).  That is
// 2 (d - 1) FMAs per key and query, so this path is bound by the FMA pipe,
// not by HBM.  The cos and sin of the centroids come from per-level tables
// in shared memory, indexed by the angle's code read from the key's code
// words in registers; the fold is a compile-time tree over 4 queries at
// once, so its partial sums stay in registers.

#include <algorithm>
#include <cmath>
#include <vector>

#include "codebook_host.h"
#include "tq_internal.cuh"

struct tq_polar {
  int d, bits, m, levels;
  int code_words, sign_words, rec_words;
  uint64_t seed_pi, seed_s;
  int device;
  std::vector<double> pi, s;             // host float64 (row-major d x d, m x d)
  std::vector<tqhost::LloydMax> books;   // level 1 first
  void* dev_block;
  float* pit32;    // [d][d]  Pi^T: (k, j) = Pi[j][k]
  float* pi32;     // [d][d]  Pi row-major
  float* st32;     // [d][m]  S^T
  float* tabs;     // [levels][4][16]: cos c, sin c, c, boundaries (2^b - 1 used)
  double qjl_scale;
};

namespace tqd {

constexpr int kPolVec = 32;        // vectors per encode CTA
constexpr int kPolThreads = 256;
constexpr int kPolLogThreads = 128;
constexpr int kPolQPass = 4;       // queries per pass of a logits thread
constexpr int kPolQBlock = 64;     // queries per logits CTA

struct PolarParams {
  int d, bits, m, levels;
  int code_words, sign_words, rec_words;   // rec_words: 32-bit words per record
  const float* pit32;
  const float* pi32;
  const float* st32;
  const float* tabs;
  float qjl_scale;
  // encode
  const void* x;
  tq_dtype dtype;
  int64_t n;
  uint32_t* rec;
  // logits
  const uint32_t* crec;
  const void* q;
  int nq;
  float* qrot;     // [nq][d + m]: Pi q, then S q (workspace)
  float* out;      // [nq][n]
  int64_t out_stride;
  uint32_t* err;
};

// First angle of level l (level l has d / 2^l angles).
__host__ __device__ constexpr int level_offset(int d, int l) { return d - (d >> (l - 1)); }

// The b-bit field at bit `bit` of a little-endian word stream (one funnel shift).
__device__ __forceinline__ uint32_t get_field(const uint32_t* w, int bit, int b) {
  return __funnelshift_r(w[bit >> 5], w[(bit >> 5) + 1], bit & 31) & ((1u << b) - 1u);
}

// ---- encode: one CTA of 256 threads per 32 vectors ----------------------------------
// Shared memory (dynamic): the vectors' working rows, then indices and words.
template <int D>
struct PolarEncSmem {
  float us[kPolVec][D];          // u = x / ||x|| (original space)
  float ys[kPolVec][D];          // Pi u, then the radii of the level being done
  float rs[kPolVec][D];          // radii of the next level; u_hat; then r
  float rt[kPolVec][D / 2];      // ping-pong buffer of the inverse recursion
  uint32_t cw[kPolVec][33];      // code words (<= 32) + 1 spare
  uint32_t sw[kPolVec][8];       // sign words (m <= 256)
  float nrm[kPolVec], rnrm[kPolVec];
  float tb[8][4][16];
  uint8_t ix[kPolVec][D];        // angle indices
};

template <int D>
__global__ void __launch_bounds__(kPolThreads) polar_encode_kernel(PolarParams p) {
  constexpr int L = D == 64 ? 6 : D == 128 ? 7 : 8;
  extern __shared__ __align__(16) uint8_t pol_enc_smem[];
  auto& sm = *reinterpret_cast<PolarEncSmem<D>*>(pol_enc_smem);
  auto& us = sm.us;
  auto& ys = sm.ys;
  auto& rs = sm.rs;
  auto& rt = sm.rt;
  auto& ix = sm.ix;
  auto& cw = sm.cw;
  auto& sw = sm.sw;
  auto& nrm = sm.nrm;
  auto& rnrm = sm.rnrm;
  auto& tb = sm.tb;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t v0 = (int64_t)blockIdx.x * kPolVec;
  const int nv = (int)min((int64_t)kPolVec, p.n - v0);
  const int B = p.bits, NB = (1 << B) - 1, M = p.m;
  for (int i = tid; i < L * 64; i += kPolThreads) (&tb[0][0][0])[i] = p.tabs[i];
  for (int i = tid; i < kPolVec * 33; i += kPolThreads) (&cw[0][0])[i] = 0u;
  for (int i = tid; i < kPolVec * 8; i += kPolThreads) (&sw[0][0])[i] = 0u;
  for (int i = tid; i < kPolVec * D; i += kPolThreads) {
    const int v = i / D, k = i % D;
    us[v][k] = v < nv ? load_elem(p.x, (v0 + v) * D + k, p.dtype) : 0.0f;
  }
  __syncthreads();
  // ||x|| (warp v)
  for (int v = warp; v < kPolVec; v += kPolThreads / 32) {
    float s2 = 0.0f;
    for (int k = lane; k < D; k += 32) s2 = fmaf(us[v][k], us[v][k], s2);
#pragma unroll
    for (int o = 16; o; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    if (lane == 0) nrm[v] = sqrtf(s2);
  }
  __syncthreads();
  for (int i = tid; i < kPolVec * D; i += kPolThreads) {
    const int v = i / D, k = i % D;
    us[v][k] = nrm[v] > 0.0f ? us[v][k] / nrm[v] : 0.0f;   // the zero vector stays zero
  }
  __syncthreads();
  // y = Pi u: thread j = tid % D for the vectors g, g + VG, ...
  {
    constexpr int VG = kPolThreads / D;              // 4, 2, 1
    constexpr int VPT = kPolVec / VG;                // vectors per thread
    const int j = tid % D, g = tid / D;
    float acc[VPT];
#pragma unroll
    for (int a = 0; a < VPT; ++a) acc[a] = 0.0f;
    for (int k = 0; k < D; k += 4) {          // 4 coordinates per 16-byte shared load
      float pk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) pk[e] = __ldg(p.pit32 + (size_t)(k + e) * D + j);   // Pi[j][k + e]
#pragma unroll
      for (int a = 0; a < VPT; ++a) {
        const float4 u4 = *reinterpret_cast<const float4*>(&us[g + VG * a][k]);
        acc[a] = fmaf(pk[0], u4.x, acc[a]);
        acc[a] = fmaf(pk[1], u4.y, acc[a]);
        acc[a] = fmaf(pk[2], u4.z, acc[a]);
        acc[a] = fmaf(pk[3], u4.w, acc[a]);
      }
    }
#pragma unroll
    for (int a = 0; a < VPT; ++a) ys[g + VG * a][j] = acc[a];
  }
  __syncthreads();
  // the recursion, level by level: angles quantized, radii passed on
#pragma unroll 1
  for (int l = 1; l <= L; ++l) {
    const int half = D >> l, off = level_offset(D, l);
    const float* bnd = tb[l - 1][3];
    for (int i = tid; i < kPolVec * half; i += kPolThreads) {
      const int v = i / half, a = i % half;
      const float x0 = ys[v][2 * a], x1 = ys[v][2 * a + 1];
      const float phi = atan2f(x1, x0);
      int idx = 0;
      for (int t = 0; t < NB; ++t) idx += phi >= bnd[t] ? 1 : 0;   // ties go up
      ix[v][off + a] = (uint8_t)idx;
      const int bit = (off + a) * B;
      atomicOr(&cw[v][bit >> 5], (uint32_t)idx << (bit & 31));
      if ((bit & 31) + B > 32) atomicOr(&cw[v][(bit >> 5) + 1], (uint32_t)idx >> (32 - (bit & 31)));
      rs[v][a] = sqrtf(fmaf(x0, x0, x1 * x1));
    }
    __syncthreads();
    for (int i = tid; i < kPolVec * half; i += kPolThreads) ys[i / half][i % half] = rs[i / half][i % half];
    __syncthreads();
  }
  if (M > 0) {
    // u_hat: the recursion backwards from radius 1 with the centroids; the
    // level-l radii alternate between rt and ys, level 1 writes rs
    for (int v = tid; v < kPolVec; v += kPolThreads) rt[v][0] = 1.0f;
    __syncthreads();
    bool in_rt = true;
#pragma unroll 1
    for (int l = L; l >= 1; --l) {
      const int cnt = D >> l, off = level_offset(D, l);
      for (int i = tid; i < kPolVec * cnt; i += kPolThreads) {
        const int v = i / cnt, a = i % cnt;
        const float r0 = in_rt ? rt[v][a] : ys[v][a];
        const int idx = ix[v][off + a];
        const float c = tb[l - 1][0][idx], s = tb[l - 1][1][idx];
        float* dst = l == 1 ? rs[v] : (in_rt ? ys[v] : rt[v]);
        dst[2 * a] = r0 * c;
        dst[2 * a + 1] = r0 * s;
      }
      __syncthreads();
      in_rt = !in_rt;
    }
    // r = u - Pi^T u_hat (original space), into ys
    {
      constexpr int VG = kPolThreads / D;
      constexpr int VPT = kPolVec / VG;
      const int k = tid % D, g = tid / D;
      float acc[VPT];
#pragma unroll
      for (int a = 0; a < VPT; ++a) acc[a] = 0.0f;
      for (int j = 0; j < D; j += 4) {
        float pjk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) pjk[e] = __ldg(p.pi32 + (size_t)(j + e) * D + k);   // Pi[j + e][k]
#pragma unroll
        for (int a = 0; a < VPT; ++a) {
          const float4 r4 = *reinterpret_cast<const float4*>(&rs[g + VG * a][j]);
          acc[a] = fmaf(pjk[0], r4.x, acc[a]);
          acc[a] = fmaf(pjk[1], r4.y, acc[a]);
          acc[a] = fmaf(pjk[2], r4.z, acc[a]);
          acc[a] = fmaf(pjk[3], r4.w, acc[a]);
        }
      }
#pragma unroll
      for (int a = 0; a < VPT; ++a) ys[g + VG * a][k] = us[g + VG * a][k] - acc[a];
    }
    __syncthreads();
    for (int v = warp; v < kPolVec; v += kPolThreads / 32) {
      float s2 = 0.0f;
      for (int k = lane; k < D; k += 32) s2 = fmaf(ys[v][k], ys[v][k], s2);
#pragma unroll
      for (int o = 16; o; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
      if (lane == 0) rnrm[v] = sqrtf(s2);
    }
    // the signs of S r: thread (row i, 8 vectors), each S^T entry loaded once
    // per 8 vectors; a warp's 32 consecutive rows make one sign word (ballot)
    constexpr int VB8 = kPolVec / 8;
    for (int t = tid; t < M * VB8; t += kPolThreads) {
      const int i = t % M, v8 = 8 * (t / M);
      float pr[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) pr[a] = 0.0f;
      for (int k = 0; k < D; k += 4) {
        float sk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) sk[e] = __ldg(p.st32 + (size_t)(k + e) * M + i);
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          const float4 y4 = *reinterpret_cast<const float4*>(&ys[v8 + a][k]);
          pr[a] = fmaf(sk[0], y4.x, pr[a]);
          pr[a] = fmaf(sk[1], y4.y, pr[a]);
          pr[a] = fmaf(sk[2], y4.z, pr[a]);
          pr[a] = fmaf(sk[3], y4.w, pr[a]);
        }
      }
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const uint32_t word = __ballot_sync(0xffffffffu, pr[a] < 0.0f);
        if ((i & 31) == 0) sw[v8 + a][i >> 5] = word;
      }
    }
  }
  __syncthreads();
  // the records
  const int CW = p.code_words, SW = p.sign_words, RW = p.rec_words;
  for (int t = tid; t < nv * RW; t += kPolThreads) {
    const int v = t / RW, w = t % RW;
    uint32_t val = 0u;
    if (w < CW) {
      val = cw[v][w];
    } else if (w < CW + SW) {
      val = sw[v][w - CW];
    } else if (w == CW + SW) {
      const __half hn = __float2half_rn(nrm[v]);
      if (__hisinf(hn)) report(p.err, TQ_DEV_ERR_RANGE);
      val = (uint32_t)__half_as_ushort(hn) | ((uint32_t)__half_as_ushort(__float2half_rn(M > 0 ? rnrm[v] : 0.0f)) << 16);
    }
    p.rec[(v0 + v) * RW + w] = val;
  }
}

// ---- query preparation: Pi q and S q in fp32, one CTA (128 threads) per query -------
template <int D>
__global__ void __launch_bounds__(128) polar_prep_kernel(PolarParams p) {
  __shared__ float qs[D];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  const int qi = blockIdx.x;
  for (int k = threadIdx.x; k < D; k += 128) qs[k] = load_elem(p.q, (int64_t)qi * D + k, p.dtype);
  __syncthreads();
  float* dst = p.qrot + (int64_t)qi * (D + p.m);
  for (int j = threadIdx.x; j < D; j += 128) {
    float a = 0.0f;
    for (int k = 0; k < D; ++k) a = fmaf(__ldg(p.pit32 + (size_t)k * D + j), qs[k], a);
    dst[j] = a;
  }
  for (int i = threadIdx.x; i < p.m; i += 128) {
    float a = 0.0f;
    for (int k = 0; k < D; ++k) a = fmaf(__ldg(p.st32 + (size_t)k * p.m + i), qs[k], a);
    dst[D + i] = a;
  }
}

// The B-bit field at compile-time bit POS of a key's code words (in registers).
template <int B, int POS, int CW>
__device__ __forceinline__ uint32_t code_field(const uint32_t (&cw)[CW]) {
  constexpr int w = POS >> 5, sh = POS & 31;
  if constexpr (sh + B <= 32 || w + 1 >= CW) return (cw[w] >> sh) & ((1u << B) - 1u);
  else return __funnelshift_r(cw[w], cw[w + 1], sh) & ((1u << B) - 1u);
}

__device__ __forceinline__ float4 fold2(float4 a, float4 b, float2 c) {
  return make_float4(fmaf(a.x, c.x, b.x * c.y), fmaf(a.y, c.x, b.y * c.y), fmaf(a.z, c.x, b.z * c.y),
                     fmaf(a.w, c.x, b.w * c.y));
}

// The fold of the subtree (level LV, index IX) for 4 queries at once: their
// coordinates IX 2^LV .. of q~ (qs: [coordinate] x 4 queries) against the
// key's angle tree; the angle's index comes from the key's code words at a
// compile-time bit position, its (cos, sin) from the level's table.
template <int D, int B, int LV, int IX, int CW>
__device__ __forceinline__ float4 polar_fold4(const float4* qs, const uint32_t (&cw)[CW], const float2 (*tb)[16]) {
  const float2 c = tb[LV - 1][code_field<B, (level_offset(D, LV) + IX) * B>(cw)];
  if constexpr (LV == 1) {
    return fold2(qs[2 * IX], qs[2 * IX + 1], c);
  } else {
    const float4 a = polar_fold4<D, B, LV - 1, 2 * IX>(qs, cw, tb);
    const float4 b = polar_fold4<D, B, LV - 1, 2 * IX + 1>(qs, cw, tb);
    return fold2(a, b, c);
  }
}

// ---- logits: one thread per key, 4 queries per pass --------------------------------
// grid (ceil(n / 128), ceil(nq / 64)), block 128.  Thread k holds key k's code
// words in registers (loaded once) and folds them against 4 queries at a
// time; shared memory holds the level tables, the 4 queries' q~ and S q
// interleaved by query (one 16-byte load gives a coordinate of all 4), and
// per group of 4 sketch rows the 16 signed sums of its z values.
template <int D, int B>
__global__ void __launch_bounds__(kPolLogThreads, D == 256 ? 2 : D == 128 ? 3 : 4) polar_logits_kernel(PolarParams p) {
  constexpr int L = D == 64 ? 6 : D == 128 ? 7 : 8;
  constexpr int CW = ((D - 1) * B + 31) / 32;
  constexpr int CW4 = (CW + 3) / 4;                 // 16-byte pieces of the code words
  __shared__ float2 tb[L][16];                      // (cos, sin) of the level's centroids
  __shared__ float4 qs[D];                          // q~[coordinate], 4 queries
  __shared__ float4 zs[D];                          // (S q)[row], 4 queries (m <= d)
  __shared__ float4 nt[D / 4][16];                  // per group of 4 rows: sum_k +-z_k (bit k set: -z_k)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int tid = threadIdx.x;
  const int64_t key = (int64_t)blockIdx.x * kPolLogThreads + tid;
  const bool has = key < p.n;
  const int M = p.m, RW = p.rec_words, SW = p.sign_words;
  for (int i = tid; i < L * 16; i += kPolLogThreads) {
    const int l = i / 16, e = i % 16;
    tb[l][e] = make_float2(p.tabs[l * 64 + e], p.tabs[l * 64 + 16 + e]);
  }
  // this key's code words and norms (records are 16-byte multiples)
  uint32_t cw[4 * CW4];
  float kn = 0.0f, kr = 0.0f;
  if (has) {
    const uint4* r4 = reinterpret_cast<const uint4*>(p.crec + key * RW);
#pragma unroll
    for (int i = 0; i < CW4; ++i) {
      const uint4 v = __ldg(r4 + i);
      cw[4 * i] = v.x; cw[4 * i + 1] = v.y; cw[4 * i + 2] = v.z; cw[4 * i + 3] = v.w;
    }
    const uint32_t nw = __ldg(p.crec + key * RW + CW + SW);
    kn = __half2float(__ushort_as_half((unsigned short)(nw & 0xFFFFu)));
    kr = __half2float(__ushort_as_half((unsigned short)(nw >> 16)));
  } else {
#pragma unroll
    for (int i = 0; i < 4 * CW4; ++i) cw[i] = 0u;
  }
  const int q_begin = blockIdx.y * kPolQBlock, q_end = min(p.nq, q_begin + kPolQBlock);
  for (int qb = q_begin; qb < q_end; qb += kPolQPass) {
    __syncthreads();                                 // the previous pass is done with qs, zs, nt
    for (int t = tid; t < kPolQPass * (D + M); t += kPolLogThreads) {
      const int s = t / (D + M), e = t % (D + M);
      const float v = qb + s < q_end ? p.qrot[(int64_t)(qb + s) * (D + M) + e] : 0.0f;
      float* dst = e < D ? reinterpret_cast<float*>(&qs[e]) : reinterpret_cast<float*>(&zs[e - D]);
      dst[s] = v;
    }
    __syncthreads();
    for (int t = tid; t < (M / 4) * 16; t += kPolLogThreads) {
      const int g4 = t / 16, v = t % 16;
      const float4 z0 = zs[4 * g4], z1 = zs[4 * g4 + 1], z2 = zs[4 * g4 + 2], z3 = zs[4 * g4 + 3];
      auto sum = [&](float a, float b, float c, float d) {
        return ((v & 1) ? -a : a) + ((v & 2) ? -b : b) + ((v & 4) ? -c : c) + ((v & 8) ? -d : d);
      };
      nt[g4][v] = make_float4(sum(z0.x, z1.x, z2.x, z3.x), sum(z0.y, z1.y, z2.y, z3.y),
                              sum(z0.z, z1.z, z2.z, z3.z), sum(z0.w, z1.w, z2.w, z3.w));
    }
    __syncthreads();
    if (!has) continue;
    float4 s = polar_fold4<D, B, L, 0>(qs, cw, tb);
    if (M > 0) {
      // <S q, sign> with sign_i = -1 where bit i is set: one table entry per 4 rows
      float4 sk = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      for (int w = 0; w < SW; ++w) {
        const uint32_t bits = __ldg(p.crec + key * RW + CW + w);
#pragma unroll
        for (int n4 = 0; n4 < 8; ++n4) {
          const float4 e = nt[8 * w + n4][(bits >> (4 * n4)) & 15u];
          sk.x += e.x; sk.y += e.y; sk.z += e.z; sk.w += e.w;
        }
      }
      const float f = p.qjl_scale * kr;
      s = make_float4(fmaf(f, sk.x, s.x), fmaf(f, sk.y, s.y), fmaf(f, sk.z, s.z), fmaf(f, sk.w, s.w));
    }
    const float o[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
    for (int j = 0; j < kPolQPass; ++j)
      if (qb + j < q_end) p.out[(int64_t)(qb + j) * p.out_stride + key] = kn * o[j];
  }
}

}  // namespace tqd

namespace tq {

tq_status polar_build(int d, int bits, int m, uint64_t seed_pi, uint64_t seed_s, tq_polar** out) {
  auto* P = new tq_polar();
  P->d = d;
  P->bits = bits;
  P->m = m;
  int L = 0;
  while ((1 << L) < d) ++L;
  P->levels = L;
  P->code_words = ((d - 1) * bits + 31) / 32;
  P->sign_words = m / 32;
  const int raw = P->code_words + P->sign_words + 1;
  P->rec_words = (raw + 3) / 4 * 4;
  P->seed_pi = seed_pi;
  P->seed_s = seed_s;
  P->device = current_device();
  std::vector<double> G((size_t)d * d);
  tqhost::gaussian_fill(seed_pi, G.size(), G.data());
  P->pi = tqhost::orthogonal_factor(G, d);
  P->s.assign((size_t)m * d, 0.0);
  if (m > 0) tqhost::gaussian_fill(seed_s, P->s.size(), P->s.data());
  P->qjl_scale = m > 0 ? std::sqrt(3.14159265358979323846 / 2.0) / m : 0.0;
  for (int l = 1; l <= L; ++l) P->books.push_back(tqhost::polar_angle_lloyd_max(l, bits));
  // device tables: Pi^T, Pi, S^T (fp32), per-level cos / sin / centroid / boundaries
  const size_t n_pit = (size_t)d * d, n_pi = n_pit, n_st = (size_t)d * std::max(m, 1), n_tab = (size_t)L * 64;
  std::vector<float> hb(n_pit + n_pi + n_st + n_tab, 0.0f);
  float* hp = hb.data();
  for (int j = 0; j < d; ++j)
    for (int k = 0; k < d; ++k) {
      hp[(size_t)k * d + j] = (float)P->pi[(size_t)j * d + k];
      hp[n_pit + (size_t)j * d + k] = (float)P->pi[(size_t)j * d + k];
    }
  for (int i = 0; i < m; ++i)
    for (int k = 0; k < d; ++k) hp[n_pit + n_pi + (size_t)k * m + i] = (float)P->s[(size_t)i * d + k];
  float* ht = hp + n_pit + n_pi + n_st;
  for (int l = 0; l < L; ++l) {
    const auto& bk = P->books[l];
    for (int i = 0; i < (1 << bits); ++i) {
      ht[l * 64 + i] = (float)std::cos(bk.centroids[i]);
      ht[l * 64 + 16 + i] = (float)std::sin(bk.centroids[i]);
      ht[l * 64 + 32 + i] = (float)bk.centroids[i];
    }
    for (int i = 0; i + 1 < (1 << bits); ++i) ht[l * 64 + 48 + i] = (float)bk.boundaries[i];
  }
  void* blk = nullptr;
  cudaError_t e = cudaMalloc(&blk, hb.size() * sizeof(float));
  if (e != cudaSuccess) {
    delete P;
    return cuda_fail(e, "tq_polar_build: device tables");
  }
  e = cudaMemcpy(blk, hb.data(), hb.size() * sizeof(float), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(blk);
    delete P;
    return cuda_fail(e, "tq_polar_build: copying the tables");
  }
  P->dev_block = blk;
  float* f = reinterpret_cast<float*>(blk);
  P->pit32 = f;
  P->pi32 = f + n_pit;
  P->st32 = f + n_pit + n_pi;
  P->tabs = f + n_pit + n_pi + n_st;
  *out = P;
  return TQ_OK;
}

int polar_record_bytes(const tq_polar* P) { return 4 * P->rec_words; }

void polar_free(tq_polar* P) {
  if (!P) return;
  if (P->dev_block) cudaFree(P->dev_block);
  delete P;
}

static tqd::PolarParams polar_params(const tq_polar* P) {
  tqd::PolarParams p{};
  p.d = P->d;
  p.bits = P->bits;
  p.m = P->m;
  p.levels = P->levels;
  p.code_words = P->code_words;
  p.sign_words = P->sign_words;
  p.rec_words = P->rec_words;
  p.pit32 = P->pit32;
  p.pi32 = P->pi32;
  p.st32 = P->st32;
  p.tabs = P->tabs;
  p.qjl_scale = (float)P->qjl_scale;
  return p;
}

template <int D>
static tq_status launch_polar_encode_t(const tqd::PolarParams& p, int64_t grid, cudaStream_t st) {
  constexpr size_t smem = sizeof(tqd::PolarEncSmem<D>);
  static PerDeviceOnce attr;
  if (const int dev_ = current_device(); attr.need(dev_)) {
    cudaError_t e = cudaFuncSetAttribute(tqd::polar_encode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "tq_polar_encode: smem attribute");
    attr.mark(dev_);
  }
  tqd::polar_encode_kernel<D><<<(unsigned)grid, tqd::kPolThreads, smem, st>>>(p);
  return cuda_fail(cudaGetLastError(), "tq_polar_encode launch");
}

tq_status polar_encode(const tq_polar* P, const void* x, tq_dtype dt, int64_t n, void* rec, uint32_t* err,
                       cudaStream_t st) {
  tqd::PolarParams p = polar_params(P);
  p.x = x;
  p.dtype = dt;
  p.n = n;
  p.rec = reinterpret_cast<uint32_t*>(rec);
  p.err = err;
  const int64_t grid = (n + tqd::kPolVec - 1) / tqd::kPolVec;
  if (grid > 0x7fffffffLL) return fail(TQ_EINVAL, "tq_polar_encode: n too large");
  switch (P->d) {
    case 64: return launch_polar_encode_t<64>(p, grid, st);
    case 128: return launch_polar_encode_t<128>(p, grid, st);
    case 256: return launch_polar_encode_t<256>(p, grid, st);
  }
  return fail(TQ_EUNSUPPORTED, "tq_polar_encode: d must be 64, 128 or 256");
}

size_t polar_logits_workspace(const tq_polar* P, int nq) {
  return (size_t)nq * (P->d + P->m) * sizeof(float);
}

template <int D, int B>
static tq_status launch_polar_logits_t(const tqd::PolarParams& p, cudaStream_t st) {
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = st;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3((unsigned)p.nq);
  cfg.blockDim = dim3(128);
  cudaError_t e = cudaLaunchKernelEx(&cfg, tqd::polar_prep_kernel<D>, p);
  if (e != cudaSuccess) return cuda_fail(e, "tq_polar_logits: query preparation launch");
  cfg.gridDim = dim3((unsigned)((p.n + tqd::kPolLogThreads - 1) / tqd::kPolLogThreads),
                     (unsigned)((p.nq + tqd::kPolQBlock - 1) / tqd::kPolQBlock));
  cfg.blockDim = dim3(tqd::kPolLogThreads);
  e = cudaLaunchKernelEx(&cfg, tqd::polar_logits_kernel<D, B>, p);
  if (e != cudaSuccess) return cuda_fail(e, "tq_polar_logits launch");
  return TQ_OK;
}

template <int D>
static tq_status launch_polar_logits_d(const tqd::PolarParams& p, cudaStream_t st) {
  switch (p.bits) {
    case 1: return launch_polar_logits_t<D, 1>(p, st);
    case 2: return launch_polar_logits_t<D, 2>(p, st);
    case 3: return launch_polar_logits_t<D, 3>(p, st);
    case 4: return launch_polar_logits_t<D, 4>(p, st);
  }
  return fail(TQ_EUNSUPPORTED, "tq_polar_logits: bits must be 1..4");
}

tq_status polar_logits(const tq_polar* P, const void* rec, int64_t n, const void* q, tq_dtype dt, int nq, float* out,
                       int64_t out_stride, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!ws || ws_bytes < polar_logits_workspace(P, nq)) return fail(TQ_EINVAL, "tq_polar_logits: workspace too small");
  if ((n + tqd::kPolLogThreads - 1) / tqd::kPolLogThreads > 0x7fffffffLL ||
      (nq + tqd::kPolQBlock - 1) / tqd::kPolQBlock > 65535)
    return fail(TQ_EINVAL, "tq_polar_logits: n or nq too large");
  tqd::PolarParams p = polar_params(P);
  p.crec = reinterpret_cast<const uint32_t*>(rec);
  p.n = n;
  p.q = q;
  p.dtype = dt;
  p.nq = nq;
  p.qrot = reinterpret_cast<float*>(ws);
  p.out = out;
  p.out_stride = out_stride;
  switch (P->d) {
    case 64: return launch_polar_logits_d<64>(p, st);
    case 128: return launch_polar_logits_d<128>(p, st);
    case 256: return launch_polar_logits_d<256>(p, st);
  }
  return fail(TQ_EUNSUPPORTED, "tq_polar_logits: d must be 64, 128 or 256");
}

}  // namespace tq
