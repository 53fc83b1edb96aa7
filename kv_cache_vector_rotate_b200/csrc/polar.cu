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
// not by HBM.  The cos and sin of the centroids come from per-level tables,
// staged per key in shared memory and shared by the CTA's queries; the fold
// is a compile-time tree, so its partial sums stay in registers.

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

constexpr int kPolVec = 8;         // vectors per encode CTA
constexpr int kPolThreads = 256;
constexpr int kPolLogThreads = 128;
constexpr int kPolQPass = 4;       // queries per pass of a logits CTA
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

// ---- encode: one CTA of 256 threads per 8 vectors -----------------------------------
template <int D>
__global__ void __launch_bounds__(kPolThreads) polar_encode_kernel(PolarParams p) {
  constexpr int L = D == 64 ? 6 : D == 128 ? 7 : 8;
  __shared__ float us[kPolVec][D];          // u = x / ||x|| (original space)
  __shared__ float ys[kPolVec][D];          // Pi u, then the radii of the level being done
  __shared__ float rs[kPolVec][D];          // radii of the next level; u_hat; then r
  __shared__ float rt[kPolVec][D / 2];      // ping-pong buffer of the inverse recursion
  __shared__ uint8_t ix[kPolVec][D];        // angle indices
  __shared__ uint32_t cw[kPolVec][33];      // code words (<= 32) + 1 spare
  __shared__ uint32_t sw[kPolVec][8];       // sign words (m <= 256)
  __shared__ float nrm[kPolVec], rnrm[kPolVec];
  __shared__ float tb[8][4][16];
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
  if (warp < kPolVec) {
    float s2 = 0.0f;
    for (int k = lane; k < D; k += 32) s2 = fmaf(us[warp][k], us[warp][k], s2);
#pragma unroll
    for (int o = 16; o; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    if (lane == 0) nrm[warp] = sqrtf(s2);
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
    for (int k = 0; k < D; ++k) {
      const float pk = __ldg(p.pit32 + (size_t)k * D + j);   // Pi[j][k]
#pragma unroll
      for (int a = 0; a < VPT; ++a) acc[a] = fmaf(pk, us[g + VG * a][k], acc[a]);
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
      for (int j = 0; j < D; ++j) {
        const float pjk = __ldg(p.pi32 + (size_t)j * D + k);   // Pi[j][k]
#pragma unroll
        for (int a = 0; a < VPT; ++a) acc[a] = fmaf(pjk, rs[g + VG * a][j], acc[a]);
      }
#pragma unroll
      for (int a = 0; a < VPT; ++a) ys[g + VG * a][k] = us[g + VG * a][k] - acc[a];
    }
    __syncthreads();
    if (warp < kPolVec) {
      float s2 = 0.0f;
      for (int k = lane; k < D; k += 32) s2 = fmaf(ys[warp][k], ys[warp][k], s2);
#pragma unroll
      for (int o = 16; o; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
      if (lane == 0) rnrm[warp] = sqrtf(s2);
    }
    // the signs of S r: thread (i, vector)
    for (int t = tid; t < kPolVec * M; t += kPolThreads) {
      const int v = t / M, i = t % M;
      float pr = 0.0f;
      for (int k = 0; k < D; ++k) pr = fmaf(__ldg(p.st32 + (size_t)k * M + i), ys[v][k], pr);
      if (pr < 0.0f) atomicOr(&sw[v][i >> 5], 1u << (i & 31));
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

// The fold of the subtree (level LV, index IX): coordinates IX 2^LV .. of
// q~ against the key's angle tree (cs: cos, sin of every angle's centroid).
template <int D, int LV, int IX>
__device__ __forceinline__ float polar_fold(const float* qv, const float2* cs) {
  if constexpr (LV == 1) {
    const float2 c = cs[IX];
    return fmaf(qv[2 * IX], c.x, qv[2 * IX + 1] * c.y);
  } else {
    const float a = polar_fold<D, LV - 1, 2 * IX>(qv, cs);
    const float b = polar_fold<D, LV - 1, 2 * IX + 1>(qv, cs);
    const float2 c = cs[level_offset(D, LV) + IX];
    return fmaf(a, c.x, b * c.y);
  }
}

// ---- logits: KEYS keys x 64 queries per CTA of 128 threads ------------------------
// grid (ceil(n / KEYS), ceil(nq / 64)).  The keys' angle tables (cos, sin of
// the centroids) are staged once; then passes of 4 queries: thread (key
// kk = tid % KEYS, query slot tid / KEYS) folds its key against its query.
template <int D>
__global__ void __launch_bounds__(kPolLogThreads) polar_logits_kernel(PolarParams p) {
  constexpr int L = D == 64 ? 6 : D == 128 ? 7 : 8;
  constexpr int KEYS = D == 256 ? 16 : 32;
  constexpr int QL = kPolLogThreads / KEYS;          // query slots per pass (4 or 8)
  constexpr int CSR = D - 1;                         // row stride (float2): an odd count, rows in distinct banks
  extern __shared__ float4 pol_dsm[];
  auto cs = reinterpret_cast<float2(*)[CSR]>(pol_dsm);                     // [KEYS][CSR]
  auto qs = reinterpret_cast<float(*)[2 * D]>(pol_dsm + (KEYS * CSR + 1) / 2);   // [QL][2D]: Pi q, then S q (m <= D)
  // per query slot and group of 4 sketch rows, the 16 values sum_k +-z_k of
  // the group's sign patterns (bit k set: -z_k)
  auto nt = reinterpret_cast<float(*)[D / 4][16]>(pol_dsm + (KEYS * CSR + 1) / 2 + QL * 2 * D / 4);   // [QL][m/4][16]
  __shared__ uint32_t recs[KEYS * 48];               // the CTA's records (<= 44 words each), copied once
  __shared__ float kn[KEYS], kr[KEYS];
  __shared__ float tb[8][2][16];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int tid = threadIdx.x;
  const int64_t k0 = (int64_t)blockIdx.x * KEYS;
  const int nk = (int)min((int64_t)KEYS, p.n - k0);
  const int B = p.bits, M = p.m, RW = p.rec_words, CW = p.code_words, SW = p.sign_words;
  for (int i = tid; i < L * 32; i += kPolLogThreads) {
    const int l = i / 32, w = (i / 16) % 2, e = i % 16;
    tb[l][w][e] = p.tabs[l * 64 + w * 16 + e];
  }
  __syncthreads();
  // the records, coalesced (consecutive keys are consecutive records)
  for (int t = tid; t < nk * RW; t += kPolLogThreads) recs[t] = p.crec[k0 * RW + t];
  __syncthreads();
  // stage the keys: angle tables, norms
  for (int t = tid; t < KEYS * (D - 1); t += kPolLogThreads) {
    const int kk = t / (D - 1), a = t % (D - 1);
    float2 c = make_float2(0.0f, 0.0f);
    if (kk < nk) {
      const uint32_t* r = recs + kk * RW;
      // level l holds the angles a with D / 2^l < D - a <= D / 2^(l - 1)
      const int l = L + 1 - (32 - __clz(D - a - 1));
      const int idx = (int)get_field(r, a * B, B);
      c = make_float2(tb[l - 1][0][idx], tb[l - 1][1][idx]);
    }
    cs[kk][a] = c;
  }
  if (tid < KEYS) {
    float a = 0.0f, b = 0.0f;
    if (tid < nk) {
      const uint32_t nw = recs[tid * RW + CW + SW];
      a = __half2float(__ushort_as_half((unsigned short)(nw & 0xFFFFu)));
      b = __half2float(__ushort_as_half((unsigned short)(nw >> 16)));
    }
    kn[tid] = a;
    kr[tid] = b;
  }
  const int kk = tid % KEYS, ql = tid / KEYS;
  const int q_begin = blockIdx.y * kPolQBlock, q_end = min(p.nq, q_begin + kPolQBlock);
  for (int qb = q_begin; qb < q_end; qb += QL) {
    __syncthreads();                                 // tables staged / the previous pass done
    for (int t = tid; t < QL * (D + M); t += kPolLogThreads) {
      const int s = t / (D + M), e = t % (D + M);
      qs[s][e] = qb + s < q_end ? p.qrot[(int64_t)(qb + s) * (D + M) + e] : 0.0f;
    }
    __syncthreads();
    for (int t = tid; t < QL * (M / 4) * 16; t += kPolLogThreads) {
      const int s = t / ((M / 4) * 16), rem = t % ((M / 4) * 16), g4 = rem / 16, v = rem % 16;
      const float* z = &qs[s][D + 4 * g4];
      nt[s][g4][v] = ((v & 1) ? -z[0] : z[0]) + ((v & 2) ? -z[1] : z[1]) + ((v & 4) ? -z[2] : z[2]) +
                     ((v & 8) ? -z[3] : z[3]);
    }
    __syncthreads();
    const int qi = qb + ql;
    if (qi < q_end && kk < nk) {
      float s = polar_fold<D, L, 0>(qs[ql], cs[kk]);
      if (M > 0) {
        // <S q, sign> with sign_i = -1 where bit i is set: one table entry per 4 rows
        float sk = 0.0f;
        for (int w = 0; w < (M >> 5); ++w) {
          const uint32_t bits = recs[kk * RW + CW + w];
#pragma unroll
          for (int n4 = 0; n4 < 8; ++n4) sk += nt[ql][8 * w + n4][(bits >> (4 * n4)) & 15u];
        }
        s = fmaf(p.qjl_scale * kr[kk], sk, s);
      }
      p.out[(int64_t)qi * p.out_stride + k0 + kk] = kn[kk] * s;
    }
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
    case 64: tqd::polar_encode_kernel<64><<<(unsigned)grid, tqd::kPolThreads, 0, st>>>(p); break;
    case 128: tqd::polar_encode_kernel<128><<<(unsigned)grid, tqd::kPolThreads, 0, st>>>(p); break;
    case 256: tqd::polar_encode_kernel<256><<<(unsigned)grid, tqd::kPolThreads, 0, st>>>(p); break;
    default: return fail(TQ_EUNSUPPORTED, "tq_polar_encode: d must be 64, 128 or 256");
  }
  return cuda_fail(cudaGetLastError(), "tq_polar_encode launch");
}

size_t polar_logits_workspace(const tq_polar* P, int nq) {
  return (size_t)nq * (P->d + P->m) * sizeof(float);
}

template <int D>
static tq_status launch_polar_logits_t(const tqd::PolarParams& p, cudaStream_t st) {
  constexpr int KEYS = D == 256 ? 16 : 32;
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
  constexpr int QL = tqd::kPolLogThreads / KEYS;
  const size_t smem = (size_t)((KEYS * (D - 1) + 1) / 2) * 16 + (size_t)QL * 2 * D * sizeof(float) +
                      (size_t)QL * (D / 4) * 16 * sizeof(float);
  static PerDeviceOnce attr;
  if (const int dev_ = current_device(); attr.need(dev_)) {
    e = cudaFuncSetAttribute(tqd::polar_logits_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "tq_polar_logits: smem attribute");
    attr.mark(dev_);
  }
  cfg.gridDim = dim3((unsigned)((p.n + KEYS - 1) / KEYS), (unsigned)((p.nq + tqd::kPolQBlock - 1) / tqd::kPolQBlock));
  cfg.blockDim = dim3(tqd::kPolLogThreads);
  cfg.dynamicSmemBytes = smem;
  e = cudaLaunchKernelEx(&cfg, tqd::polar_logits_kernel<D>, p);
  if (e != cudaSuccess) return cuda_fail(e, "tq_polar_logits launch");
  return TQ_OK;
}

tq_status polar_logits(const tq_polar* P, const void* rec, int64_t n, const void* q, tq_dtype dt, int nq, float* out,
                       int64_t out_stride, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!ws || ws_bytes < polar_logits_workspace(P, nq)) return fail(TQ_EINVAL, "tq_polar_logits: workspace too small");
  const int keys = P->d == 256 ? 16 : 32;
  if ((n + keys - 1) / keys > 0x7fffffffLL || (nq + tqd::kPolQBlock - 1) / tqd::kPolQBlock > 65535)
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
    case 64: return launch_polar_logits_t<64>(p, st);
    case 128: return launch_polar_logits_t<128>(p, st);
    case 256: return launch_polar_logits_t<256>(p, st);
  }
  return fail(TQ_EUNSUPPORTED, "tq_polar_logits: d must be 64, 128 or 256");
}

}  // namespace tq
