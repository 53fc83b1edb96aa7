// Quantize-and-append on CUDA cores, one thread per coordinate.
//
// "TurboQuant explained" (a2a-mcp.org) §Stage 1: normalize, rotate by Pi,
// map each rotated coordinate to its Lloyd-Max cell; §Stage 2: signs of a
// Gaussian projection of the residual; §How to implement: quantize on every
// cache update.  This kernel serves the small appends of a decode step (a few
// new tokens per call) and the shapes the tensor-core kernel does not cover;
// it writes exactly the same records.
//
// A CTA of d_pad threads codes up to R vectors at once.  Thread j owns rotated
// coordinate j (and QJL row j).  The projection matrices are streamed through
// shared memory in blocks of KB rows of Pi^T (resp. (S Pi^T)^T), each block
// fetched with all of its 16-byte loads in flight at once, so a vector costs
// a couple of memory round trips rather than one per few multiply-adds; each
// block then serves all R vectors.  The packed words are assembled in shared
// memory, each thread ORing its code bits into its chunk's words.

#include "pack.cuh"

namespace tqd {

struct QuantizeSimtParams {
  const void* x;
  tq_dtype dtype;
  int64_t rows;        // batch * n_kv_heads * n_new
  int64_t n_new;
  int n_kv_heads;
  int d;
  int rows_per_cta;    // <= kSimtRows
  const int32_t* start_pos;
  tq::CacheView cv;
  const float* pit32;    // Pi^T       [d][d_pad]
  const float* srott32;  // (S Pi^T)^T [d_pad][m_pad]
  const float* bound32;
  const float* cent32;
};

constexpr int kSimtRows = 8;          // vectors per CTA
constexpr int kSimtStageFloats = 16384;  // 64 KB of matrix rows staged at a time

// acc[r] += sum_k Mt[k][j] * vec[r][k] for k < klen, Mt row-major [klen][DP],
// staged through `stage` (kSimtStageFloats floats) in blocks of KB rows.
template <int DP>
__device__ __forceinline__ void stream_matvec(const float* __restrict__ Mt, int klen, const float* vec,
                                              int vstride, int R, float* stage, float (&acc)[kSimtRows]) {
  constexpr int KB = kSimtStageFloats / DP;
  const int j = threadIdx.x;
  for (int k0 = 0; k0 < klen; k0 += KB) {
    const int kn = min(KB, klen - k0);
    const int n4 = kn * DP / 4;
    const float4* src = reinterpret_cast<const float4*>(Mt + (size_t)k0 * DP);
    __syncthreads();                  // the previous block is consumed
    // every 16-byte copy of the block in flight at once, no registers held
    for (int e = j; e < n4; e += DP) {
      const unsigned dst = (unsigned)__cvta_generic_to_shared(stage + 4 * e);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src + e) : "memory");
    }
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    for (int k = 0; k < kn; ++k) {
      const float m = stage[k * DP + j];
#pragma unroll
      for (int r = 0; r < kSimtRows; ++r)
        if (r < R) acc[r] = fmaf(m, vec[r * vstride + k0 + k], acc[r]);
    }
  }
}

template <int BITS, int E, int F>
__global__ void __launch_bounds__(4 * E) quantize_simt_kernel(QuantizeSimtParams p) {
  constexpr int DP = 4 * E;          // threads = padded coordinates
  constexpr int K = 1 << BITS;
  constexpr int H = K / 2;
  using CW = ChunkWords<BITS, E, F>;
  extern __shared__ float4 dyn_stage[];
  float* stage = reinterpret_cast<float*>(dyn_stage);
  __shared__ float xs[kSimtRows][DP];
  __shared__ float rs[kSimtRows][DP];
  __shared__ float red[kSimtRows][DP / 32];
  __shared__ float nrm[kSimtRows];
  __shared__ uint32_t wsm[kSimtRows][4 * CW::W];
  __shared__ float sb[K];
  __shared__ float sc[K];
  const int j = threadIdx.x;         // coordinate (and QJL row) of this thread
  const int lane = j & 31, warp = j >> 5;
  const int t = j / E, l = j % E;    // chunk and local position
  const int d = p.d;
  if (j < K) {
    sb[j] = j == 0 ? 0.0f : p.bound32[j - 1];
    sc[j] = p.cent32[j];
  }
  const int64_t per_seq = (int64_t)p.n_kv_heads * p.n_new;
  const int64_t stride = (int64_t)gridDim.x * p.rows_per_cta;

  for (int64_t row0 = (int64_t)blockIdx.x * p.rows_per_cta; row0 < p.rows; row0 += stride) {
    const int R = (int)min((int64_t)p.rows_per_cta, p.rows - row0);
    __syncthreads();                 // the previous rows' shared data is consumed
    for (int r = 0; r < R; ++r) {
      const float xv = j < d ? load_elem(p.x, (row0 + r) * d + j, p.dtype) : 0.0f;
      xs[r][j] = xv;
      float n2 = xv * xv;
#pragma unroll
      for (int o = 16; o; o >>= 1) n2 += __shfl_xor_sync(0xffffffffu, n2, o);
      if (lane == 0) red[r][warp] = n2;
    }
    for (int i = j; i < kSimtRows * 4 * CW::W; i += DP) (&wsm[0][0])[i] = 0u;
    __syncthreads();
    if (j < R) {
      float tot = 0.0f;
#pragma unroll
      for (int w = 0; w < DP / 32; ++w) tot += red[j][w];
      nrm[j] = sqrtf(tot);
    }
    // y_j = (Pi x)_j for every row
    float acc[kSimtRows];
#pragma unroll
    for (int r = 0; r < kSimtRows; ++r) acc[r] = 0.0f;
    stream_matvec<DP>(p.pit32, d, &xs[0][0], DP, R, stage, acc);   // syncs before use of nrm

    int idxs[kSimtRows];
#pragma unroll
    for (int r = 0; r < kSimtRows; ++r) {
      idxs[r] = H;
      if (r < R) {
        const float norm = nrm[r];
        const float u = acc[r] * (norm > 0.0f ? 1.0f / norm : 0.0f);
        int idx = 0;
#pragma unroll
        for (int step = K / 2; step >= 1; step >>= 1)
          if (u >= sb[idx + step]) idx += step;
        idxs[r] = idx;
        const float res = j < d ? u - sc[idx] : 0.0f;
        rs[r][j] = res;
        float r2 = res * res;
#pragma unroll
        for (int o = 16; o; o >>= 1) r2 += __shfl_xor_sync(0xffffffffu, r2, o);
        if (lane == 0) red[r][warp] = r2;
      }
    }
    // index codes -> words (each thread ORs its bits into its chunk's words)
#pragma unroll
    for (int r = 0; r < kSimtRows; ++r) {
      if (r >= R) break;
      if (j < d) or_code_bits<BITS, E>(&wsm[r][t * CW::W], l, idxs[r]);
    }
    if constexpr (F > 0) {
      // QJL row j: (S Pi^T r)_j; rows past m are padding and store 0
#pragma unroll
      for (int r = 0; r < kSimtRows; ++r) acc[r] = 0.0f;
      stream_matvec<DP>(p.srott32, DP, &rs[0][0], DP, R, stage, acc);
#pragma unroll
      for (int r = 0; r < kSimtRows; ++r) {
        if (r >= R) break;
        if (acc[r] < 0.0f) atomicOr(&wsm[r][t * CW::W + CW::q0 + l / 32], 1u << qjl_bit(l));
      }
    }
    __syncthreads();                 // words and residual norms complete

    // store: 4 * W words per record, then the norm slot
    for (int r = 0; r < R; ++r) {
      const int64_t row = row0 + r;
      const int64_t b = row / per_seq;
      const int h = (int)((row / p.n_new) % p.n_kv_heads);
      const int64_t pos = p.start_pos[b] + row % p.n_new;
      const int64_t hb = head_block_offset(p.cv, b, h, pos);
      if (hb < 0) continue;
      const int slot = (int)(pos % p.cv.page_tokens);
      uint32_t* rec = reinterpret_cast<uint32_t*>(p.cv.pages + hb + (int64_t)slot * 16 * CW::W);
      if (j < 4 * CW::W) rec[j] = wsm[r][j];
      if (j == 0) {
        const __half nh = __float2half_rn(nrm[r]);
        if (__hisinf(nh)) report(p.cv.err, TQ_DEV_ERR_RANGE);
        __half* nslot = reinterpret_cast<__half*>(p.cv.pages + hb + (int64_t)p.cv.page_tokens * 16 * CW::W +
                                                  (int64_t)slot * (F > 0 ? 4 : 2));
        nslot[0] = nh;
        if constexpr (F > 0) {
          float r2 = 0.0f;
#pragma unroll
          for (int w = 0; w < DP / 32; ++w) r2 += red[r][w];
          nslot[1] = __float2half_rn(sqrtf(r2));
        }
      }
    }
  }
}

}  // namespace tqd

namespace tq {

template <int BITS, int E, int F>
static tq_status launch_simt(tqd::QuantizeSimtParams p, cudaStream_t st) {
  // one vector per CTA while the GPU is not full, up to kSimtRows after that
  const int64_t sms = device_sm_count();
  int rpc = (int)((p.rows + sms * 4 - 1) / (sms * 4));
  rpc = rpc < 1 ? 1 : rpc > tqd::kSimtRows ? tqd::kSimtRows : rpc;
  p.rows_per_cta = rpc;
  const int64_t ctas = (p.rows + rpc - 1) / rpc;
  const unsigned blocks = (unsigned)(ctas < sms * 8 ? ctas : sms * 8);
  const size_t smem = tqd::kSimtStageFloats * sizeof(float);
  static PerDeviceOnce attr_set;   // per instantiation
  if (const int dev_ = current_device(); attr_set.need(dev_)) {
    cudaError_t e = cudaFuncSetAttribute(tqd::quantize_simt_kernel<BITS, E, F>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "quantize_simt: smem attribute");
    attr_set.mark(dev_);
  }
  tqd::quantize_simt_kernel<BITS, E, F><<<blocks, 4 * E, smem, st>>>(p);
  return TQ_OK;
}

template <int BITS>
static int dispatch_simt_e(const Layout& L, const tqd::QuantizeSimtParams& p, cudaStream_t st,
                           tq_status* s) {
  if (L.E == 32 && L.F == 32) return *s = launch_simt<BITS, 32, 32>(p, st), 1;
  if (L.E == 32 && L.F == 0) return *s = launch_simt<BITS, 32, 0>(p, st), 1;
  if (L.E == 16 && L.F == 16) return *s = launch_simt<BITS, 16, 16>(p, st), 1;
  if (L.E == 16 && L.F == 0) return *s = launch_simt<BITS, 16, 0>(p, st), 1;
  if (L.E == 64 && L.F == 64) return *s = launch_simt<BITS, 64, 64>(p, st), 1;
  if (L.E == 64 && L.F == 0) return *s = launch_simt<BITS, 64, 0>(p, st), 1;
  if (L.E == 48 && L.F == 48) return *s = launch_simt<BITS, 48, 48>(p, st), 1;
  if (L.E == 48 && L.F == 0) return *s = launch_simt<BITS, 48, 0>(p, st), 1;
  return 0;
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
  p.rows_per_cta = 1;
  p.start_pos = start_pos;
  p.cv = cv;
  p.pit32 = cb->pit32;
  p.srott32 = cb->srott32;
  p.bound32 = cb->bound32;
  p.cent32 = cb->cent32;
  int ok = 0;
  tq_status s = TQ_OK;
  switch (cb->lay.bits) {
    case 1: ok = dispatch_simt_e<1>(cb->lay, p, st, &s); break;
    case 2: ok = dispatch_simt_e<2>(cb->lay, p, st, &s); break;
    case 3: ok = dispatch_simt_e<3>(cb->lay, p, st, &s); break;
    case 4: ok = dispatch_simt_e<4>(cb->lay, p, st, &s); break;
  }
  if (!ok) return fail(TQ_EUNSUPPORTED, "quantize: no kernel for this (d, m)");
  if (s != TQ_OK) return s;
  return cuda_fail(cudaGetLastError(), "quantize_simt launch");
}

}  // namespace tq
