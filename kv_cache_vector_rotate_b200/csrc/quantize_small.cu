// Quantize-and-append for the small appends of a decode step (head_dim 128).
//
// "TurboQuant explained" (a2a-mcp.org) §Stage 1: normalize, rotate by Pi,
// map each rotated coordinate to its Lloyd-Max cell; §Stage 2: signs of a
// Gaussian projection of the residual; §How to implement: quantize on every
// cache update.  A decode step appends one token per KV head, so the work
// per call is a few matrix-vector products: on one SM it would be bound by
// reading the 128 KB of Pi and S Pi^T into that SM.  Here each vector gets a
// cluster of 8 CTAs on 8 SMs; CTA c reads only rows [16 c, 16 c + 16) of Pi
// and of S_rot = S Pi^T (16 KB), computes those 16 rotated coordinates
// (codes and residual) and, once every CTA of the cluster has sent its part
// of the residual through distributed shared memory, those 16 rows of the
// sketch.  Code and sign bits are ORed into CTA 0's record words, which CTA
// 0 stores with the norm slot.  The records are those the other quantize
// kernels write (up to fp32 summation order inside the cells' 1e-5 window).

#include "pack.cuh"

namespace tqd {

constexpr int kSmCluster = 8;        // CTAs per vector
constexpr int kSmThreads = 128;      // 16 output rows x 8 threads (16 columns each)
constexpr int kSmMaxRows = 256;      // larger appends go to the other kernels

struct QuantizeSmallParams {
  const void* x;
  tq_dtype dtype;
  int64_t rows, n_new;       // rows = batch * n_kv_heads * n_new
  int n_kv_heads;
  const int32_t* start_pos;
  tq::CacheView cv;
  const float* pi32;         // [128][128] Pi, row-major
  const float* srot32;       // [128][128] S Pi^T, row-major (m_pad = 128)
  const float* bound32;
  const float* cent32;
};

__device__ __forceinline__ uint32_t sm_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t sm_map(const void* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(remote) : "r"((uint32_t)__cvta_generic_to_shared(local)), "r"(rank));
  return remote;
}
__device__ __forceinline__ void sm_remote_or(uint32_t addr, uint32_t v) {
  asm volatile("atom.shared::cluster.or.b32 _, [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void sm_remote_st(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void sm_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void sm_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// One vector (row) by one cluster of 8 CTAs of 128 threads.  Thread (o, q) =
// (tid / 8, tid % 8) takes rotated coordinate j = 16 c + o and sketch row
// i = 16 c + o, over columns [16 q, 16 q + 16).
template <int BITS, int F>
__device__ __forceinline__ void quantize_small_row(const QuantizeSmallParams& p, int64_t row) {
  constexpr int E = 32;
  constexpr int K = 1 << BITS;
  using CW = ChunkWords<BITS, E, F>;
  constexpr int W = CW::W;
  __shared__ uint32_t wsm[4 * W];      // CTA 0: the record words
  __shared__ float rfull[128];         // the whole residual (rotated space)
  __shared__ float rn2[kSmCluster];    // CTA 0: per-CTA sums of squares of the residual
  __shared__ float sb[16], sc[16];
  const int tid = threadIdx.x, o = tid >> 3, q = tid & 7;
  const uint32_t c = sm_cluster_rank();
  const int j = 16 * (int)c + o;

  // every operand load first: x columns, this row of Pi (and of S_rot)
  float xk[16], pk[16], sk[16];
  {
    const int64_t xo = row * 128 + 16 * q;
    if (p.dtype == TQ_F32) {
      const float4* xs = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.x) + xo);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = __ldg(xs + i);
        xk[4 * i] = v.x; xk[4 * i + 1] = v.y; xk[4 * i + 2] = v.z; xk[4 * i + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) xk[i] = load_elem(p.x, xo + i, p.dtype);
    }
    const float4* ps = reinterpret_cast<const float4*>(p.pi32 + (size_t)j * 128 + 16 * q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldg(ps + i);
      pk[4 * i] = v.x; pk[4 * i + 1] = v.y; pk[4 * i + 2] = v.z; pk[4 * i + 3] = v.w;
    }
    if constexpr (F > 0) {
      const float4* ss = reinterpret_cast<const float4*>(p.srot32 + (size_t)j * 128 + 16 * q);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = __ldg(ss + i);
        sk[4 * i] = v.x; sk[4 * i + 1] = v.y; sk[4 * i + 2] = v.z; sk[4 * i + 3] = v.w;
      }
    }
  }
  if (tid < K) sc[tid] = p.cent32[tid];
  if (tid < K - 1) sb[tid + 1] = p.bound32[tid];
  if (tid == 0) sb[0] = 0.0f;
  if (c == 0 && tid < 4 * W) wsm[tid] = 0u;
  __syncthreads();
  sm_arrive_release();                 // phase 0: CTA 0's words are zero, every CTA has started

  // ||x||^2 and y_j over the 8 threads of the row group
  float n2 = 0.0f, y = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    n2 = fmaf(xk[i], xk[i], n2);
    y = fmaf(pk[i], xk[i], y);
  }
#pragma unroll
  for (int s = 1; s < 8; s <<= 1) {
    n2 += __shfl_xor_sync(0xffffffffu, n2, s);
    y += __shfl_xor_sync(0xffffffffu, y, s);
  }
  const float nrm = sqrtf(n2);
  const float u = y * (nrm > 0.0f ? 1.0f / nrm : 0.0f);
  int idx = 0;
#pragma unroll
  for (int step = K / 2; step >= 1; step >>= 1)
    if (u >= sb[idx + step]) idx += step;
  const float res = u - sc[idx];
  // sum of squares of this CTA's 16 residuals (one value per row group)
  float r2 = q == 0 ? res * res : 0.0f;
#pragma unroll
  for (int s = 8; s < 32; s <<= 1) r2 += __shfl_xor_sync(0xffffffffu, r2, s);

  sm_wait_acquire();                   // phase 0 complete: remote shared memory may be written
  // the residual to every CTA (thread q of the group to CTA q), the code bits to CTA 0
  sm_remote_st(sm_map(&rfull[j], (uint32_t)q), res);
  if (q == 0) {
    const uint32_t code = stored_code<BITS>(idx);
    const int t = j / E, l = j % E;
#pragma unroll
    for (int kb = 0; kb < (BITS == 4 ? 4 : BITS); ++kb) {
      const uint32_t bit = ((code >> kb) & 1u) << code_bit<BITS, E>(l, kb);
      if (bit) sm_remote_or(sm_map(&wsm[t * W + code_word<BITS, E>(l, kb)], 0), bit);
    }
  }
  __shared__ float wr2[4];
  if ((tid & 31) == 0) wr2[tid >> 5] = r2;
  __syncthreads();
  if (tid == 0) sm_remote_st(sm_map(&rn2[c], 0), (wr2[0] + wr2[1]) + (wr2[2] + wr2[3]));
  sm_arrive_release();
  sm_wait_acquire();                   // phase 1: the residual, code bits and sums delivered

  if constexpr (F > 0) {
    // sketch row i = j: sign of (S_rot r)_i
    float pv = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) pv = fmaf(sk[i], rfull[16 * q + i], pv);
#pragma unroll
    for (int s = 1; s < 8; s <<= 1) pv += __shfl_xor_sync(0xffffffffu, pv, s);
    if (q == 0 && pv < 0.0f) {
      const int t = j / F, l = j % F;
      sm_remote_or(sm_map(&wsm[t * W + CW::q0 + l / 32], 0), 1u << qjl_bit(l));
    }
  }
  sm_arrive_release();
  sm_wait_acquire();                   // phase 2: every bit in CTA 0; no remote access after this

  if (c == 0) {
    const int64_t per_seq = (int64_t)p.n_kv_heads * p.n_new;
    const int64_t b = row / per_seq;
    const int h = (int)((row / p.n_new) % p.n_kv_heads);
    const int64_t pos = p.start_pos[b] + row % p.n_new;
    const int64_t hb = head_block_offset(p.cv, b, h, pos);
    if (hb >= 0) {
      const int slot = (int)(pos % p.cv.page_tokens);
      uint32_t* rec = reinterpret_cast<uint32_t*>(p.cv.pages + hb + (int64_t)slot * 16 * W);
      if (tid < 4 * W) rec[tid] = wsm[tid];
      if (tid == 0) {
        const __half nh = __float2half_rn(nrm);
        if (__hisinf(nh)) report(p.cv.err, TQ_DEV_ERR_RANGE);
        __half* ns = reinterpret_cast<__half*>(p.cv.pages + hb + (int64_t)p.cv.page_tokens * 16 * W +
                                               (int64_t)slot * (F > 0 ? 4 : 2));
        ns[0] = nh;
        if constexpr (F > 0) {
          float t2 = 0.0f;
#pragma unroll
          for (int i = 0; i < kSmCluster; ++i) t2 += rn2[i];
          ns[1] = __float2half_rn(sqrtf(t2));
        }
      }
    }
  }
}

// grid: 8 x rows CTAs in clusters of 8 (cluster = vector blockIdx.x / 8), block 128.
template <int BITS, int F>
__global__ void __cluster_dims__(kSmCluster, 1, 1) __launch_bounds__(kSmThreads)
    quantize_small_kernel(QuantizeSmallParams p) {
  // a programmatic dependent of the previous kernel: nothing is read before it finishes
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  quantize_small_row<BITS, F>(p, blockIdx.x / kSmCluster);
}

// Keys (with the sketch) and values (without) of a decode step in one launch:
// clusters [0, pk.rows) code keys, the next pv.rows clusters code values.
template <int KB, int VB>
__global__ void __cluster_dims__(kSmCluster, 1, 1) __launch_bounds__(kSmThreads)
    quantize_small_kv_kernel(QuantizeSmallParams pk, QuantizeSmallParams pv) {
  asm volatile("griddepcontrol.wait;" ::: "memory");   // as quantize_small_kernel
  asm volatile("griddepcontrol.launch_dependents;");
  const int64_t v = blockIdx.x / kSmCluster;       // cluster-uniform
  if (v < pk.rows) quantize_small_row<KB, 32>(pk, v);
  else quantize_small_row<VB, 0>(pv, v - pk.rows);
}

}  // namespace tqd

namespace tq {

// A launch on `st` that may start while the previous kernel finishes (the
// kernels wait for it before touching memory).
template <class... KArgs, class... Args>
static void launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  (void)cudaLaunchKernelEx(&cfg, kern, args...);   // errors are read by the caller (cudaGetLastError)
}

// head_dim 128 (d_pad 128, m 0 or m_pad 128), up to kSmMaxRows vectors, rows
// of f32 16-byte aligned; everything else goes to the other kernels.
tq_status launch_quantize_small(const tq_codebook* cb, const void* x, tq_dtype dt, int64_t batch,
                                int n_kv_heads, int64_t n_new, const int32_t* start_pos,
                                const CacheView& cv, cudaStream_t st, bool* handled) {
  const Layout& L = cb->lay;
  *handled = false;
  const int64_t rows = batch * n_kv_heads * n_new;
  if (L.d != 128 || L.d_pad != 128 || !(L.m_pad == 0 || L.m_pad == 128) || rows < 1 ||
      rows > tqd::kSmMaxRows || (dt == TQ_F32 && (reinterpret_cast<uintptr_t>(x) & 15u) != 0))
    return TQ_OK;
  tqd::QuantizeSmallParams p;
  p.x = x;
  p.dtype = dt;
  p.rows = rows;
  p.n_new = n_new;
  p.n_kv_heads = n_kv_heads;
  p.start_pos = start_pos;
  p.cv = cv;
  p.pi32 = cb->pi32;
  p.srot32 = cb->srot32;
  p.bound32 = cb->bound32;
  p.cent32 = cb->cent32;
  const dim3 grid((unsigned)(rows * tqd::kSmCluster));
  const bool q = L.m_pad == 128;
  switch (L.bits) {
    case 1:
      if (q) launch_dependent(tqd::quantize_small_kernel<1, 32>, grid, dim3(tqd::kSmThreads), st, p);
      else launch_dependent(tqd::quantize_small_kernel<1, 0>, grid, dim3(tqd::kSmThreads), st, p);
      break;
    case 2:
      if (q) launch_dependent(tqd::quantize_small_kernel<2, 32>, grid, dim3(tqd::kSmThreads), st, p);
      else launch_dependent(tqd::quantize_small_kernel<2, 0>, grid, dim3(tqd::kSmThreads), st, p);
      break;
    case 3:
      if (q) launch_dependent(tqd::quantize_small_kernel<3, 32>, grid, dim3(tqd::kSmThreads), st, p);
      else launch_dependent(tqd::quantize_small_kernel<3, 0>, grid, dim3(tqd::kSmThreads), st, p);
      break;
    case 4:
      if (q) launch_dependent(tqd::quantize_small_kernel<4, 32>, grid, dim3(tqd::kSmThreads), st, p);
      else launch_dependent(tqd::quantize_small_kernel<4, 0>, grid, dim3(tqd::kSmThreads), st, p);
      break;
    default: return TQ_OK;
  }
  *handled = true;
  return cuda_fail(cudaGetLastError(), "quantize_small launch");
}

// Keys and values of the same shape in one launch: both codebooks d = 128,
// keys with m_pad = 128 and values with m = 0, up to kSmMaxRows vectors each.
// *handled = false when the shapes do not qualify (nothing launched).
tq_status launch_quantize_small_kv(const tq_codebook* kcb, const void* k, const tq_codebook* vcb, const void* v,
                                   tq_dtype dt, int64_t batch, int n_kv_heads, int64_t n_new,
                                   const int32_t* start_pos, const CacheView& kcv, const CacheView& vcv,
                                   cudaStream_t st, bool* handled) {
  const Layout &K = kcb->lay, &V = vcb->lay;
  *handled = false;
  const int64_t rows = batch * n_kv_heads * n_new;
  const bool f32_ok = dt != TQ_F32 || ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15u) == 0;
  if (K.d != 128 || K.d_pad != 128 || K.m_pad != 128 || V.d != 128 || V.d_pad != 128 || V.m_pad != 0 || rows < 1 ||
      rows > tqd::kSmMaxRows || !f32_ok)
    return TQ_OK;
  auto fill = [&](const tq_codebook* cb, const void* x, const CacheView& cv) {
    tqd::QuantizeSmallParams p;
    p.x = x;
    p.dtype = dt;
    p.rows = rows;
    p.n_new = n_new;
    p.n_kv_heads = n_kv_heads;
    p.start_pos = start_pos;
    p.cv = cv;
    p.pi32 = cb->pi32;
    p.srot32 = cb->srot32;
    p.bound32 = cb->bound32;
    p.cent32 = cb->cent32;
    return p;
  };
  const tqd::QuantizeSmallParams pk = fill(kcb, k, kcv), pv = fill(vcb, v, vcv);
  const dim3 grid((unsigned)(2 * rows * tqd::kSmCluster));
#define TQ_KV(KB_, VB_) \
  if (K.bits == KB_ && V.bits == VB_) \
    launch_dependent(tqd::quantize_small_kv_kernel<KB_, VB_>, grid, dim3(tqd::kSmThreads), st, pk, pv);
#define TQ_KV_ROW(KB_) TQ_KV(KB_, 1) else TQ_KV(KB_, 2) else TQ_KV(KB_, 3) else TQ_KV(KB_, 4)
  TQ_KV_ROW(1) else TQ_KV_ROW(2) else TQ_KV_ROW(3) else TQ_KV_ROW(4) else return TQ_OK;
#undef TQ_KV_ROW
#undef TQ_KV
  *handled = true;
  return cuda_fail(cudaGetLastError(), "quantize_small_kv launch");
}

}  // namespace tq
