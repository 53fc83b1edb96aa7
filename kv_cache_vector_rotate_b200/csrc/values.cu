// Value path from packed records: v_hat = ||v|| Pi^T c16[idx].
//
// "TurboQuant explained" (a2a-mcp.org), §Stage 1: the MSE stage alone codes
// the values; reconstruction is the centroid vector rotated back.
//  * mode A writes v_hat for every token;
//  * mode B forms o_h = sum_t w_{h,t} v_hat_t for the query heads of a KV head.
//    The sum is accumulated in the rotated space (acc_h = sum_t w_{h,t}
//    ||v_t|| c16[idx_t]) and rotated back once per head (o_h = Pi^T acc_h),
//    so the per-token work is a decode and G multiply-adds per coordinate.
//    Partial sums of context chunks go to the workspace; a second kernel adds
//    them and applies Pi^T.

#include "pack.cuh"

namespace tqd {

struct ValuesParams {
  tq::CacheView cv;
  const int32_t* ctx_len;
  int n_kv_heads, n_q_heads, G;
  int d;
  const float* pi32;        // [d_pad][d]
  const float* cent32;      // [2^b]
  const float* w;           // mode B weights
  int64_t w_stride;
  void* out;
  tq_dtype odt;
  int64_t out_stride;
  float* partial;           // mode B: [chunks][groups][G][d_pad]
  int tokens_per_cta;
  int n_chunks;
  int max_ctx;              // ctx_len values are clamped to [0, max_ctx]
};

// Level index of local element l of a chunk (layout version 3).
template <int BITS, int E>
__device__ __forceinline__ int unpack_index(const uint32_t* w, int l) {
  uint32_t code = 0u;
  if (BITS == 3 && l / 32 < E / 32 && l % 32 >= 24) {
#pragma unroll
    for (int k = 0; k < 3; ++k) code |= ((w[code_word<BITS, E>(l, k)] >> code_bit<BITS, E>(l, k)) & 1u) << k;
  } else {
    code = (w[code_word<BITS, E>(l, 0)] >> code_bit<BITS, E>(l, 0)) & ((1u << BITS) - 1u);
  }
  return level_index<BITS>(code);
}

// Stages 16 tokens: cs[tok][j] = ||v|| c16[idx_j] (0 past the context or for
// an unusable page).  128 threads: 8 threads per token, each decoding every
// 8th coordinate.
template <int BITS, int E>
__device__ __forceinline__ void stage_tokens(const ValuesParams& p, int b, int h, int base, int ctx,
                                             float (*cs)[4 * E + 1], const float* sc) {
  constexpr int W = ChunkWords<BITS, E, 0>::W;
  constexpr int CB = 16 * W;
  const int tok = threadIdx.x >> 3, sub = threadIdx.x & 7;
  const int pos = base + tok;
  bool ok = pos < ctx;
  const uint8_t* hb = nullptr;
  if (ok) {
    const int64_t page = p.cv.block_table[(int64_t)b * p.cv.max_pages + pos / p.cv.page_tokens];
    if (page < 0 || page >= p.cv.n_pages) {
      if (sub == 0) report(p.cv.err, TQ_DEV_ERR_PAGE);
      ok = false;
    } else {
      hb = p.cv.pages + page * p.cv.page_bytes + (int64_t)h * p.cv.head_block_bytes;
    }
  }
  const int slot = pos % p.cv.page_tokens;
  float nrm = 0.0f;
  if (ok) nrm = __half2float(*reinterpret_cast<const __half*>(hb + (int64_t)p.cv.page_tokens * CB + slot * 2));
  for (int j = sub; j < 4 * E; j += 8) {
    float v = 0.0f;
    if (ok && j < p.d) {
      const uint32_t* cw = reinterpret_cast<const uint32_t*>(hb + (int64_t)slot * CB) + (j / E) * W;
      v = nrm * sc[unpack_index<BITS, E>(cw, j % E)];
    }
    cs[tok][j] = v;
  }
}

// Mode A.  grid: (ceil(max_ctx / 16), batch * n_kv_heads); block 128.
template <int BITS, int E>
__global__ void __launch_bounds__(128) dequant_kernel(ValuesParams p) {
  constexpr int DP = 4 * E;
  __shared__ float cs[16][DP + 1];
  __shared__ float sc[16];
  const int gi = blockIdx.y, b = gi / p.n_kv_heads, h = gi % p.n_kv_heads;
  const int ctx = min(p.ctx_len[b], p.max_ctx);
  const int base = blockIdx.x * 16;
  if (base >= ctx) return;
  if (threadIdx.x < (1 << BITS)) sc[threadIdx.x] = p.cent32[threadIdx.x];
  __syncthreads();
  stage_tokens<BITS, E>(p, b, h, base, ctx, cs, sc);
  __syncthreads();
  const int d = p.d;
  for (int k = threadIdx.x; k < d; k += 128) {
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
    for (int j = 0; j < d; ++j) {
      const float pk = __ldg(p.pi32 + (size_t)j * d + k);   // (Pi^T)_{k j}
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = fmaf(pk, cs[i][j], acc[i]);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int pos = base + i;
      if (pos >= ctx) break;
      const int64_t o = (((int64_t)gi) * p.out_stride + pos) * d + k;
      if (p.odt == TQ_F32) reinterpret_cast<float*>(p.out)[o] = acc[i];
      else if (p.odt == TQ_BF16) reinterpret_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(acc[i]);
      else reinterpret_cast<__half*>(p.out)[o] = __float2half_rn(acc[i]);
    }
  }
}

// Mode B, pass 1.  grid: (n_chunks, batch * n_kv_heads); block 128.
// Dynamic shared memory: acc [G][4E] floats and weights [16][G].
template <int BITS, int E>
__global__ void __launch_bounds__(128) accumulate_kernel(ValuesParams p) {
  constexpr int DP = 4 * E;
  __shared__ float cs[16][DP + 1];
  __shared__ float sc[16];
  extern __shared__ float dyn[];
  const int G = p.G;
  float* acc = dyn;                 // [G][DP]
  float* ws = dyn + G * DP;         // [16][G]
  const int gi = blockIdx.y, b = gi / p.n_kv_heads, h = gi % p.n_kv_heads;
  const int ctx = min(p.ctx_len[b], p.max_ctx);
  const int k0 = blockIdx.x * p.tokens_per_cta;
  const int k1 = min(k0 + p.tokens_per_cta, ctx);
  for (int i = threadIdx.x; i < G * DP; i += 128) acc[i] = 0.0f;
  if (threadIdx.x < (1 << BITS)) sc[threadIdx.x] = p.cent32[threadIdx.x];
  __syncthreads();
  for (int base = k0; base < k1; base += 16) {
    stage_tokens<BITS, E>(p, b, h, base, k1, cs, sc);
    for (int i = threadIdx.x; i < 16 * G; i += 128) {
      const int tok = i / G, hh = i % G;
      const int pos = base + tok;
      ws[i] = pos < k1 ? __ldg(p.w + ((int64_t)b * p.n_q_heads + h * G + hh) * p.w_stride + pos) : 0.0f;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < DP; j += 128) {
      for (int hh = 0; hh < G; ++hh) {
        float a = acc[hh * DP + j];
#pragma unroll
        for (int tok = 0; tok < 16; ++tok) a = fmaf(ws[tok * G + hh], cs[tok][j], a);
        acc[hh * DP + j] = a;
      }
    }
    __syncthreads();
  }
  float* dst = p.partial + (((int64_t)blockIdx.x * gridDim.y + gi) * G) * DP;
  for (int i = threadIdx.x; i < G * DP; i += 128) dst[i] = acc[i];
}

// Mode B, pass 2: sum the chunk partials and rotate back, o = Pi^T acc.
// grid: (batch * n_q_heads); block 128.
template <int E>
__global__ void __launch_bounds__(128) finish_kernel(ValuesParams p) {
  constexpr int DP = 4 * E;
  __shared__ float a[DP];
  const int qrow = blockIdx.x;
  const int b = qrow / p.n_q_heads, hq = qrow % p.n_q_heads;
  const int h = hq / p.G, hh = hq % p.G;
  const int gi = b * p.n_kv_heads + h;
  const int groups = gridDim.x / p.n_q_heads * p.n_kv_heads;
  for (int j = threadIdx.x; j < DP; j += 128) {
    float s = 0.0f;
    for (int c = 0; c < p.n_chunks; ++c)
      s += p.partial[(((int64_t)c * groups + gi) * p.G + hh) * DP + j];
    a[j] = s;
  }
  __syncthreads();
  const int d = p.d;
  float* o = reinterpret_cast<float*>(p.out) + (int64_t)qrow * d;
  for (int k = threadIdx.x; k < d; k += 128) {
    float s = 0.0f;
    for (int j = 0; j < d; ++j) s = fmaf(__ldg(p.pi32 + (size_t)j * d + k), a[j], s);
    o[k] = s;
  }
}

}  // namespace tqd

namespace tq {

static int values_chunks(int64_t groups, int64_t max_ctx, int* tokens_per_cta) {
  int64_t target = 2 * 148;
  int64_t chunks = (target + groups - 1) / groups;
  int64_t tpc = (max_ctx + chunks - 1) / chunks;
  tpc = ((tpc + 15) / 16) * 16;
  if (tpc < 16) tpc = 16;
  *tokens_per_cta = (int)tpc;
  return (int)((max_ctx + tpc - 1) / tpc);
}

size_t values_workspace(const tq_codebook* cb, int64_t batch, int n_kv_heads, int n_q_heads,
                        int64_t max_ctx) {
  if (n_kv_heads <= 0 || n_q_heads <= 0 || max_ctx <= 0) return 0;
  int tpc;
  const int64_t groups = batch * n_kv_heads;
  const int chunks = values_chunks(groups, max_ctx, &tpc);
  const int G = n_q_heads / n_kv_heads;
  return (size_t)chunks * groups * G * cb->lay.d_pad * sizeof(float);
}

template <int BITS, int E>
static tq_status run_values(tqd::ValuesParams p, int64_t batch, int64_t max_ctx, bool mode_b,
                            cudaStream_t st) {
  const int64_t groups = batch * p.n_kv_heads;
  if (!mode_b) {
    dim3 grid((unsigned)((max_ctx + 15) / 16), (unsigned)groups);
    tqd::dequant_kernel<BITS, E><<<grid, 128, 0, st>>>(p);
    return TQ_OK;
  }
  const size_t dyn = ((size_t)p.G * 4 * E + 16 * p.G) * sizeof(float);
  if (dyn > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(tqd::accumulate_kernel<BITS, E>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
    if (e != cudaSuccess) return cuda_fail(e, "values: smem attribute");
  }
  dim3 grid((unsigned)p.n_chunks, (unsigned)groups);
  tqd::accumulate_kernel<BITS, E><<<grid, 128, dyn, st>>>(p);
  tqd::finish_kernel<E><<<(unsigned)(batch * p.n_q_heads), 128, 0, st>>>(p);
  return TQ_OK;
}

template <int BITS>
static int dispatch_values(const Layout& L, const tqd::ValuesParams& p, int64_t batch,
                           int64_t max_ctx, bool mode_b, cudaStream_t st, tq_status* s) {
  switch (L.E) {
    case 16: *s = run_values<BITS, 16>(p, batch, max_ctx, mode_b, st); return 1;
    case 32: *s = run_values<BITS, 32>(p, batch, max_ctx, mode_b, st); return 1;
    case 48: *s = run_values<BITS, 48>(p, batch, max_ctx, mode_b, st); return 1;
    case 64: *s = run_values<BITS, 64>(p, batch, max_ctx, mode_b, st); return 1;
  }
  return 0;
}

tq_status launch_values(const tq_codebook* cb, const CacheView& cv, const float* w,
                        int64_t w_stride, int64_t batch, int n_q_heads, const int32_t* ctx_len,
                        int64_t max_ctx, void* out, tq_dtype odt, int64_t out_stride, void* ws,
                        size_t ws_bytes, cudaStream_t st) {
  const Layout& L = cb->lay;
  if (L.m != 0) return fail(TQ_EUNSUPPORTED, "tq_dequant_values: values codebooks have m = 0");
  const bool mode_b = w != nullptr;
  if (max_ctx == 0 || batch == 0) return TQ_OK;
  tqd::ValuesParams p;
  p.cv = cv;
  p.ctx_len = ctx_len;
  p.n_kv_heads = cv.n_kv_heads;
  p.n_q_heads = n_q_heads;
  p.G = mode_b ? n_q_heads / cv.n_kv_heads : 1;
  p.d = L.d;
  p.pi32 = cb->pi32;
  p.cent32 = cb->cent32;
  p.w = w;
  p.w_stride = w_stride;
  p.out = out;
  p.odt = odt;
  p.out_stride = out_stride;
  p.partial = reinterpret_cast<float*>(ws);
  p.n_chunks = values_chunks(batch * cv.n_kv_heads, max_ctx, &p.tokens_per_cta);
  p.max_ctx = (int)max_ctx;
  if (mode_b && ws_bytes < values_workspace(cb, batch, cv.n_kv_heads, n_q_heads, max_ctx))
    return fail(TQ_EINVAL, "tq_dequant_values: workspace too small");
  tq_status s = TQ_OK;
  int ok = 0;
  switch (L.bits) {
    case 1: ok = dispatch_values<1>(L, p, batch, max_ctx, mode_b, st, &s); break;
    case 2: ok = dispatch_values<2>(L, p, batch, max_ctx, mode_b, st, &s); break;
    case 3: ok = dispatch_values<3>(L, p, batch, max_ctx, mode_b, st, &s); break;
    case 4: ok = dispatch_values<4>(L, p, batch, max_ctx, mode_b, st, &s); break;
  }
  if (!ok) return fail(TQ_EUNSUPPORTED, "tq_dequant_values: no kernel for this d");
  if (s != TQ_OK) return s;
  return cuda_fail(cudaGetLastError(), "tq_dequant_values launch");
}

}  // namespace tq
