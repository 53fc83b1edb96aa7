// Decode attention from the packed caches: o = softmax(scale * L) V_hat.
//
// "TurboQuant explained" (a2a-mcp.org), §How it works: the attention logits
// are computed from the compressed keys (the fused logit of §Stage 2) and the
// values are read back from their codes (§Stage 1).
//
// d <= 128 with equal page sizes: the fused split-K pass (attend_fused.cuh:
// query preparation, one pass over both caches with an online softmax, a
// finish kernel).  Otherwise this file's composition of the library's
// kernels on the caller's stream:
//   1. tq_logits into a scores buffer of the workspace (query preparation +
//      logits kernel);
//   2. softmax_rows_kernel: each (sequence, query head) row of the scores
//      becomes softmax weights over the valid positions, in place;
//   3. tq_dequant_values mode B with those weights (accumulate in the rotated
//      space, Pi^T once per query head).

#include <algorithm>
#include <cmath>

#include "attend_fused.cuh"

namespace tqd {

constexpr int kSmaxCluster = 8;    // CTAs per row, one eighth of the row each
constexpr int kSmaxThreads = 512;
constexpr int kSmaxUnroll = 8;     // independent loads in flight per thread

// Online (max, sum of exp) pair of two partial rows.
__device__ __forceinline__ void smax_merge(float& m, float& l, float m2, float l2) {
  if (m2 > m) {
    l = l * expf(m - m2) + l2;       // expf(-inf) = 0 when m = -inf
    m = m2;
  } else if (m2 > -INFINITY) {
    l += l2 * expf(m2 - m);
  }
}

__device__ __forceinline__ uint32_t smax_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// One cluster of kSmaxCluster CTAs per row (sequence b, query head): the
// scores s[t] for t < ctx_len[b] become exp(scale s[t] - max) / sum, in place;
// positions past the context are left as they are (the value pass does not
// read them).  CTA c reduces its segment of the row to a (max, sum) pair and
// stores it into slot c of every CTA of the cluster (distributed shared
// memory); after the cluster barrier each CTA merges the eight pairs and
// rewrites its segment, whose second read comes from L2.
__global__ void __cluster_dims__(kSmaxCluster, 1, 1) __launch_bounds__(kSmaxThreads)
    softmax_rows_kernel(float* s, const int32_t* ctx_len, int n_q_heads, int64_t stride, int max_ctx,
                        float scale) {
  constexpr int kStep = kSmaxThreads * kSmaxUnroll;
  __shared__ float wm[kSmaxThreads / 32], wl[kSmaxThreads / 32];
  __shared__ float pm[kSmaxCluster], pl[kSmaxCluster];
  // phase 0 opens: every CTA of the cluster has started before any remote store
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  const uint32_t c = smax_cluster_rank();
  const int64_t row = blockIdx.x / kSmaxCluster;
  const int b = (int)(row / n_q_heads);
  const int n = max(0, min(ctx_len[b], max_ctx));
  const int seg = ((n + kSmaxCluster - 1) / kSmaxCluster + 31) & ~31;
  const int lo = min(n, (int)c * seg), hi = min(n, lo + seg);
  float* x = s + row * stride;
  float m = -INFINITY, l = 0.0f;
  for (int t0 = lo + (int)threadIdx.x; t0 < hi; t0 += kStep) {
    float v[kSmaxUnroll];
#pragma unroll
    for (int i = 0; i < kSmaxUnroll; ++i) {
      const int t = t0 + i * kSmaxThreads;
      v[i] = t < hi ? scale * x[t] : -INFINITY;
    }
    float mv = v[0];
#pragma unroll
    for (int i = 1; i < kSmaxUnroll; ++i) mv = fmaxf(mv, v[i]);
    float lv = 0.0f;
#pragma unroll
    for (int i = 0; i < kSmaxUnroll; ++i) lv += expf(v[i] - mv);   // v[0] is finite: mv > -inf
    smax_merge(m, l, mv, lv);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), l2 = __shfl_xor_sync(0xffffffffu, l, o);
    smax_merge(m, l, m2, l2);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    wm[warp] = m;
    wl[warp] = l;
  }
  __syncthreads();
  m = wm[0];
  l = wl[0];
#pragma unroll
  for (int w = 1; w < kSmaxThreads / 32; ++w) smax_merge(m, l, wm[w], wl[w]);
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  if (threadIdx.x < kSmaxCluster) {
    uint32_t am, al;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                 : "=r"(am) : "r"((uint32_t)__cvta_generic_to_shared(&pm[c])), "r"((uint32_t)threadIdx.x));
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                 : "=r"(al) : "r"((uint32_t)__cvta_generic_to_shared(&pl[c])), "r"((uint32_t)threadIdx.x));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(am), "f"(m) : "memory");
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(al), "f"(l) : "memory");
  }
  // phase 1: every pair delivered; no remote access after this
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
  m = pm[0];
  l = pl[0];
#pragma unroll
  for (int r = 1; r < kSmaxCluster; ++r) smax_merge(m, l, pm[r], pl[r]);
  const float inv = l > 0.0f ? 1.0f / l : 0.0f;
  for (int t0 = lo + (int)threadIdx.x; t0 < hi; t0 += kStep) {
    float v[kSmaxUnroll];
#pragma unroll
    for (int i = 0; i < kSmaxUnroll; ++i) {
      const int t = t0 + i * kSmaxThreads;
      v[i] = t < hi ? x[t] : 0.0f;
    }
#pragma unroll
    for (int i = 0; i < kSmaxUnroll; ++i) {
      const int t = t0 + i * kSmaxThreads;
      if (t < hi) x[t] = expf(scale * v[i] - m) * inv;
    }
  }
}

}  // namespace tqd

namespace tq {

// The fused kernels, one translation unit per key width.
tq_status launch_attend_fused_k1(const tqd::AttendParams& p, int vbits, int E, int F, int lines, cudaStream_t st);
tq_status launch_attend_fused_k2(const tqd::AttendParams& p, int vbits, int E, int F, int lines, cudaStream_t st);
tq_status launch_attend_fused_k3(const tqd::AttendParams& p, int vbits, int E, int F, int lines, cudaStream_t st);
tq_status launch_attend_fused_k4(const tqd::AttendParams& p, int vbits, int E, int F, int lines, cudaStream_t st);
tqd::KeyTables key_tables(const tq_codebook* cb);

static bool fused_attend_ok(const tq_codebook* kcb, const tq_codebook* vcb, int kpt, int vpt) {
  const Layout &K = kcb->lay, &V = vcb->lay;
  return K.E <= 32 && K.E == V.E && (K.F == 0 || K.F == K.E) && kpt == vpt;
}

// Grid of the fused kernel: one CTA per SM at least, at least one per line,
// and few enough units per CTA that its block-table entries fit.
struct AttendGrid {
  int64_t lines, units, items, n_cta;
};
static AttendGrid attend_grid(int64_t batch, int n_kv_heads, int n_q_heads, int64_t max_ctx, int page_tokens) {
  AttendGrid gr;
  const int G = n_q_heads / n_kv_heads;
  gr.lines = batch * n_kv_heads * ((G + 3) / 4);
  gr.units = (max_ctx + 63) / 64;
  gr.items = gr.lines * gr.units;
  const int64_t max_upc = (int64_t)(tqd::kAttPages - 4) * page_tokens / 64;
  int64_t n = std::max<int64_t>(device_sm_count(), gr.lines);
  n = std::max(n, (gr.items + max_upc - 1) / max_upc);
  gr.n_cta = std::max<int64_t>(1, std::min(n, gr.items));
  return gr;
}

struct FusedWs {
  size_t prep, partial, total;
};
static FusedWs fused_ws_layout(const tq_codebook* kcb, int64_t batch, int n_kv_heads, int n_q_heads,
                               int64_t n_cta) {
  auto al = [](size_t n) { return (n + 255) / 256 * 256; };
  FusedWs w;
  w.prep = al(query_prep_workspace(kcb, batch, n_kv_heads, n_q_heads));
  w.partial = al((size_t)n_cta * 2 * 4 * (4 * kcb->lay.E + 2) * sizeof(float));
  w.total = w.prep + w.partial;
  return w;
}

static tq_status launch_attend_fused(const tq_codebook* kcb, const CacheView& kcv, const tq_codebook* vcb,
                                     const CacheView& vcv, const void* q, tq_dtype dt, int64_t batch,
                                     int n_q_heads, const int32_t* ctx_len, int64_t max_ctx, float scale,
                                     float* out, void* ws, size_t ws_bytes, cudaStream_t st) {
  const int nkv = kcv.n_kv_heads;
  const AttendGrid gr = attend_grid(batch, nkv, n_q_heads, max_ctx, kcv.page_tokens);
  const FusedWs w = fused_ws_layout(kcb, batch, nkv, n_q_heads, gr.n_cta);
  // every check before the first launch
  if (!ws || ws_bytes < w.total) return fail(TQ_EINVAL, "tq_attend: workspace too small");
  const int G = n_q_heads / nkv;
  if (batch * nkv > 65535 || gr.lines > 65535 || gr.items > 0x7fffffffLL || gr.lines * 4 > 0x7fffffffLL)
    return fail(TQ_EINVAL, "tq_attend: batch * heads * context too large");
  tqd::AttendParams p;
  p.kcv = kcv;
  p.vcv = vcv;
  int ps = 0;
  while ((1 << ps) < kcv.page_tokens) ++ps;
  p.page_shift = ps;
  p.ctx_len = ctx_len;
  p.n_kv_heads = nkv;
  p.n_q_heads = n_q_heads;
  p.G = G;
  p.qtiles = (G + 3) / 4;
  p.units = (int)gr.units;
  p.max_ctx = (int)max_ctx;
  p.n_cta = (int)gr.n_cta;
  p.per_cta = (int)(gr.items / gr.n_cta);
  p.extra = (int)(gr.items % gr.n_cta);
  p.div_u = tqd::make_fastdiv((uint32_t)gr.units);
  p.div_qtiles = tqd::make_fastdiv((uint32_t)p.qtiles);
  p.div_kv = tqd::make_fastdiv((uint32_t)nkv);
  p.sl2 = scale * 1.4426950408889634f;   // log2(e)
  p.kt = key_tables(kcb);
  {
    const uint16_t* T = vcb->lay.bits == 4 ? vcb->mag16 : vcb->cent16;   // 8 entries
    p.tlo0 = p.tlo1 = p.thi0 = p.thi1 = 0u;
    for (int i = 0; i < 4; ++i) {
      p.tlo0 |= (uint32_t)(T[i] & 0xFF) << (8 * i);
      p.tlo1 |= (uint32_t)(T[4 + i] & 0xFF) << (8 * i);
      p.thi0 |= (uint32_t)(T[i] >> 8) << (8 * i);
      p.thi1 |= (uint32_t)(T[4 + i] >> 8) << (8 * i);
    }
  }
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  p.partial = reinterpret_cast<float*>(base + w.prep);
  p.pi32 = vcb->pi32;
  p.out = out;
  p.d = kcb->lay.d;
  const int kb = kcb->lay.bits;
  if (kb < 1 || kb > 4 || vcb->lay.bits < 1 || vcb->lay.bits > 4) return fail(TQ_EUNSUPPORTED, "tq_attend: bits");
  PreparedQueries pq;
  tq_status s = launch_query_prep(kcb, q, dt, batch, nkv, n_q_heads, base, &pq, st);
  if (s != TQ_OK) return s;
  p.frag = pq.frag;
  p.qfrag = pq.qfrag;
  p.scal = pq.scal;
  const int E = kcb->lay.E, F = kcb->lay.F, vb = vcb->lay.bits, lines = (int)gr.lines;
  switch (kb) {
    case 1: return launch_attend_fused_k1(p, vb, E, F, lines, st);
    case 2: return launch_attend_fused_k2(p, vb, E, F, lines, st);
    case 3: return launch_attend_fused_k3(p, vb, E, F, lines, st);
    default: return launch_attend_fused_k4(p, vb, E, F, lines, st);
  }
}

struct AttendWs {
  size_t scores, logits, values, total;
};

static AttendWs attend_ws_layout(const tq_codebook* kcb, const tq_codebook* vcb, int64_t batch, int n_kv_heads,
                                 int n_q_heads, int64_t max_ctx) {
  auto al = [](size_t n) { return (n + 255) / 256 * 256; };
  AttendWs w;
  w.scores = al((size_t)batch * n_q_heads * max_ctx * sizeof(float));
  w.logits = al(logits_workspace(kcb, batch * n_kv_heads, n_q_heads / n_kv_heads));
  w.values = al(values_workspace(vcb, batch, n_kv_heads, n_q_heads, max_ctx));
  w.total = w.scores + w.logits + w.values;
  return w;
}

size_t attend_workspace(const tq_codebook* kcb, const tq_codebook* vcb, int64_t batch, int n_kv_heads,
                        int n_q_heads, int64_t max_ctx) {
  // the fused path needs equal page sizes, which only the call knows: the
  // workspace covers both paths
  size_t fused = 0;
  if (kcb->lay.E <= 32 && kcb->lay.E == vcb->lay.E && batch > 0 && max_ctx > 0) {
    size_t worst = 0;
    for (int pt = 16; pt <= 1024; pt *= 2) {   // the grid grows as pages shrink
      const AttendGrid gr = attend_grid(batch, n_kv_heads, n_q_heads, max_ctx, pt);
      worst = std::max(worst, fused_ws_layout(kcb, batch, n_kv_heads, n_q_heads, gr.n_cta).total);
    }
    fused = worst;
  }
  return std::max(fused, attend_ws_layout(kcb, vcb, batch, n_kv_heads, n_q_heads, max_ctx).total);
}

static tq_status launch_attend_composed(const tq_codebook* kcb, const CacheView& kcv, const tq_codebook* vcb,
                                        const CacheView& vcv, const void* q, tq_dtype dt, int64_t batch,
                                        int n_q_heads, const int32_t* ctx_len, int64_t max_ctx, float scale,
                                        float* out, void* ws, size_t ws_bytes, cudaStream_t st) {
  const AttendWs w = attend_ws_layout(kcb, vcb, batch, kcv.n_kv_heads, n_q_heads, max_ctx);
  if (!ws || ws_bytes < w.total) return fail(TQ_EINVAL, "tq_attend: workspace too small");
  if (batch == 0) return TQ_OK;
  // every check before the first launch
  if (batch * n_q_heads > 0x7fffffffLL / tqd::kSmaxCluster || max_ctx > 0x7fff0000LL)
    return fail(TQ_EINVAL, "tq_attend: batch * n_q_heads or max_ctx too large");
  {
    const int G = n_q_heads / kcv.n_kv_heads;
    const int64_t groups = batch * kcv.n_kv_heads;
    if (groups > 65535 || groups * ((G + 3) / 4) > 65535 || groups * ((G + 3) / 4) * 4 > 0x7fffffffLL)
      return fail(TQ_EINVAL, "tq_attend: batch * n_kv_heads too large");
  }
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  float* scores = reinterpret_cast<float*>(base);
  if (max_ctx > 0) {
    tq_status s = launch_logits(kcb, kcv, q, dt, batch, n_q_heads, ctx_len, max_ctx, scores, max_ctx,
                                base + w.scores, w.logits, st);
    if (s != TQ_OK) return s;
    tqd::softmax_rows_kernel<<<(unsigned)(batch * n_q_heads * tqd::kSmaxCluster), tqd::kSmaxThreads, 0, st>>>(
        scores, ctx_len, n_q_heads, max_ctx, (int)max_ctx, scale);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "tq_attend: softmax launch");
  }
  // the value pass writes every output row when max_ctx > 0 (zeros where
  // ctx_len is 0)
  return launch_values(vcb, vcv, scores, max_ctx, batch, n_q_heads, ctx_len, max_ctx, out, TQ_F32,
                       vcb->lay.d, base + w.scores + w.logits, w.values, st);
}

tq_status launch_attend(const tq_codebook* kcb, const CacheView& kcv, const tq_codebook* vcb, const CacheView& vcv,
                        const void* q, tq_dtype dt, int64_t batch, int n_q_heads, const int32_t* ctx_len,
                        int64_t max_ctx, float scale, float* out, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (batch == 0) return TQ_OK;
  if (max_ctx > 0 && fused_attend_ok(kcb, vcb, kcv.page_tokens, vcv.page_tokens))
    return launch_attend_fused(kcb, kcv, vcb, vcv, q, dt, batch, n_q_heads, ctx_len, max_ctx, scale, out, ws,
                               ws_bytes, st);
  return launch_attend_composed(kcb, kcv, vcb, vcv, q, dt, batch, n_q_heads, ctx_len, max_ctx, scale, out, ws,
                                ws_bytes, st);
}

}  // namespace tq
