// Decode attention from the packed caches: o = softmax(scale * L) V_hat.
//
// "TurboQuant explained" (a2a-mcp.org), §How it works: the attention logits
// are computed from the compressed keys (the fused logit of §Stage 2) and the
// values are read back from their codes (§Stage 1).  This entry point chains
// the library's kernels on the caller's stream:
//   1. tq_logits into a scores buffer of the workspace (query preparation +
//      logits kernel);
//   2. softmax_rows_kernel: each (sequence, query head) row of the scores
//      becomes softmax weights over the valid positions, in place;
//   3. tq_dequant_values mode B with those weights (accumulate in the rotated
//      space, Pi^T once per query head).
// The fused form (one split-K pass with an online softmax) is the next step;
// this composition fixes the semantics and is the baseline it must beat.

#include <cmath>

#include "tq_internal.cuh"

namespace tqd {

constexpr int kSmaxThreads = 1024;
constexpr int kSmaxUnroll = 8;      // independent loads in flight per thread

// Online (max, sum of exp) pair of two partial rows.
__device__ __forceinline__ void smax_merge(float& m, float& l, float m2, float l2) {
  if (m2 > m) {
    l = l * expf(m - m2) + l2;       // expf(-inf) = 0 when m = -inf
    m = m2;
  } else if (m2 > -INFINITY) {
    l += l2 * expf(m2 - m);
  }
}

// One CTA per row (sequence b, query head): the scores s[t] for t < ctx_len[b]
// become exp(scale s[t] - max) / sum, in place; positions past the context are
// left as they are (the value pass does not read them).  Each thread reads
// kSmaxUnroll scores per step, all loads in flight before any is used.
__global__ void __launch_bounds__(kSmaxThreads) softmax_rows_kernel(float* s, const int32_t* ctx_len, int n_q_heads,
                                                                    int64_t stride, int max_ctx, float scale) {
  constexpr int kStep = kSmaxThreads * kSmaxUnroll;
  __shared__ float sm[kSmaxThreads / 32], sl[kSmaxThreads / 32];
  const int64_t row = blockIdx.x;
  const int b = (int)(row / n_q_heads);
  const int n = max(0, min(ctx_len[b], max_ctx));
  float* x = s + row * stride;
  float m = -INFINITY, l = 0.0f;
  for (int t0 = threadIdx.x; t0 < n; t0 += kStep) {
    float v[kSmaxUnroll];
#pragma unroll
    for (int i = 0; i < kSmaxUnroll; ++i) {
      const int t = t0 + i * kSmaxThreads;
      v[i] = t < n ? scale * x[t] : -INFINITY;
    }
#pragma unroll
    for (int i = 0; i < kSmaxUnroll; ++i)
      if (v[i] > -INFINITY) smax_merge(m, l, v[i], 1.0f);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), l2 = __shfl_xor_sync(0xffffffffu, l, o);
    smax_merge(m, l, m2, l2);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    sm[warp] = m;
    sl[warp] = l;
  }
  __syncthreads();
  m = sm[0];
  l = sl[0];
#pragma unroll
  for (int w = 1; w < kSmaxThreads / 32; ++w) smax_merge(m, l, sm[w], sl[w]);
  const float inv = l > 0.0f ? 1.0f / l : 0.0f;
  for (int t0 = threadIdx.x; t0 < n; t0 += kStep) {
    float v[kSmaxUnroll];
#pragma unroll
    for (int i = 0; i < kSmaxUnroll; ++i) {
      const int t = t0 + i * kSmaxThreads;
      v[i] = t < n ? x[t] : 0.0f;
    }
#pragma unroll
    for (int i = 0; i < kSmaxUnroll; ++i) {
      const int t = t0 + i * kSmaxThreads;
      if (t < n) x[t] = expf(scale * v[i] - m) * inv;
    }
  }
}

}  // namespace tqd

namespace tq {

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
  return attend_ws_layout(kcb, vcb, batch, n_kv_heads, n_q_heads, max_ctx).total;
}

tq_status launch_attend(const tq_codebook* kcb, const CacheView& kcv, const tq_codebook* vcb, const CacheView& vcv,
                        const void* q, tq_dtype dt, int64_t batch, int n_q_heads, const int32_t* ctx_len,
                        int64_t max_ctx, float scale, float* out, void* ws, size_t ws_bytes, cudaStream_t st) {
  const AttendWs w = attend_ws_layout(kcb, vcb, batch, kcv.n_kv_heads, n_q_heads, max_ctx);
  if (!ws || ws_bytes < w.total) return fail(TQ_EINVAL, "tq_attend: workspace too small");
  if (batch == 0) return TQ_OK;
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  float* scores = reinterpret_cast<float*>(base);
  if (max_ctx > 0) {
    tq_status s = launch_logits(kcb, kcv, q, dt, batch, n_q_heads, ctx_len, max_ctx, scores, max_ctx,
                                base + w.scores, w.logits, st);
    if (s != TQ_OK) return s;
    if (batch * n_q_heads > 0x7fffffffLL) return fail(TQ_EINVAL, "tq_attend: batch * n_q_heads too large");
    tqd::softmax_rows_kernel<<<(unsigned)(batch * n_q_heads), tqd::kSmaxThreads, 0, st>>>(
        scores, ctx_len, n_q_heads, max_ctx, (int)max_ctx, scale);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "tq_attend: softmax launch");
  }
  // the value pass writes every output row when max_ctx > 0 (zeros where
  // ctx_len is 0)
  return launch_values(vcb, vcv, scores, max_ctx, batch, n_q_heads, ctx_len, max_ctx, out, TQ_F32,
                       vcb->lay.d, base + w.scores + w.logits, w.values, st);
}

}  // namespace tq
