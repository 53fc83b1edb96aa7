// Fused attention logits straight from the packed keys.
//
// "TurboQuant explained" (a2a-mcp.org), §Stage 2 and §How it works: the
// query is rotated once (Pi q) and sketched once (S q); every logit is then
//   L = ||k|| ( sum_j (Pi q)_j c16[idx_j] + sqrt(pi/2)/m ||r|| sum_i (S q)_i s_i )
// evaluated from the indices and sign bits without dequantizing the key.
//
// Design.  The two sums are dot products of a decoded key row with the
// query group that shares its KV head.  A warp takes 16 keys at a time, turns
// each key's bits into fp16 operand registers (the centroid magnitudes come
// out of a byte-permute of the magnitude table, the signs are OR-ed into bit
// 15), and runs m16n8k16 tensor-core MMAs against the query group held as
// fp16 hi + lo halves (4 queries x {hi, lo} = the 8 columns).  The operand
// never leaves registers, so HBM traffic is the 68-byte records plus the
// logits.  The per-coordinate fragment order is fixed by the record layout:
// thread t of a quad owns chunk t, i.e. the bits it loads are exactly the
// bits its A fragment needs.

#include "tq_internal.cuh"

namespace tqd {

// ---- query preparation ------------------------------------------------------
// Workspace: fragments uint2 [groups][qtiles][KS0 + KS1][32 lanes], then
// inverse scales float [batch * n_q_heads][2].

struct PrepParams {
  const void* q;
  tq_dtype dtype;
  int d, E, F;           // E, F: coordinates / QJL rows per chunk
  int n_q_heads, n_kv_heads, G, qtiles;
  const float* pi32;     // [d_pad][d]
  const float* s32;      // [m_pad][d]
  float s_row_norm_max;
  uint2* frag;
  float* inv_scale;
};

// One warp per (group, query tile, k-step) writes the 32 lane fragments of
// that k-step, zeros included (padding rows and query slots past G), so the
// workspace needs no clearing.  Lane (g, t) holds column g = 2 * query +
// {0: hi, 1: lo} at rows t * Ep + 4 ks + {0, 1} (first register) and
// {2, 3} (second register) of Pi q (codebook part) or S q (QJL part).
// grid: (groups * qtiles, KS0 + KS1); block 32.
__global__ void __launch_bounds__(32) prep_queries_kernel(PrepParams p) {
  const int lane = threadIdx.x;
  const int g = lane >> 2, t = lane & 3;
  const int gq = blockIdx.x;
  const int gi = gq / p.qtiles, qt = gq % p.qtiles;
  const int b = gi / p.n_kv_heads, kv = gi % p.n_kv_heads;
  const int KS0 = p.E / 4;
  const int ksg = blockIdx.y;
  const int part = ksg < KS0 ? 0 : 1;
  const int ks = part == 0 ? ksg : ksg - KS0;
  const int Ep = part == 0 ? p.E : p.F;
  const int ql = qt * 4 + (g >> 1);
  const int hl = g & 1;
  const int d = p.d;
  uint32_t regs[2] = {0u, 0u};
  if (ql < p.G) {
    const int hq = kv * p.G + ql;
    const int64_t qrow = (int64_t)b * p.n_q_heads + hq;
    float n2 = 0.0f;
    for (int k = 0; k < d; ++k) {
      const float v = load_elem(p.q, qrow * d + k, p.dtype);
      n2 = fmaf(v, v, n2);
    }
    // |(Pi q)_j| <= ||q|| and |(S q)_i| <= max_i ||S_i|| ||q||: a power-of-two
    // scale puts every entry below 2^14, so the fp16 hi part cannot overflow
    // and hi + lo keep about 22 significant bits.
    const float qn = sqrtf(n2);
    const float bound = part == 0 ? qn : qn * p.s_row_norm_max;
    int e = 0;
    if (bound > 0.0f) frexpf(bound, &e);
    const float scale = ldexpf(1.0f, 14 - e);
    if (t == 0 && ks == 0 && hl == 0) p.inv_scale[qrow * 2 + part] = 1.0f / scale;
    const float* M = part == 0 ? p.pi32 : p.s32;
    __half vals[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = t * Ep + 4 * ks + r;          // row of Pi (or S), padded rows are zero
      const float* mr = M + (size_t)i * d;
      float v = 0.0f;
      for (int k = 0; k < d; ++k) v = fmaf(__ldg(mr + k), load_elem(p.q, qrow * d + k, p.dtype), v);
      const float vs = v * scale;
      const __half hi = __float2half_rn(vs);
      vals[r] = hl == 0 ? hi : __float2half_rn(vs - __half2float(hi));
    }
    regs[0] = (uint32_t)__half_as_ushort(vals[0]) | ((uint32_t)__half_as_ushort(vals[1]) << 16);
    regs[1] = (uint32_t)__half_as_ushort(vals[2]) | ((uint32_t)__half_as_ushort(vals[3]) << 16);
  }
  const int KS = KS0 + p.F / 4;
  p.frag[((int64_t)gq * KS + ksg) * 32 + lane] = make_uint2(regs[0], regs[1]);
}

// ---- logits ---------------------------------------------------------------------

struct LogitsParams {
  tq::CacheView cv;
  const int32_t* ctx_len;
  int n_kv_heads, n_q_heads, G, qtiles;
  int keys_per_cta;
  int max_ctx;               // ctx_len values are clamped to [0, max_ctx]
  const uint2* frag;
  const float* inv_scale;
  float* out;
  int64_t out_stride;
  uint32_t pool0, pool1;     // fp16 magnitude table for the byte permute (b <= 3)
  uint32_t lo0, lo1, hi0, hi1;  // low / high bytes of the 8 magnitudes (b = 4)
  float qjl_scale;
};

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint2 b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b.x), "r"(b.y));
}

// The two fp16 pairs (h = 0: elements 4ks, 4ks+1; h = 1: 4ks+2, 4ks+3) of
// k-step ks of the codebook part, decoded from one chunk's words.
template <int BITS, int E>
__device__ __forceinline__ void decode_index_pair(const uint32_t* w, int ks, const LogitsParams& p,
                                                  uint32_t& h0, uint32_t& h1) {
  constexpr int n_sign = BITS == 4 ? 0 : (E + 31) / 32;
  if constexpr (BITS == 4) {
    const uint32_t x = w[ks / 2] >> (8 * (ks % 2));
    const uint32_t sel = (x & 0x77u) | ((x >> 8) & 0x7700u);
    const uint32_t lo = prmt(p.lo0, p.lo1, sel);
    const uint32_t hi = prmt(p.hi0, p.hi1, sel);
    h0 = prmt(lo, hi, 0x6240u) | ((x << 12) & 0x80008000u);
    h1 = prmt(lo, hi, 0x7351u) | ((x << 8) & 0x80008000u);
  } else {
    const uint32_t sw = w[ks / 8];
    const int pi0 = 2 * (ks % 8);
    const uint32_t s0 = (sw << (15 - pi0)) & 0x80008000u;
    const uint32_t s1 = (sw << (14 - pi0)) & 0x80008000u;
    uint32_t m0, m1;
    if constexpr (BITS == 1) {
      m0 = m1 = p.pool0;
    } else {
      uint32_t v;
      if constexpr (BITS == 2) v = (w[n_sign + ks / 8] >> (ks % 8)) & 0x01010101u;
      else v = (w[n_sign + ks / 4] >> (2 * (ks % 4))) & 0x03030303u;
      const uint32_t sel = v * 0x22u + 0x10101010u;
      m0 = prmt(p.pool0, p.pool1, sel);
      m1 = prmt(p.pool0, p.pool1, sel >> 16);
    }
    h0 = m0 | s0;
    h1 = m1 | s1;
  }
}

// The +-1 fp16 pairs of k-step ks of the QJL part.
__device__ __forceinline__ void decode_sign_pair(uint32_t qw, int ks, uint32_t& h0, uint32_t& h1) {
  const int pi0 = 2 * (ks % 8);
  h0 = 0x3C003C00u | ((qw << (15 - pi0)) & 0x80008000u);
  h1 = 0x3C003C00u | ((qw << (14 - pi0)) & 0x80008000u);
}

template <int W>
__device__ __forceinline__ void load_chunk(const uint8_t* src, uint32_t (&w)[W]) {
  if constexpr (W % 4 == 0) {
#pragma unroll
    for (int i = 0; i < W / 4; ++i) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + i);
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  } else if constexpr (W % 2 == 0) {
#pragma unroll
    for (int i = 0; i < W / 2; ++i) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(src) + i);
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < W; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t*>(src) + i);
  }
}

// grid: (chunks of keys, batch * n_kv_heads, query tiles of 4); block 128.
template <int BITS, int E, int F>
__global__ void __launch_bounds__(128) logits_kernel(LogitsParams p) {
  constexpr int KS0 = E / 4, KS1 = F / 4;
  constexpr int n_sign = BITS == 4 ? 0 : (E + 31) / 32;
  constexpr int n_mag = BITS == 2 ? (E + 31) / 32 : BITS == 3 ? E / 16 : 0;
  constexpr int n_nib = BITS == 4 ? E / 8 : 0;
  constexpr int q0 = n_sign + n_mag + n_nib;
  constexpr int W = q0 + (F + 31) / 32;
  constexpr int CB = 16 * W;
  constexpr int NB = F > 0 ? 4 : 2;

  const int gi = blockIdx.y;
  const int b = gi / p.n_kv_heads, h = gi % p.n_kv_heads;
  const int qt = blockIdx.z;
  const int ctx = min(p.ctx_len[b], p.max_ctx);
  const int k0 = blockIdx.x * p.keys_per_cta;
  if (k0 >= ctx) return;
  const int k1 = min(k0 + p.keys_per_cta, ctx);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;

  // query fragments of this group / query tile, kept in registers
  uint2 bq[KS0 + KS1];
  const uint2* fsrc = p.frag + ((int64_t)gi * p.qtiles + qt) * (KS0 + KS1) * 32 + lane;
#pragma unroll
  for (int ks = 0; ks < KS0 + KS1; ++ks) bq[ks] = fsrc[ks * 32];
  const int qidx = qt * 4 + t;                  // this thread's query within the group
  const bool qvalid = qidx < p.G;
  const int hq = h * p.G + (qvalid ? qidx : 0);
  const float inv0 = p.inv_scale[((int64_t)b * p.n_q_heads + hq) * 2];
  const float inv1 = F > 0 ? p.inv_scale[((int64_t)b * p.n_q_heads + hq) * 2 + 1] : 0.0f;
  float* orow = p.out + ((int64_t)b * p.n_q_heads + hq) * p.out_stride;

  const int n_tiles = (k1 - k0 + 15) >> 4;
  for (int tile = warp; tile < n_tiles; tile += 4) {
    const int base = k0 + tile * 16;
    const int64_t page = p.cv.block_table[(int64_t)b * p.cv.max_pages + base / p.cv.page_tokens];
    if (page < 0 || page >= p.cv.n_pages) {
      if (lane == 0) report(p.cv.err, TQ_DEV_ERR_PAGE);
      continue;
    }
    const uint8_t* hb = p.cv.pages + page * p.cv.page_bytes + (int64_t)h * p.cv.head_block_bytes;
    const int slot = base % p.cv.page_tokens;
    const int ra = base + g, rb = base + g + 8;
    uint32_t wa[W], wb[W];
    float kna = 0.f, rna = 0.f, knb = 0.f, rnb = 0.f;
    if (ra < k1) {
      load_chunk<W>(hb + (int64_t)(slot + g) * CB + t * 4 * W, wa);
      const uint8_t* ns = hb + (int64_t)p.cv.page_tokens * CB + (int64_t)(slot + g) * NB;
      if constexpr (F > 0) {
        const __half2 nr = __ldg(reinterpret_cast<const __half2*>(ns));
        kna = __low2float(nr); rna = __high2float(nr);
      } else {
        kna = __half2float(__ldg(reinterpret_cast<const __half*>(ns)));
      }
    } else {
#pragma unroll
      for (int i = 0; i < W; ++i) wa[i] = 0u;
    }
    if (rb < k1) {
      load_chunk<W>(hb + (int64_t)(slot + g + 8) * CB + t * 4 * W, wb);
      const uint8_t* ns = hb + (int64_t)p.cv.page_tokens * CB + (int64_t)(slot + g + 8) * NB;
      if constexpr (F > 0) {
        const __half2 nr = __ldg(reinterpret_cast<const __half2*>(ns));
        knb = __low2float(nr); rnb = __high2float(nr);
      } else {
        knb = __half2float(__ldg(reinterpret_cast<const __half*>(ns)));
      }
    } else {
#pragma unroll
      for (int i = 0; i < W; ++i) wb[i] = 0u;
    }

    float acc0[4] = {0.f, 0.f, 0.f, 0.f};
    float acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < KS0; ++ks) {
      uint32_t a0, a2, a1, a3;
      decode_index_pair<BITS, E>(wa, ks, p, a0, a2);
      decode_index_pair<BITS, E>(wb, ks, p, a1, a3);
      mma16816(acc0, a0, a1, a2, a3, bq[ks]);
    }
    if constexpr (F > 0) {
#pragma unroll
      for (int ks = 0; ks < KS1; ++ks) {
        uint32_t a0, a2, a1, a3;
        decode_sign_pair(wa[q0 + ks / 8], ks, a0, a2);
        decode_sign_pair(wb[q0 + ks / 8], ks, a1, a3);
        mma16816(acc1, a0, a1, a2, a3, bq[KS0 + ks]);
      }
    }
    // columns 2t (hi) and 2t+1 (lo) belong to query t of this tile
    const float la = kna * fmaf(p.qjl_scale * rna * inv1, acc1[0] + acc1[1], inv0 * (acc0[0] + acc0[1]));
    const float lb = knb * fmaf(p.qjl_scale * rnb * inv1, acc1[2] + acc1[3], inv0 * (acc0[2] + acc0[3]));
    if (qvalid) {
      if (ra < k1) orow[ra] = la;
      if (rb < k1) orow[rb] = lb;
    }
  }
}

}  // namespace tqd

namespace tq {

size_t logits_workspace(const tq_codebook* cb, int64_t groups, int G) {
  const int qtiles = (G + 3) / 4;
  const size_t frag = (size_t)groups * qtiles * (cb->lay.E / 4 + cb->lay.F / 4) * 32 * sizeof(uint2);
  const size_t inv = (size_t)groups * G * 2 * sizeof(float);
  return ((frag + 255) / 256) * 256 + inv;
}

template <int BITS, int E, int F>
static void run_logits(const tqd::LogitsParams& p, dim3 grid, cudaStream_t st) {
  tqd::logits_kernel<BITS, E, F><<<grid, 128, 0, st>>>(p);
}

template <int BITS>
static bool dispatch_logits(const Layout& L, const tqd::LogitsParams& p, dim3 grid, cudaStream_t st) {
  if (L.E == 32 && L.F == 32) return run_logits<BITS, 32, 32>(p, grid, st), true;
  if (L.E == 32 && L.F == 0) return run_logits<BITS, 32, 0>(p, grid, st), true;
  if (L.E == 16 && L.F == 16) return run_logits<BITS, 16, 16>(p, grid, st), true;
  if (L.E == 16 && L.F == 0) return run_logits<BITS, 16, 0>(p, grid, st), true;
  if (L.E == 64 && L.F == 64) return run_logits<BITS, 64, 64>(p, grid, st), true;
  if (L.E == 64 && L.F == 0) return run_logits<BITS, 64, 0>(p, grid, st), true;
  if (L.E == 48 && L.F == 48) return run_logits<BITS, 48, 48>(p, grid, st), true;
  if (L.E == 48 && L.F == 0) return run_logits<BITS, 48, 0>(p, grid, st), true;
  return false;
}

static uint32_t pack2(uint16_t lo, uint16_t hi) { return (uint32_t)lo | ((uint32_t)hi << 16); }

tq_status launch_logits(const tq_codebook* cb, const CacheView& cv, const void* q, tq_dtype dt,
                        int64_t batch, int n_q_heads, const int32_t* ctx_len, int64_t max_ctx,
                        float* out, int64_t out_stride, void* ws, size_t ws_bytes,
                        cudaStream_t st) {
  const Layout& L = cb->lay;
  const int G = n_q_heads / cv.n_kv_heads;
  const int qtiles = (G + 3) / 4;
  const int64_t groups = batch * cv.n_kv_heads;
  const size_t need = logits_workspace(cb, groups, G);
  if (ws_bytes < need) return fail(TQ_EINVAL, "tq_logits: workspace too small");
  if (max_ctx == 0 || batch == 0) return TQ_OK;
  const size_t frag_bytes = (size_t)groups * qtiles * (L.E / 4 + L.F / 4) * 32 * sizeof(uint2);
  uint2* frag = reinterpret_cast<uint2*>(ws);
  float* inv = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + ((frag_bytes + 255) / 256) * 256);
  tqd::PrepParams pp;
  pp.q = q;
  pp.dtype = dt;
  pp.d = L.d;
  pp.E = L.E;
  pp.F = L.F;
  pp.n_q_heads = n_q_heads;
  pp.n_kv_heads = cv.n_kv_heads;
  pp.G = G;
  pp.qtiles = qtiles;
  pp.pi32 = cb->pi32;
  pp.s32 = cb->s32;
  pp.s_row_norm_max = (float)cb->s_row_norm_max;
  pp.frag = frag;
  pp.inv_scale = inv;
  dim3 pgrid((unsigned)(groups * qtiles), (unsigned)(L.E / 4 + L.F / 4));
  tqd::prep_queries_kernel<<<pgrid, 32, 0, st>>>(pp);

  tqd::LogitsParams lp;
  lp.cv = cv;
  lp.ctx_len = ctx_len;
  lp.n_kv_heads = cv.n_kv_heads;
  lp.n_q_heads = n_q_heads;
  lp.G = G;
  lp.qtiles = qtiles;
  // Split the context so that the grid fills the GPU about twice over.
  const int64_t total_units = groups * qtiles;
  int64_t target = 2 * 148;
  int64_t chunks = (target + total_units - 1) / total_units;
  int64_t kpc = (max_ctx + chunks - 1) / chunks;
  kpc = ((kpc + 63) / 64) * 64;
  if (kpc < 64) kpc = 64;
  lp.keys_per_cta = (int)kpc;
  lp.max_ctx = (int)max_ctx;
  lp.frag = frag;
  lp.inv_scale = inv;
  lp.out = out;
  lp.out_stride = out_stride;
  const uint16_t* M = cb->mag16;
  lp.pool0 = L.bits == 1 ? pack2(M[0], M[0]) : L.bits == 2 ? pack2(M[0], M[1]) : pack2(M[0], M[1]);
  lp.pool1 = L.bits == 3 ? pack2(M[2], M[3]) : 0u;
  lp.lo0 = lp.lo1 = lp.hi0 = lp.hi1 = 0u;
  if (L.bits == 4) {
    for (int i = 0; i < 4; ++i) {
      lp.lo0 |= (uint32_t)(M[i] & 0xFF) << (8 * i);
      lp.lo1 |= (uint32_t)(M[4 + i] & 0xFF) << (8 * i);
      lp.hi0 |= (uint32_t)(M[i] >> 8) << (8 * i);
      lp.hi1 |= (uint32_t)(M[4 + i] >> 8) << (8 * i);
    }
  }
  lp.qjl_scale = (float)cb->qjl_scale;
  dim3 grid((unsigned)((max_ctx + kpc - 1) / kpc), (unsigned)groups, (unsigned)qtiles);
  bool ok = false;
  switch (L.bits) {
    case 1: ok = dispatch_logits<1>(L, lp, grid, st); break;
    case 2: ok = dispatch_logits<2>(L, lp, grid, st); break;
    case 3: ok = dispatch_logits<3>(L, lp, grid, st); break;
    case 4: ok = dispatch_logits<4>(L, lp, grid, st); break;
  }
  if (!ok) return fail(TQ_EUNSUPPORTED, "tq_logits: no kernel for this (d, m)");
  return cuda_fail(cudaGetLastError(), "tq_logits launch");
}

}  // namespace tq
