// Fused attention logits straight from the packed keys.
//
// "TurboQuant explained" (a2a-mcp.org), §Stage 2 and §How it works: the
// query is rotated once (Pi q) and sketched once (S q); every logit is then
//   L = ||k|| ( sum_j (Pi q)_j c16[idx_j] + sqrt(pi/2)/m ||r|| sum_i (S q)_i s_i )
// evaluated from the indices and sign bits without dequantizing the key.
//
// Design.  Both sums are dot products of a decoded key row with the query
// group that shares its KV head, so a warp takes 16 keys at a time and runs
// them through the tensor cores with the key operand built in registers:
//  * codebook term, b <= 3: m16n8k32 int8 MMAs.  c16 * 2^f is an integer of
//    at most 16 bits for every level, so a key element is two int8 slices;
//    eight stored codes form one byte-permute selector after a single mask,
//    and two permutes of 8-byte tables give the high and low slices of four
//    elements.  (Pi q) is quantized to 16-bit integers scaled by its largest
//    entry, also as two int8 slices; the four slice products are accumulated
//    exactly in int32 and combined in fp32.
//  * codebook term, b = 4: m16n8k16 fp16 MMAs on sign-magnitude codes (16
//    levels do not fit one 8-byte permute table), the query as fp16 hi + lo.
//  * sign term: m16n8k32 int8 MMAs.  The stored sign bits are spread to 0/1
//    bytes with one shift and mask per 4 bits; S q is quantized to 16-bit
//    integers z, and sum_i s_i z_i = sum_i z_i - 2 sum_i beta_i z_i.
// The operands never leave registers, so HBM traffic is the 68-byte records
// plus the logits.  Thread t of a quad owns chunk t of every record: the bits
// it loads are exactly the bits its fragments need.

#include "tq_internal.cuh"

namespace tqd {

// ---- query preparation ------------------------------------------------------
// Workspace: codebook fragments uint2 [gq][KC][32] (KC = E/8 int8 k-steps, or
// E/4 fp16 k-steps for b = 4), QJL fragments uint2 [gq][F/8][32]
// (gq = group x query tile), per-query scalars float4 [batch * n_q_heads] =
// {codebook scale, QJL step, sum z, 0}.

constexpr int kSliceMax = 32639;   // |z| bound: the high int8 slice stays in [-128, 127]
constexpr int kPrepStageFloats = 16384;   // 64 KB of the matrix staged at a time

struct PrepParams {
  const void* q;
  tq_dtype dtype;
  int d, d_pad, m_pad, E, F;   // E, F: coordinates / QJL rows per chunk
  int n_q_heads, n_kv_heads, G, qtiles;
  int cb_int8;           // codebook fragments as int8 slices (b <= 3) or fp16 hi/lo (b = 4)
  float cb_unscale;      // 2^-f: c16 * 2^f are the integer table entries
  const float* pit32;    // Pi^T [d][d_pad]
  const float* st32;     // S^T  [d][m_pad]
  uint2* frag;
  uint2* qfrag;
  float4* scal;
};

// Writes the int8 slices of z into the fragment of MMA k-step l / 8: lane
// (2 * query + slice) * 4 + t, register (l / 4) % 2, byte l % 4.
__device__ __forceinline__ void put_slices(uint2* base, int Ep, int row, int query, int z) {
  const int zh = (z + 128) >> 8;            // floor((z + 128) / 256)
  const int zl = z - 256 * zh;              // in [-128, 127]
  const int t = row / Ep, l = row % Ep;
  const int kk = l / 8, hreg = (l >> 2) & 1, e = l & 3;
  int8_t* fr = reinterpret_cast<int8_t*>(base + kk * 32);
  fr[((2 * query) * 4 + t) * 8 + hreg * 4 + e] = (int8_t)zh;
  fr[((2 * query + 1) * 4 + t) * 8 + hreg * 4 + e] = (int8_t)zl;
}

// Rotates and sketches each query once (TQ §How it works: the query is
// pre-rotated once and reused over the whole context).  CTA (group x query
// tile, part): part 0 computes every row of Pi q, part 1 every row of S q;
// warp w handles query w of the tile, lane l rows l, l + 32, ...  The matrix
// (Pi^T or S^T) streams through shared memory in 64 KB tiles with all copies
// in flight at once.  Every fragment slot is written (zeros for padding rows
// and for query slots past G), so the workspace needs no clearing.
// grid: (groups * qtiles, 1 + (m_pad > 0)); block 128; dynamic smem 64 KB.
__global__ void __launch_bounds__(128) prep_queries_kernel(PrepParams p) {
  asm volatile("griddepcontrol.launch_dependents;");
  extern __shared__ float4 prep_dyn[];
  float* mt = reinterpret_cast<float*>(prep_dyn);
  __shared__ float qs[4][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = blockIdx.x;
  const int gi = gq / p.qtiles, qt = gq % p.qtiles;
  const int b = gi / p.n_kv_heads, kv = gi % p.n_kv_heads;
  const int d = p.d;
  const int ql = qt * 4 + warp;
  const bool valid = ql < p.G;
  const int64_t qrow = (int64_t)b * p.n_q_heads + kv * p.G + (valid ? ql : 0);
  float n2 = 0.0f;
  for (int k = lane; k < d; k += 32) {
    const float v = valid ? load_elem(p.q, qrow * d + k, p.dtype) : 0.0f;
    qs[warp][k] = v;
    n2 = fmaf(v, v, n2);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) n2 += __shfl_xor_sync(0xffffffffu, n2, o);
  const float qn = sqrtf(n2);
  const int part = blockIdx.y;
  const int rows = part == 0 ? p.d_pad : p.m_pad;     // multiple of 64, <= 256
  const float* Mt = part == 0 ? p.pit32 : p.st32;     // [d][rows]
  const int tile = min(rows, (kPrepStageFloats / d) & ~31);

  float v[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) v[r] = 0.0f;
  for (int r0 = 0; r0 < rows; r0 += tile) {
    const int tn = min(tile, rows - r0);
    __syncthreads();                 // previous tile consumed (and qs complete)
    const int n4 = d * tn / 4;
    for (int e = threadIdx.x; e < n4; e += 128) {
      const int k = e / (tn / 4), c4 = e % (tn / 4);
      const unsigned dst = (unsigned)__cvta_generic_to_shared(mt + k * tn + 4 * c4);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst),
                   "l"(Mt + (size_t)k * rows + r0 + 4 * c4) : "memory");
    }
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int row = 32 * r + lane;
      if (row >= r0 && row < r0 + tn) {
        float acc = 0.0f;
#pragma unroll 8
        for (int k = 0; k < d; ++k) acc = fmaf(mt[k * tn + row - r0], qs[warp][k], acc);
        v[r] = acc;
      }
    }
  }
  const int nr = rows / 32;
  if (part == 0 && !p.cb_int8) {
    // fp16 hi + lo: a power of two puts every |(Pi q)_j| <= ||q|| below 2^14
    int e = 0;
    if (qn > 0.0f) frexpf(qn, &e);
    const float scale = ldexpf(1.0f, 14 - e);
    const int KS = p.E / 4;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if (r >= nr) break;
      const int row = 32 * r + lane;
      __half hi = __float2half_rn(0.0f), lo = hi;
      if (valid) {
        const float vs = v[r] * scale;
        hi = __float2half_rn(vs);
        lo = __float2half_rn(vs - __half2float(hi));
      }
      const int t = row / p.E, l = row % p.E;
      __half* fr = reinterpret_cast<__half*>(p.frag + ((int64_t)gq * KS + l / 4) * 32);
      const int half_idx = ((l >> 1) & 1) * 2 + (l & 1);
      fr[((2 * warp) * 4 + t) * 4 + half_idx] = hi;       // column 2 * query: hi part
      fr[((2 * warp + 1) * 4 + t) * 4 + half_idx] = lo;   // column 2 * query + 1: lo part
    }
    if (valid && lane == 0) p.scal[qrow].x = 1.0f / scale;
    return;
  }
  // 16-bit fixed point scaled by the largest entry, as two int8 slices
  float mx = 0.0f;
#pragma unroll
  for (int r = 0; r < 8; ++r)
    if (r < nr) mx = fmaxf(mx, fabsf(v[r]));
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float step = mx > 0.0f ? mx / (float)kSliceMax : 0.0f;
  const int Ep = part == 0 ? p.E : p.F;
  const int ksteps = Ep / 8;
  uint2* base = (part == 0 ? p.frag : p.qfrag) + (int64_t)gq * ksteps * 32;
  int zsum = 0;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    if (r >= nr) break;
    int z = 0;
    if (valid && step > 0.0f) z = max(-kSliceMax, min(kSliceMax, __float2int_rn(v[r] / step)));
    zsum += z;
    put_slices(base, Ep, 32 * r + lane, warp, z);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) zsum += __shfl_xor_sync(0xffffffffu, zsum, o);
  if (valid && lane == 0) {
    if (part == 0) {
      p.scal[qrow].x = step * p.cb_unscale;
    } else {
      p.scal[qrow].y = step;
      p.scal[qrow].z = (float)zsum;   // exact: |sum| < 2^24
    }
  }
}

// ---- logits ---------------------------------------------------------------------

struct LogitsParams {
  tq::CacheView cv;
  int page_shift;            // log2(page_tokens)
  const int32_t* ctx_len;
  int n_kv_heads, n_q_heads, G, qtiles;
  int keys_per_cta;
  int max_ctx;               // ctx_len values are clamped to [0, max_ctx]
  const uint2* frag;
  const uint2* qfrag;
  const float4* scal;
  float* out;
  int64_t out_stride;
  uint32_t th0, th1, tl0, tl1;  // b <= 3: high / low int8 slices of c16 * 2^f, levels 0..7
  uint32_t lo0, lo1, hi0, hi1;  // b = 4: low / high bytes of the 8 fp16 magnitudes
  float qjl_scale;
};

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint2 b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b.x), "r"(b.y));
}

__device__ __forceinline__ void mma_s8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint2 b) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b.x), "r"(b.y));
}

__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint2 b) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b.x), "r"(b.y));
}

// Byte-permute selector of the codes of local elements 8 kk .. 8 kk + 7 of a
// chunk (layout version 3, b <= 3): nibble i holds the code of element 8 kk + i.
template <int BITS, int E>
__device__ __forceinline__ uint32_t code_selector(const uint32_t* w, int kk) {
  if constexpr (BITS == 1) {
    return (w[kk / 4] >> (kk % 4)) & 0x11111111u;
  } else if constexpr (BITS == 2) {
    return (w[kk / 2] >> (2 * (kk % 2))) & 0x33333333u;
  } else {
    constexpr int full = E / 32;          // complete 32-element groups
    const int g = kk / 4, j = kk % 4;
    if (g < full) {
      if (j < 3) return w[3 * g + j] & 0x77777777u;
      return ((w[3 * g] >> 3) & 0x11111111u) | ((w[3 * g + 1] >> 2) & 0x22222222u) |
             ((w[3 * g + 2] >> 1) & 0x44444444u);
    }
    return w[3 * full + (kk - 4 * full)] & 0x77777777u;
  }
}

// b = 4: the two fp16 pairs (elements 4ks, 4ks+1 and 4ks+2, 4ks+3) of k-step
// ks from the sign-magnitude nibbles (magnitude bytes by permute, sign ORed
// into bit 15 of each half).
__device__ __forceinline__ void decode_nibble_pair(const uint32_t* w, int ks, const LogitsParams& p,
                                                   uint32_t& h0, uint32_t& h1) {
  const uint32_t x = w[ks / 2] >> (8 * (ks % 2));
  const uint32_t sel = (x & 0x77u) | ((x >> 8) & 0x7700u);
  const uint32_t lo = prmt(p.lo0, p.lo1, sel);
  const uint32_t hi = prmt(p.hi0, p.hi1, sel);
  h0 = prmt(lo, hi, 0x6240u) | ((x << 12) & 0x80008000u);
  h1 = prmt(lo, hi, 0x7351u) | ((x << 8) & 0x80008000u);
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

constexpr int kLogitsWarps = 8;     // warps per CTA
constexpr int kPrefetch = 3;        // 16-key tiles in flight per warp
constexpr int kCtaPages = 64;       // block-table entries staged per CTA

// One warp's share of a 16-key tile: this thread's chunk of keys g and g+8,
// and their norm slots.
template <int W>
struct KeyTile {
  uint32_t wa[W], wb[W];
  uint32_t na, nb;
};

template <int W, int NB>
__device__ __forceinline__ void load_tile(KeyTile<W>& kt, const uint8_t* hb, int P, int slot, int g,
                                          int t, bool va, bool vb) {
  constexpr int CB = 16 * W;
  if (va) {
    load_chunk<W>(hb + (slot + g) * CB + t * 4 * W, kt.wa);
    const uint8_t* ns = hb + P * CB + (slot + g) * NB;
    kt.na = NB == 4 ? __ldg(reinterpret_cast<const uint32_t*>(ns))
                    : (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(ns));
  } else {
#pragma unroll
    for (int i = 0; i < W; ++i) kt.wa[i] = 0u;
    kt.na = 0u;
  }
  if (vb) {
    load_chunk<W>(hb + (slot + g + 8) * CB + t * 4 * W, kt.wb);
    const uint8_t* ns = hb + P * CB + (slot + g + 8) * NB;
    kt.nb = NB == 4 ? __ldg(reinterpret_cast<const uint32_t*>(ns))
                    : (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(ns));
  } else {
#pragma unroll
    for (int i = 0; i < W; ++i) kt.wb[i] = 0u;
    kt.nb = 0u;
  }
}

__device__ __forceinline__ float lo_half(uint32_t v) {
  return __half2float(__ushort_as_half((unsigned short)(v & 0xFFFFu)));
}
__device__ __forceinline__ float hi_half(uint32_t v) {
  return __half2float(__ushort_as_half((unsigned short)(v >> 16)));
}

// grid: (chunks of keys, batch * n_kv_heads, query tiles of 4); block 256.
// Each warp walks the CTA's 16-key tiles with stride kLogitsWarps, keeping
// kPrefetch tiles of 128-bit loads in flight.  The CTA's block-table entries
// are staged in shared memory first, so a tile's loads never wait on a
// dependent page-id load; page_tokens is a power of two, so page and slot
// are a shift and a mask.  The query fragments are read only after
// griddepcontrol.wait: the kernel may start while the query preparation
// kernel (programmatic dependent launch) is still running.
template <int BITS, int E, int F>
__global__ void __launch_bounds__(kLogitsWarps * 32, E >= 64 ? 1 : 2) logits_kernel(LogitsParams p) {
  constexpr bool kInt8 = BITS <= 3;
  constexpr int KC = kInt8 ? E / 8 : E / 4;   // codebook MMA k-steps
  constexpr int KQ = F / 8;                   // sign-term MMA k-steps
  constexpr int q0 = BITS == 1 ? (E + 31) / 32 : BITS == 2 ? E / 16
                   : BITS == 3 ? 3 * (E / 32) + 2 * ((E % 32) / 16) : E / 8;
  constexpr int W = q0 + (F + 31) / 32;
  constexpr int NB = F > 0 ? 4 : 2;
  __shared__ int64_t page_base[kCtaPages];   // byte offset of this head's block, -1 if bad

  const int gi = blockIdx.y;
  const int b = gi / p.n_kv_heads, h = gi % p.n_kv_heads;
  const int qt = blockIdx.z;
  const int ctx = min(p.ctx_len[b], p.max_ctx);
  const int k0 = blockIdx.x * p.keys_per_cta;
  if (k0 >= ctx) return;
  const int k1 = min(k0 + p.keys_per_cta, ctx);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int ps = p.page_shift;
  const int P = 1 << ps;
  const int first_page = k0 >> ps;
  const int n_pages = ((k1 - 1) >> ps) - first_page + 1;
  for (int j = threadIdx.x; j < n_pages; j += blockDim.x) {
    const int64_t page = p.cv.block_table[(int64_t)b * p.cv.max_pages + first_page + j];
    int64_t off = -1;
    if (page >= 0 && page < p.cv.n_pages) off = page * p.cv.page_bytes + (int64_t)h * p.cv.head_block_bytes;
    else report(p.cv.err, TQ_DEV_ERR_PAGE);
    page_base[j] = off;
  }
  __syncthreads();

  const int n_tiles = (k1 - k0 + 15) >> 4;
  const int n_my = warp < n_tiles ? (n_tiles - warp + kLogitsWarps - 1) / kLogitsWarps : 0;
  auto issue = [&](KeyTile<W>& kt, int i) {
    const int base = k0 + 16 * (warp + kLogitsWarps * i);
    const int64_t off = page_base[(base >> ps) - first_page];
    const bool ok = off >= 0;
    load_tile<W, NB>(kt, p.cv.pages + (ok ? off : 0), P, base & (P - 1), g, t, ok && base + g < k1,
                     ok && base + g + 8 < k1);
  };

  KeyTile<W> buf[kPrefetch];
#pragma unroll
  for (int s = 0; s < kPrefetch; ++s)
    if (s < n_my) issue(buf[s], s);

  // the query fragments come from the preparation kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int gq = gi * p.qtiles + qt;
  uint2 bq[KC];
  const uint2* fsrc = p.frag + (int64_t)gq * KC * 32 + lane;
#pragma unroll
  for (int kk = 0; kk < KC; ++kk) bq[kk] = fsrc[kk * 32];
  uint2 bz[KQ > 0 ? KQ : 1];
  if constexpr (KQ > 0) {
    const uint2* qsrc = p.qfrag + (int64_t)gq * KQ * 32 + lane;
#pragma unroll
    for (int kk = 0; kk < KQ; ++kk) bz[kk] = qsrc[kk * 32];
  }
  const int qidx = qt * 4 + t;                  // this thread's query within the group
  const bool qvalid = qidx < p.G;
  const int hq = h * p.G + (qvalid ? qidx : 0);
  const float4 sc = p.scal[(int64_t)b * p.n_q_heads + hq];
  const float c0 = sc.x;
  const float c1 = F > 0 ? p.qjl_scale * sc.y : 0.0f;
  const float zsum = sc.z;
  float* orow = p.out + ((int64_t)b * p.n_q_heads + hq) * p.out_stride;

  for (int i0 = 0; i0 < n_my; i0 += kPrefetch) {
#pragma unroll
    for (int s = 0; s < kPrefetch; ++s) {
      const int i = i0 + s;
      if (i < n_my) {
        const KeyTile<W> cur = buf[s];
        if (i + kPrefetch < n_my) issue(buf[s], i + kPrefetch);
        const int base = k0 + 16 * (warp + kLogitsWarps * i);
        if (page_base[(base >> ps) - first_page] < 0) continue;
        float la, lb;
        if constexpr (kInt8) {
          // codebook term: int8 slices of c16 * 2^f against those of (Pi q)
          int ah[4] = {0, 0, 0, 0}, al[4] = {0, 0, 0, 0};
#pragma unroll
          for (int kk = 0; kk < KC; ++kk) {
            const uint32_t sa = code_selector<BITS, E>(cur.wa, kk);
            const uint32_t sb = code_selector<BITS, E>(cur.wb, kk);
            const uint32_t sa2 = sa >> 16, sb2 = sb >> 16;
            mma_s8s8(ah, prmt(p.th0, p.th1, sa), prmt(p.th0, p.th1, sb), prmt(p.th0, p.th1, sa2),
                     prmt(p.th0, p.th1, sb2), bq[kk]);
            mma_s8s8(al, prmt(p.tl0, p.tl1, sa), prmt(p.tl0, p.tl1, sb), prmt(p.tl0, p.tl1, sa2),
                     prmt(p.tl0, p.tl1, sb2), bq[kk]);
          }
          // columns 2t / 2t+1: high / low slice of query t
          la = c0 * fmaf(65536.0f, (float)ah[0], fmaf(256.0f, (float)(ah[1] + al[0]), (float)al[1]));
          lb = c0 * fmaf(65536.0f, (float)ah[2], fmaf(256.0f, (float)(ah[3] + al[2]), (float)al[3]));
        } else {
          float acc0[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ks = 0; ks < KC; ++ks) {
            uint32_t a0, a2, a1, a3;
            decode_nibble_pair(cur.wa, ks, p, a0, a2);
            decode_nibble_pair(cur.wb, ks, p, a1, a3);
            mma_f16(acc0, a0, a1, a2, a3, bq[ks]);
          }
          // columns 2t (hi) and 2t+1 (lo) belong to query t of this tile
          la = c0 * (acc0[0] + acc0[1]);
          lb = c0 * (acc0[2] + acc0[3]);
        }
        if constexpr (F > 0) {
          // sign term: 0/1 bytes of the sign bits against the int8 slices of z
          int acc1[4] = {0, 0, 0, 0};
#pragma unroll
          for (int kk = 0; kk < KQ; ++kk) {
            const uint32_t xa = cur.wa[q0 + kk / 4] >> (2 * (kk % 4));
            const uint32_t xb = cur.wb[q0 + kk / 4] >> (2 * (kk % 4));
            mma_u8s8(acc1, xa & 0x01010101u, xb & 0x01010101u, (xa >> 1) & 0x01010101u,
                     (xb >> 1) & 0x01010101u, bz[kk]);
          }
          const float ta = zsum - 2.0f * (float)(256 * acc1[0] + acc1[1]);
          const float tb = zsum - 2.0f * (float)(256 * acc1[2] + acc1[3]);
          la = fmaf(c1 * hi_half(cur.na), ta, la);
          lb = fmaf(c1 * hi_half(cur.nb), tb, lb);
        }
        la *= lo_half(cur.na);
        lb *= lo_half(cur.nb);
        const int ra = base + g, rb = ra + 8;
        if (qvalid) {
          if (ra < k1) __stcs(orow + ra, la);
          if (rb < k1) __stcs(orow + rb, lb);
        }
      }
    }
  }
}

}  // namespace tqd

namespace tq {

struct LogitsWs {
  size_t frag, qfrag, scal, total;
};

static int codebook_ksteps(const Layout& L) { return L.bits <= 3 ? L.E / 8 : L.E / 4; }

static LogitsWs logits_ws_layout(const tq_codebook* cb, int64_t groups, int G, int64_t batch_heads) {
  auto al = [](size_t n) { return (n + 255) / 256 * 256; };
  const int qtiles = (G + 3) / 4;
  LogitsWs w;
  w.frag = al((size_t)groups * qtiles * codebook_ksteps(cb->lay) * 32 * sizeof(uint2));
  w.qfrag = al((size_t)groups * qtiles * (cb->lay.F / 8) * 32 * sizeof(uint2));
  w.scal = al((size_t)batch_heads * sizeof(float4));
  w.total = w.frag + w.qfrag + w.scal;
  return w;
}

size_t logits_workspace(const tq_codebook* cb, int64_t groups, int G) {
  return logits_ws_layout(cb, groups, G, groups * G).total;
}

template <int BITS, int E, int F>
static void run_logits(const tqd::LogitsParams& p, dim3 grid, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(tqd::kLogitsWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, tqd::logits_kernel<BITS, E, F>, p);
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

tq_status launch_logits(const tq_codebook* cb, const CacheView& cv, const void* q, tq_dtype dt,
                        int64_t batch, int n_q_heads, const int32_t* ctx_len, int64_t max_ctx,
                        float* out, int64_t out_stride, void* ws, size_t ws_bytes,
                        cudaStream_t st) {
  const Layout& L = cb->lay;
  const int G = n_q_heads / cv.n_kv_heads;
  const int qtiles = (G + 3) / 4;
  const int64_t groups = batch * cv.n_kv_heads;
  const LogitsWs wl = logits_ws_layout(cb, groups, G, batch * n_q_heads);
  if (ws_bytes < wl.total) return fail(TQ_EINVAL, "tq_logits: workspace too small");
  if (max_ctx == 0 || batch == 0) return TQ_OK;
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  uint2* frag = reinterpret_cast<uint2*>(wsb);
  uint2* qfrag = reinterpret_cast<uint2*>(wsb + wl.frag);
  float4* scal = reinterpret_cast<float4*>(wsb + wl.frag + wl.qfrag);

  tqd::PrepParams pp;
  pp.q = q;
  pp.dtype = dt;
  pp.d = L.d;
  pp.d_pad = L.d_pad;
  pp.m_pad = L.m_pad;
  pp.E = L.E;
  pp.F = L.F;
  pp.n_q_heads = n_q_heads;
  pp.n_kv_heads = cv.n_kv_heads;
  pp.G = G;
  pp.qtiles = qtiles;
  pp.cb_int8 = L.bits <= 3 ? 1 : 0;
  pp.cb_unscale = std::ldexp(1.0f, -cb->table_exp);
  pp.pit32 = cb->pit32;
  pp.st32 = cb->st32;
  pp.frag = frag;
  pp.qfrag = qfrag;
  pp.scal = scal;
  static bool prep_attr = false;
  const int prep_smem = tqd::kPrepStageFloats * (int)sizeof(float);
  if (!prep_attr) {
    cudaError_t e = cudaFuncSetAttribute(tqd::prep_queries_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, prep_smem);
    if (e != cudaSuccess) return cuda_fail(e, "tq_logits: smem attribute");
    prep_attr = true;
  }
  dim3 pgrid((unsigned)(groups * qtiles), (unsigned)(L.m_pad > 0 ? 2 : 1));
  tqd::prep_queries_kernel<<<pgrid, 128, prep_smem, st>>>(pp);

  tqd::LogitsParams lp;
  lp.cv = cv;
  int ps = 0;
  while ((1 << ps) < cv.page_tokens) ++ps;
  lp.page_shift = ps;
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
  // a CTA stages at most kCtaPages block-table entries (its range may start
  // inside a page, hence the 2 spare entries)
  const int64_t kpc_cap = ((int64_t)(tqd::kCtaPages - 2) * cv.page_tokens / 64) * 64;
  if (kpc > kpc_cap) kpc = kpc_cap;
  lp.keys_per_cta = (int)kpc;
  lp.max_ctx = (int)max_ctx;
  lp.frag = frag;
  lp.qfrag = qfrag;
  lp.scal = scal;
  lp.out = out;
  lp.out_stride = out_stride;
  lp.th0 = cb->int8_hi[0];
  lp.th1 = cb->int8_hi[1];
  lp.tl0 = cb->int8_lo[0];
  lp.tl1 = cb->int8_lo[1];
  const uint16_t* M = cb->mag16;
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
