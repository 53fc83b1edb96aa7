// Fused attention logits straight from the packed keys.
//
// "TurboQuant explained" (a2a-mcp.org), §Stage 2 and §How it works: the
// query is rotated once (Pi q) and sketched once (S q); every logit is then
//   L = ||k|| ( sum_j (Pi q)_j c16[idx_j] + sqrt(pi/2)/m ||r|| sum_i (S q)_i s_i )
// evaluated from the indices and sign bits without dequantizing the key.
//
// Two kernels per call, chained by programmatic dependent launch:
//  * prep_queries_kernel: [Pi q ; S q] is split into parts of 32 rows; a
//    part is computed by one CTA on the tensor cores (bf16 hi + lo fragments
//    of [Pi ; S], pre-swizzled in the codebook, times the bf16 hi + lo split
//    of the queries, fp32 accumulation) and written as MMA B-fragment bytes
//    to the workspace.  Every part quantizes with a scale that needs no
//    other part: |(Pi q)_j| <= ||q|| (Pi is orthogonal) and
//    |(S q)_i| <= max_i ||S_i|| ||q||.
//  * logits_kernel (below), which streams the cache while the queries are
//    prepared.
//
// The logits kernel: every CTA owns an equal share of one sequence's keys;
// its warps stream 32-key units into shared-memory rings with bulk copies
// and run them through the tensor cores with the key operand built in
// registers:
//  - codebook term, b <= 3: m16n8k32 int8 MMAs.  c16 * 2^f is an integer of
//    at most 16 bits for every level, so a key element is two int8 slices;
//    eight stored codes form one byte-permute selector after a single mask,
//    and two permutes of 8-byte tables give the high and low slices of four
//    elements.  (Pi q) is quantized to 16-bit integers, also as two int8
//    slices; the slice products are accumulated exactly in int32 and
//    combined at the end.
//  - codebook term, b = 4: m16n8k16 fp16 MMAs on sign-magnitude codes (16
//    levels do not fit one 8-byte permute table), the query as fp16 hi + lo.
//  - sign term: m16n8k32 int8 MMAs.  The stored sign bits enter in place as
//    0 / 2^p bytes (one mask per operand register); S q is quantized to
//    integers z, and sum_i s_i z_i = sum_i z_i - 2 sum_i beta_i z_i.
// The MMA's N = 8 columns are the high and low slices of 4 queries.
// HBM traffic is the packed records plus the logits.

#include "stream.cuh"

namespace tqd {

constexpr int kSliceMax = 32639;   // |z| bound of Pi q: the high int8 slice stays in [-128, 127]
constexpr int kSliceMaxQ = 16319;  // |z| bound of S q: 2 z still splits into int8 slices
constexpr int kLogitsWarps = 4;    // warps per CTA
constexpr int kCtaPages = 64;      // block-table entries staged per CTA
constexpr int kPartRows = 32;      // rows of [Pi q ; S q] per preparation part

// CTAs of the logits kernel resident per SM, and its registers per thread:
// for d <= 128 few enough that a preparation CTA (128 threads x 64
// registers) still fits beside them (a warp scheduler's share of the
// register file is 16384: 5 x 88 x 32 + 64 x 32, or 4 x 104 x 32 + 64 x 32),
// so that no logits CTA has to wait for a preparation CTA to finish
__host__ __device__ constexpr int logits_min_blocks(int bits, int E) { return E >= 48 ? 4 : bits == 4 ? 4 : 5; }
__host__ __device__ constexpr int logits_max_regs(int bits, int E) {
  return E >= 48 ? 128 : logits_min_blocks(bits, E) == 5 ? 88 : 104;
}

// Per-warp shared-memory ring: a stage holds one 32-key unit, two 16-key
// tiles of 16 consecutive records each (16 * 16W bytes, contiguous in its
// page), then the two tiles' 16 norm slots (16 * NB <= 64 bytes each).
template <int W>
struct RingShape {
  static constexpr int kTileCode = 256 * W;
  static constexpr int kStageBytes = 2 * 256 * W + 128;
  static constexpr int kStages = kStageBytes <= 2304 ? 4 : 2;   // a power of two
};

struct PrepParams {
  const void* q;             // [batch][n_q_heads][d]
  tq_dtype dtype;
  int d, E, F;               // d_pad = 4E, m_pad = 4F
  int n_q_heads, n_kv_heads, G, qtiles;
  int cb_int8;               // codebook fragments as int8 slices (b <= 3) or fp16 hi / lo (b = 4)
  float cb_unscale;          // 2^-f
  float qjl_scale;           // sqrt(pi/2) / m
  float s_rowmax;            // >= max_i ||S_i||
  const uint4* qprep;        // [Pi ; S] bf16 hi + lo A fragments (tq_codebook::qprep_frag)
  uint2* frag;
  uint2* qfrag;
  float2* scal;
};

struct LogitsParams {
  tq::CacheView cv;
  int page_shift;            // log2(page_tokens)
  const int32_t* ctx_len;
  int n_kv_heads, n_q_heads, G, qtiles;
  int n_chunks;              // CTAs per (group, query tile) along the keys
  int units;                 // 32-key units of max_ctx
  int max_ctx;               // ctx_len values are clamped to [0, max_ctx]
  const uint2* frag;         // workspace: query fragments and scales
  const uint2* qfrag;
  const float2* scal;
  float* out;
  int64_t out_stride;
  uint32_t th0, th1, tl0, tl1;  // b <= 3: high / low int8 slices of c16 * 2^f, levels 0..7
  uint32_t lo0, lo1, hi0, hi1;  // b = 4: low / high bytes of the 8 fp16 magnitudes
  int pre_stages;            // ring stages filled before the query fragments are ready (1 .. 4)
};

// ---- loads of the workspace written by the preparation kernel (L2) ------------

__device__ __forceinline__ uint2 ld_cg(const uint2* p) {
  uint2 v;
  asm volatile("ld.global.cg.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ float2 ld_cg(const float2* p) {
  float2 v;
  asm volatile("ld.global.cg.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(p));
  return v;
}

// ---- MMA wrappers -------------------------------------------------------------------

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint4 a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
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

// ---- key operand decoding ---------------------------------------------------------

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

// ---- copies -------------------------------------------------------------------------

// The W words of one chunk from shared memory (4W-byte aligned).
template <int W>
__device__ __forceinline__ void lds_chunk(const uint8_t* src, uint32_t (&w)[W]) {
  if constexpr (W % 4 == 0) {
#pragma unroll
    for (int i = 0; i < W / 4; ++i) {
      const uint4 v = reinterpret_cast<const uint4*>(src)[i];
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  } else if constexpr (W % 2 == 0) {
#pragma unroll
    for (int i = 0; i < W / 2; ++i) {
      const uint2 v = reinterpret_cast<const uint2*>(src)[i];
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < W; ++i) w[i] = reinterpret_cast<const uint32_t*>(src)[i];
  }
}

__device__ __forceinline__ float lo_half(uint32_t v) {
  return __half2float(__ushort_as_half((unsigned short)(v & 0xFFFFu)));
}
__device__ __forceinline__ float hi_half(uint32_t v) {
  return __half2float(__ushort_as_half((unsigned short)(v >> 16)));
}
__device__ __forceinline__ uint16_t bf16_bits(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// ---- query preparation -----------------------------------------------------------
//
// Workspace: codebook fragments uint2 [gq][KC][32] (gq = group x query tile;
// KC = E/8 int8 k-steps, or E/4 fp16 k-steps for b = 4), QJL fragments uint2
// [gq][F/8][32], per-query scales float2 [batch * n_q_heads] = {c0, c1}.
// Lane (2 q + s) * 4 + t of a fragment holds slice s (0 high, 1 low) of
// query slot q for chunk t; byte e % 8 (half e % 4 for fp16) of it is row e
// of the k-step.  In the QJL part rows 8 kk .. 8 kk + 3 of a k-step hold the
// slices of 2 z, rows 8 kk + 4 .. 8 kk + 7 those of z (|z| <= kSliceMaxQ),
// matching the key operand of the logits kernel (sign bytes 2^(2 kk) beta
// and 2^(2 kk + 1) beta).

// Shared memory of one preparation part.
struct PrepSmem {
  uint16_t qsb[8][256 + 8];   // column 2 q + s: bf16 slice s of query slot q (padded rows: no bank conflicts)
  float4 ksum[2][32];         // k-split partial sums
  float qn2[4];               // ||q||^2 of the 4 query slots
};

// Part `r` of query tile gq (TQ §How it works: the query is pre-rotated once
// and reused over the whole context): rows [32 r, 32 r + 32) of
// [Pi q ; S q] for the 4 query slots of the tile, on the tensor cores
// (warp w: 16-row tile w % 2, k half w / 2), quantized and written as
// fragment bytes.  Every fragment byte of the part is written (zeros for
// padding rows and slots past G).  Part 0 also writes the slots' scales.
// All 128 threads of the CTA call it.
__device__ __forceinline__ void prep_part(const PrepParams& p, int gq, int r, PrepSmem& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int gi = gq / p.qtiles, qt = gq % p.qtiles;
  const int b = gi / p.n_kv_heads, kv = gi % p.n_kv_heads;
  const int64_t qbase = (int64_t)b * p.n_q_heads + kv * p.G + qt * 4;   // first query row of the tile
  const int nq = min(4, p.G - qt * 4);
  const int d = p.d, d16 = (d + 15) >> 4;

  const int mt = warp & 1, ksp = warp >> 1;
  const int kb = ksp * d16 / 2, ke = (ksp + 1) * d16 / 2;     // this warp's k-steps
  const uint4* afr = p.qprep + (size_t)(r * 2 + mt) * d16 * 64 + lane;
  uint4 af[4][2];
#pragma unroll
  for (int u = 0; u < 4; ++u)
    if (kb + u < ke) {
      af[u][0] = __ldg(afr + ((kb + u) * 2) * 32);
      af[u][1] = __ldg(afr + ((kb + u) * 2 + 1) * 32);
    }
  {
    // warp w: query slot w, lanes over k; every load in flight before any use
    float x[8];
    const int64_t qoff = (qbase + warp) * d;
    const bool valid = warp < nq;
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = 0.0f;
    if (valid) {
      if (p.dtype == TQ_BF16) {
        const __nv_bfloat16* qp = reinterpret_cast<const __nv_bfloat16*>(p.q) + qoff;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (lane + 32 * i < d) x[i] = __bfloat162float(qp[lane + 32 * i]);
      } else if (p.dtype == TQ_F16) {
        const __half* qp = reinterpret_cast<const __half*>(p.q) + qoff;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (lane + 32 * i < d) x[i] = __half2float(qp[lane + 32 * i]);
      } else {
        const float* qp = reinterpret_cast<const float*>(p.q) + qoff;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (lane + 32 * i < d) x[i] = qp[lane + 32 * i];
      }
    }
    float s2 = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int k = lane + 32 * i;
      if (k < 16 * d16) {
        const uint16_t hb = bf16_bits(x[i]);
        sm.qsb[2 * warp][k] = hb;
        sm.qsb[2 * warp + 1][k] = bf16_bits(x[i] - __bfloat162float(__ushort_as_bfloat16(hb)));
      }
      s2 = fmaf(x[i], x[i], s2);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    if (lane == 0) sm.qn2[warp] = s2;
  }
  __syncthreads();

  // column pair (2t, 2t+1) of the accumulator is (A q_hi, A q_lo) of query
  // slot t: rows g and g + 8 of tile mt are acc[0] + acc[1], acc[2] + acc[3]
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int kc = kb; kc < ke; kc += 4) {
    if (kc != kb) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (kc + u < ke) {
          af[u][0] = __ldg(afr + ((kc + u) * 2) * 32);
          af[u][1] = __ldg(afr + ((kc + u) * 2 + 1) * 32);
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (kc + u < ke) {
        const int k = kc + u;
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&sm.qsb[g][16 * k + 2 * t]);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(&sm.qsb[g][16 * k + 2 * t + 8]);
        mma_bf16(acc, af[u][0], b0, b1);
        mma_bf16(acc, af[u][1], b0, b1);
      }
  }
  if (ksp == 1) sm.ksum[mt][lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  __syncthreads();
  const float qn = sqrtf(sm.qn2[t]);
  const bool sk = r * kPartRows >= 4 * p.E;   // the part holds S q rows
  if (warp < 2) {
    const float4 o = sm.ksum[mt][lane];
    const float va = acc[0] + acc[1] + o.x + o.y, vb = acc[2] + acc[3] + o.z + o.w;
    const int Ep = sk ? p.F : p.E;
    const int zmax = sk ? kSliceMaxQ : kSliceMax;
    const float bound = sk ? p.s_rowmax * qn : qn;
    const float scale = bound > 0.0f ? (float)zmax * __frcp_rn(bound) : 0.0f;
    int e2 = 0;                       // b = 4: ||q|| in [2^(e2-1), 2^e2)
    if (!p.cb_int8 && qn > 0.0f) frexpf(qn, &e2);
    const float f16scale = p.cb_int8 ? 1.0f : ldexpf(1.0f, 14 - e2);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int l = r * kPartRows - (sk ? 4 * p.E : 0) + 16 * mt + g + 8 * hh;   // row within its half
      const float v = hh ? vb : va;
      const int tc = l / Ep, e = l % Ep;        // chunk, row within the chunk
      if (!sk && !p.cb_int8) {
        const float vs = v * f16scale;
        const __half hi = __float2half_rn(vs);
        const __half lo = __float2half_rn(vs - __half2float(hi));
        __half* fr = reinterpret_cast<__half*>(p.frag + ((int64_t)gq * (p.E / 4) + e / 4) * 32);
        fr[((2 * t) * 4 + tc) * 4 + (e & 3)] = hi;
        fr[((2 * t + 1) * 4 + tc) * 4 + (e & 3)] = lo;
      } else {
        int z = max(-zmax, min(zmax, __float2int_rn(v * scale)));
        if (sk && (e & 7) < 4) z *= 2;          // rows 8 kk .. 8 kk + 3 of a QJL k-step: 2 z
        const int zh = (z + 128) >> 8;          // floor((z + 128) / 256)
        const int zl = z - 256 * zh;            // in [-128, 127]
        int8_t* fr = reinterpret_cast<int8_t*>((sk ? p.qfrag : p.frag) + ((int64_t)gq * (Ep / 8) + e / 8) * 32);
        fr[((2 * t) * 4 + tc) * 8 + (e & 7)] = (int8_t)zh;
        fr[((2 * t + 1) * 4 + tc) * 8 + (e & 7)] = (int8_t)zl;
      }
    }
  }
  if (r == 0 && (int)threadIdx.x < nq) {
    const float qq = sqrtf(sm.qn2[threadIdx.x]);
    int e = 0;
    if (qq > 0.0f) frexpf(qq, &e);
    const float c0 = p.cb_int8 ? qq * (1.0f / (float)kSliceMax) * p.cb_unscale : ldexpf(1.0f, e - 14);
    const float c1 = p.qjl_scale * (p.s_rowmax * qq) * (1.0f / (float)kSliceMaxQ);
    p.scal[qbase + threadIdx.x] = make_float2(c0, c1);
  }
  __syncthreads();                  // the shared buffers may be reused
}

// Two-launch form: grid (parts, groups * qtiles), block 128; the logits
// kernel follows by programmatic dependent launch.
__global__ void __launch_bounds__(kLogitsWarps * 32) prep_queries_kernel(PrepParams p) {
  __shared__ PrepSmem sm;
  asm volatile("griddepcontrol.launch_dependents;");
  prep_part(p, blockIdx.y, blockIdx.x, sm);
}

// ---- logits -----------------------------------------------------------------------
//
// grid: (n_chunks, batch * n_kv_heads, query tiles of 4), block 128, dynamic
// smem kLogitsWarps * S * stage bytes.  CTA x of a (group, query tile) owns
// the 32-key units [x U / n_chunks, (x + 1) U / n_chunks) of the sequence
// (U = ceil(max_ctx / 32)): every CTA gets the same work to within one unit.
// Before it needs the query fragments a CTA stages its block-table entries
// (page_tokens is a power of two: page and slot are a shift and a mask) and
// every warp puts its first S units in flight: lane 0 issues bulk copies of
// the unit's 32 records and 32 norm slots into ring stage i % S, completing
// on that stage's mbarrier; then it waits for the preparation kernel
// (griddepcontrol.wait).  Warp w
// takes the CTA's units w, w + 4, ...  The two tiles of a unit are read
// before either is computed, so their MMA chains interleave; a tile whose
// page is bad or that lies past the context computes on stale bytes and
// stores nothing.
// Sign term: k-step kk of a QJL word uses bit planes 2 kk and 2 kk + 1 in
// place (one mask per operand register), weighted 2^(2 kk + 1) after the
// query side's 2 z / z slots; a Horner step (x 4) between k-steps brings
// every k-step of a word to weight 2^(2 n - 1) (n k-steps in the word), and
// words are scaled to the common weight 128.
template <int BITS, int E, int F>
__global__ void __maxnreg__(logits_max_regs(BITS, E)) logits_kernel(LogitsParams p) {
  constexpr bool kInt8 = BITS <= 3;
  constexpr int KC = kInt8 ? E / 8 : E / 4;   // codebook MMA k-steps
  constexpr int KQ = F / 8;                   // sign-term MMA k-steps
  constexpr int q0 = BITS == 1 ? (E + 31) / 32 : BITS == 2 ? E / 16
                   : BITS == 3 ? 3 * (E / 32) + 2 * ((E % 32) / 16) : E / 8;
  constexpr int QW = (F + 31) / 32;           // QJL words per chunk
  constexpr int W = q0 + QW;
  constexpr int NB = F > 0 ? 4 : 2;
  using RS = RingShape<W>;
  constexpr int S = RS::kStages;
  constexpr int TILE = RS::kTileCode;
  constexpr int STAGE = RS::kStageBytes;
  extern __shared__ __align__(16) uint8_t ring_smem[];
  __shared__ int64_t page_base[kCtaPages];    // byte offset of this head's block, -1 if bad
  __shared__ uint64_t ring_bar[kLogitsWarps][4];   // one per ring stage (S <= 4)

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int gi = blockIdx.y;
  const int b = gi / p.n_kv_heads, h = gi % p.n_kv_heads;
  const int qt = blockIdx.z;
  const int u0 = (int)((int64_t)blockIdx.x * p.units / p.n_chunks);
  const int u1 = (int)((int64_t)(blockIdx.x + 1) * p.units / p.n_chunks);
  const int k0 = 32 * u0;
  const int kend = min(32 * u1, p.max_ctx);
  const int ps = p.page_shift;
  const int P = 1 << ps;
  const int first_page = k0 >> ps;
  const int n_pgx = k0 < kend ? ((kend - 1) >> ps) - first_page + 1 : 0;   // <= kCtaPages
  const int ctx = min(p.ctx_len[b], p.max_ctx);
  const int jt = threadIdx.x;
  static_assert(kCtaPages <= kLogitsWarps * 32, "one block-table entry per thread");
  const int64_t pg = jt < n_pgx ? p.cv.block_table[(int64_t)b * p.cv.max_pages + first_page + jt] : 0;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < S; ++s) mbar_init(&ring_bar[warp][s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  const int k1 = min(kend, ctx);     // keys [k0, k1) of this CTA (none when k1 <= k0)
  const bool has_keys = k0 < k1;
  bool bad = false;
  if (jt < n_pgx) {
    const bool valid = pg >= 0 && pg < p.cv.n_pages;
    page_base[jt] = valid ? pg * p.cv.page_bytes + (int64_t)h * p.cv.head_block_bytes : -1;
    // pages past the context are not used: an invalid entry there is no error
    if (!valid && has_keys && jt <= ((k1 - 1) >> ps) - first_page) {
      bad = true;
      report(p.cv.err, TQ_DEV_ERR_PAGE);
    }
  }
  // fast path: every used page valid and 32-key units never straddle a page
  const bool fast = !__syncthreads_or(bad) && P >= 32;   // also publishes the barriers' init

  const int n_units = has_keys ? (k1 - k0 + 31) >> 5 : 0;
  const int n_my = warp < n_units ? (n_units - warp + kLogitsWarps - 1) / kLogitsWarps : 0;
  const uint8_t* ring = ring_smem + warp * S * STAGE;
  const uint32_t ring_s = smem_addr(ring);
  const int64_t norm_off = (int64_t)P * (16 * W);   // norm slots follow the P records
  const uint64_t pol = evict_first_policy();   // the cache is streamed once per call

  // lane 0 copies unit i of this warp (32 records + 32 norm slots) into stage
  // i % S with bulk copies completing on that stage's barrier
  auto issue = [&](int i) {
    if (lane != 0) return;
    uint64_t* bar = &ring_bar[warp][i & (S - 1)];
    const uint32_t dst = ring_s + (i & (S - 1)) * STAGE;
    const int ubase = k0 + 32 * (warp + kLogitsWarps * i);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // earlier reads of the stage first
    if (fast) {
      // one page holds the whole unit (records past the context are read and not used)
      const int slot = ubase & (P - 1);
      const uint8_t* hb = p.cv.pages + page_base[(ubase >> ps) - first_page];
      mbar_arrive_tx(bar, 2 * TILE + 32 * NB);
      bulk_copy(dst, hb + (int64_t)slot * (16 * W), 2 * TILE, bar, pol);
      bulk_copy(dst + 2 * TILE, hb + norm_off + slot * NB, 32 * NB, bar, pol);
      return;
    }
    uint32_t bytes = 0;
    int64_t off[2] = {-1, -1};
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int base = ubase + 16 * hf;
      if (base < k1) off[hf] = page_base[(base >> ps) - first_page];
      if (off[hf] >= 0) bytes += TILE + 16 * NB;
    }
    mbar_arrive_tx(bar, bytes);        // 0 bytes: the phase completes on the arrival alone
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      if (off[hf] < 0) continue;
      const int slot = (ubase + 16 * hf) & (P - 1);
      const uint8_t* hb = p.cv.pages + off[hf];
      bulk_copy(dst + hf * TILE, hb + (int64_t)slot * (16 * W), TILE, bar, pol);
      bulk_copy(dst + 2 * TILE + 16 * NB * hf, hb + norm_off + slot * NB, 16 * NB, bar, pol);
    }
  };
  // the first p.pre_stages units now, the rest of the ring once the query
  // fragments are in registers (they would queue behind the copies at the SM)
  int issued = 0;                    // units whose copies were issued
#pragma unroll
  for (int s = 0; s < S; ++s)
    if (s < n_my && s < p.pre_stages) issue(issued++);

  const int gq = gi * p.qtiles + qt;
  // the query fragments and scales come from the preparation kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  uint2 bq[KC];
  const uint2* fsrc = p.frag + (int64_t)gq * KC * 32 + lane;
#pragma unroll
  for (int kk = 0; kk < KC; ++kk) bq[kk] = ld_cg(fsrc + kk * 32);
  uint2 bz[KQ > 0 ? KQ : 1];
  float zsumf = 0.0f;
  if constexpr (KQ > 0) {
    const uint2* qsrc = p.qfrag + (int64_t)gq * KQ * 32 + lane;
#pragma unroll
    for (int kk = 0; kk < KQ; ++kk) bz[kk] = ld_cg(qsrc + kk * 32);
    // sum_i z_i of query t from its own fragments: weights 1 on the 2 z
    // slots and 2 on the z slots give 2 sum z in columns (2t, 2t+1)
    int zs[4] = {0, 0, 0, 0};
#pragma unroll
    for (int kk = 0; kk < KQ; ++kk) mma_s8s8(zs, 0x01010101u, 0x01010101u, 0x02020202u, 0x02020202u, bz[kk]);
    zsumf = 0.5f * (float)(256 * zs[0] + zs[1]);
  }
  const int qidx = qt * 4 + t;                  // this thread's query within the group
  const bool qvalid = qidx < p.G;
  const int hq = h * p.G + (qvalid ? qidx : 0);
  const float2 sc = ld_cg(p.scal + (int64_t)b * p.n_q_heads + hq);
  const float c0 = sc.x;
  const float c1 = F > 0 ? sc.y : 0.0f;
  float* orow = p.out + ((int64_t)b * p.n_q_heads + hq) * p.out_stride;
  // logits of rows g (la) and g + 8 (lb) of one tile, for query t
  auto tile = [&](const uint32_t (&wa)[W], const uint32_t (&wb)[W], uint32_t na, uint32_t nb,
                  float& la, float& lb) {
    float cba, cbb;
    if constexpr (kInt8) {
      // codebook term: int8 slices of c16 * 2^f against those of (Pi q)
      int ah[4] = {0, 0, 0, 0}, al[4] = {0, 0, 0, 0};
#pragma unroll
      for (int kk = 0; kk < KC; ++kk) {
        const uint32_t sa = code_selector<BITS, E>(wa, kk);
        const uint32_t sb = code_selector<BITS, E>(wb, kk);
        const uint32_t sa2 = sa >> 16, sb2 = sb >> 16;
        mma_s8s8(ah, prmt(p.th0, p.th1, sa), prmt(p.th0, p.th1, sb), prmt(p.th0, p.th1, sa2),
                 prmt(p.th0, p.th1, sb2), bq[kk]);
        mma_s8s8(al, prmt(p.tl0, p.tl1, sa), prmt(p.tl0, p.tl1, sb), prmt(p.tl0, p.tl1, sa2),
                 prmt(p.tl0, p.tl1, sb2), bq[kk]);
      }
      // columns 2t / 2t+1: high / low slice of query t.  256 hh + hl + lh
      // stays below 2^31 (|hh| <= 2^22 for d <= 256).
      cba = fmaf(256.0f, (float)(256 * ah[0] + ah[1] + al[0]), (float)al[1]);
      cbb = fmaf(256.0f, (float)(256 * ah[2] + ah[3] + al[2]), (float)al[3]);
    } else {
      float acc0[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < KC; ++ks) {
        uint32_t a0, a2, a1, a3;
        decode_nibble_pair(wa, ks, p, a0, a2);
        decode_nibble_pair(wb, ks, p, a1, a3);
        mma_f16(acc0, a0, a1, a2, a3, bq[ks]);
      }
      // columns 2t (hi) and 2t+1 (lo) belong to query t of this tile
      cba = acc0[0] + acc0[1];
      cbb = acc0[2] + acc0[3];
    }
    if constexpr (F > 0) {
      // sign term: in-place bit planes against the int8 slices of 2 z / z
      int qa[4] = {0, 0, 0, 0};                 // 128 sum beta z (hi, lo columns)
#pragma unroll
      for (int w = 0; w < QW; ++w) {
        const int nk = min(4, (F - 32 * w) / 8);   // k-steps of this word (4, or 2 for a half word)
        int a4[4] = {0, 0, 0, 0};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (k < nk) {
            if (k > 0) {
#pragma unroll
              for (int r = 0; r < 4; ++r) a4[r] *= 4;
            }
            const uint32_t m0 = 0x01010101u << (2 * k), m1 = m0 << 1;
            mma_u8s8(a4, wa[q0 + w] & m0, wb[q0 + w] & m0, wa[q0 + w] & m1, wb[q0 + w] & m1, bz[4 * w + k]);
          }
        }
        const int sh = 6 - 2 * (nk - 1);           // weight 2^(2 nk - 1) -> 128
#pragma unroll
        for (int r = 0; r < 4; ++r) qa[r] += a4[r] << sh;
      }
      // sum_i s_i z_i = sum z - 2 sum beta z
      const float ta = fmaf(-1.0f / 64.0f, (float)(256 * qa[0] + qa[1]), zsumf);
      const float tb = fmaf(-1.0f / 64.0f, (float)(256 * qa[2] + qa[3]), zsumf);
      const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&na));   // ||k||, ||r||
      const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&nb));
      la = fa.x * fmaf(c1 * fa.y, ta, c0 * cba);
      lb = fb.x * fmaf(c1 * fb.y, tb, c0 * cbb);
    } else {
      la = lo_half(na) * (c0 * cba);
      lb = lo_half(nb) * (c0 * cbb);
    }
  };

#pragma unroll
  for (int s = 1; s < S; ++s)
    if (issued == s && s < n_my) issue(issued++);
  bool timed_out = false;
  for (int i = 0; i < n_my; ++i) {
    if (!mbar_wait(&ring_bar[warp][i & (S - 1)], (uint32_t)(i / S) & 1u)) {
      timed_out = true;
      break;
    }
    const int ubase = k0 + 32 * (warp + kLogitsWarps * i);
    const uint8_t* stg = ring + (i & (S - 1)) * STAGE;
    uint32_t wa0[W], wb0[W], wa1[W], wb1[W];
    lds_chunk<W>(stg + g * (16 * W) + t * (4 * W), wa0);
    lds_chunk<W>(stg + (g + 8) * (16 * W) + t * (4 * W), wb0);
    lds_chunk<W>(stg + TILE + g * (16 * W) + t * (4 * W), wa1);
    lds_chunk<W>(stg + TILE + (g + 8) * (16 * W) + t * (4 * W), wb1);
    uint32_t na0, nb0, na1, nb1;
    if constexpr (NB == 4) {
      const uint32_t* nsl = reinterpret_cast<const uint32_t*>(stg + 2 * TILE);
      na0 = nsl[g]; nb0 = nsl[g + 8]; na1 = nsl[16 + g]; nb1 = nsl[24 + g];
    } else {
      const uint8_t* nsl = stg + 2 * TILE;
      na0 = *reinterpret_cast<const unsigned short*>(nsl + 2 * g);
      nb0 = *reinterpret_cast<const unsigned short*>(nsl + 2 * (g + 8));
      na1 = *reinterpret_cast<const unsigned short*>(nsl + 32 + 2 * g);
      nb1 = *reinterpret_cast<const unsigned short*>(nsl + 32 + 2 * (g + 8));
    }
    bool ok0 = true, ok1 = ubase + 16 < k1;
    if (!fast) {
      ok0 = page_base[(ubase >> ps) - first_page] >= 0;
      ok1 = ok1 && page_base[((ubase + 16) >> ps) - first_page] >= 0;
    }
    __syncwarp();                    // every read of this stage precedes its reuse
    if (i + S < n_my) {
      issue(i + S);
      issued = i + S + 1;
    }
    float la0, lb0, la1, lb1;
    tile(wa0, wb0, na0, nb0, la0, lb0);
    tile(wa1, wb1, na1, nb1, la1, lb1);
    if (qvalid) {
      const int r = ubase + g;
      if (fast && ubase + 32 <= k1) {
        __stcs(orow + r, la0);
        __stcs(orow + r + 8, lb0);
        __stcs(orow + r + 16, la1);
        __stcs(orow + r + 24, lb1);
      } else {
        if (ok0 && r < k1) __stcs(orow + r, la0);
        if (ok0 && r + 8 < k1) __stcs(orow + r + 8, lb0);
        if (ok1 && r + 16 < k1) __stcs(orow + r + 16, la1);
        if (ok1 && r + 24 < k1) __stcs(orow + r + 24, lb1);
      }
    }
  }
  if (timed_out) {
    // report, then let the copies already issued land (the last unit issued
    // into each stage; each wait bounded) before the CTA's shared memory is
    // released
    if (lane == 0) report(p.cv.err, TQ_DEV_ERR_TIMEOUT);
    for (int u = max(0, issued - S); u < issued; ++u) mbar_wait(&ring_bar[warp][u & (S - 1)], (uint32_t)(u / S) & 1u);
  }
}

}  // namespace tqd

namespace tq {

struct LogitsWs {
  size_t frag, qfrag, scal, total;
};

static LogitsWs logits_ws_layout(const tq_codebook* cb, int64_t groups, int G, int64_t batch_heads) {
  auto al = [](size_t n) { return (n + 255) / 256 * 256; };
  const int qtiles = (G + 3) / 4;
  const int kc = cb->lay.bits <= 3 ? cb->lay.E / 8 : cb->lay.E / 4;
  LogitsWs w;
  w.frag = al((size_t)groups * qtiles * kc * 32 * sizeof(uint2));
  w.qfrag = al((size_t)groups * qtiles * (cb->lay.F / 8) * 32 * sizeof(uint2));
  w.scal = al((size_t)batch_heads * sizeof(float2));
  w.total = w.frag + w.qfrag + w.scal;
  return w;
}

size_t logits_workspace(const tq_codebook* cb, int64_t groups, int G) {
  return logits_ws_layout(cb, groups, G, groups * G).total;
}

template <int BITS, int E, int F>
static tq_status run_logits(const tqd::LogitsParams& p, const tqd::PrepParams& pp, int parts, int64_t groups,
                            int qtiles, cudaStream_t st) {
  constexpr int q0 = BITS == 1 ? (E + 31) / 32 : BITS == 2 ? E / 16
                   : BITS == 3 ? 3 * (E / 32) + 2 * ((E % 32) / 16) : E / 8;
  constexpr int W = q0 + (F + 31) / 32;
  using RS = tqd::RingShape<W>;
  const int smem = tqd::kLogitsWarps * RS::kStages * RS::kStageBytes;
  static PerDeviceOnce attr;           // per template instance
  if (const int dev_ = current_device(); attr.need(dev_)) {
    cudaError_t e = cudaFuncSetAttribute(tqd::logits_kernel<BITS, E, F>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "tq_logits: smem attribute");
    // the preparation kernel asks for the logits kernel's shared-memory
    // split, or its CTAs would keep logits CTAs off their SMs
    e = cudaFuncSetAttribute(tqd::prep_queries_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return cuda_fail(e, "tq_logits: carveout attribute");
    attr.mark(dev_);
  }
  tqd::prep_queries_kernel<<<dim3((unsigned)parts, (unsigned)(groups * qtiles)), tqd::kLogitsWarps * 32, 0, st>>>(pp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "tq_logits: query preparation launch");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.n_chunks, (unsigned)groups, (unsigned)qtiles);
  cfg.blockDim = dim3(tqd::kLogitsWarps * 32);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, tqd::logits_kernel<BITS, E, F>, p);
  if (e != cudaSuccess) return cuda_fail(e, "tq_logits launch");
  return TQ_OK;
}

template <int BITS>
static tq_status dispatch_logits(const Layout& L, const tqd::LogitsParams& p, const tqd::PrepParams& pp,
                                 int parts, int64_t groups, int qtiles, cudaStream_t st) {
  if (L.E == 32 && L.F == 32) return run_logits<BITS, 32, 32>(p, pp, parts, groups, qtiles, st);
  if (L.E == 32 && L.F == 0) return run_logits<BITS, 32, 0>(p, pp, parts, groups, qtiles, st);
  if (L.E == 16 && L.F == 16) return run_logits<BITS, 16, 16>(p, pp, parts, groups, qtiles, st);
  if (L.E == 16 && L.F == 0) return run_logits<BITS, 16, 0>(p, pp, parts, groups, qtiles, st);
  if (L.E == 64 && L.F == 64) return run_logits<BITS, 64, 64>(p, pp, parts, groups, qtiles, st);
  if (L.E == 64 && L.F == 0) return run_logits<BITS, 64, 0>(p, pp, parts, groups, qtiles, st);
  if (L.E == 48 && L.F == 48) return run_logits<BITS, 48, 48>(p, pp, parts, groups, qtiles, st);
  if (L.E == 48 && L.F == 0) return run_logits<BITS, 48, 0>(p, pp, parts, groups, qtiles, st);
  return fail(TQ_EUNSUPPORTED, "tq_logits: no kernel for this (d, m)");
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
  if (ws_bytes < wl.total || !ws) return fail(TQ_EINVAL, "tq_logits: workspace too small");
  if (max_ctx == 0 || batch == 0) return TQ_OK;
  if (groups > 65535 || groups * qtiles > 65535) return fail(TQ_EINVAL, "tq_logits: batch * n_kv_heads too large");
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  uint2* frag = reinterpret_cast<uint2*>(wsb);
  uint2* qfrag = reinterpret_cast<uint2*>(wsb + wl.frag);
  float2* scal = reinterpret_cast<float2*>(wsb + wl.frag + wl.qfrag);

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
  pp.cb_int8 = L.bits <= 3 ? 1 : 0;
  pp.cb_unscale = std::ldexp(1.0f, -cb->table_exp);
  pp.qjl_scale = (float)cb->qjl_scale;
  // |(S q)_i| <= ||S_i|| ||q||: the float bound is rounded up
  pp.s_rowmax = (float)(cb->s_row_norm_max * (1.0 + 1e-6));
  pp.qprep = cb->qprep_frag;
  pp.frag = frag;
  pp.qfrag = qfrag;
  pp.scal = scal;
  const int parts = (L.d_pad + L.m_pad) / tqd::kPartRows;

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
  // Every CTA slot of the GPU (SMs x resident CTAs) gets one CTA, each an
  // equal share (to one 32-key unit) of one sequence's keys; more CTAs when a
  // share would need more than kCtaPages - 2 block-table entries, and then as
  // many as fill whole waves of the slots (a last, partly filled wave would
  // run at a fraction of the GPU for as long as a full one).
  const int64_t units = (max_ctx + 31) / 32;
  const int64_t tiles = groups * qtiles;
  const int64_t slots = (int64_t)device_sm_count() * tqd::logits_min_blocks(L.bits, L.E);
  int64_t n_chunks = std::max<int64_t>(1, slots / tiles);
  const int64_t max_units_cta = (int64_t)(tqd::kCtaPages - 2) * cv.page_tokens / 32;
  n_chunks = std::max<int64_t>(n_chunks, (units + max_units_cta - 1) / max_units_cta);
  n_chunks = std::min<int64_t>(n_chunks, units);
  const int64_t waves = (n_chunks * tiles + slots - 1) / slots;
  n_chunks = std::min<int64_t>(std::max<int64_t>(n_chunks, waves * slots / tiles), units);
  if (n_chunks > 0x7fffffffLL) return fail(TQ_EINVAL, "tq_logits: context too long");
  lp.n_chunks = (int)n_chunks;
  lp.units = (int)units;
  lp.max_ctx = (int)max_ctx;
  lp.frag = frag;
  lp.qfrag = qfrag;
  lp.scal = scal;
  lp.out = out;
  lp.out_stride = out_stride;
  lp.pre_stages = 1;
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
  switch (L.bits) {
    case 1: return dispatch_logits<1>(L, lp, pp, parts, groups, qtiles, st);
    case 2: return dispatch_logits<2>(L, lp, pp, parts, groups, qtiles, st);
    case 3: return dispatch_logits<3>(L, lp, pp, parts, groups, qtiles, st);
    case 4: return dispatch_logits<4>(L, lp, pp, parts, groups, qtiles, st);
  }
  return fail(TQ_EUNSUPPORTED, "tq_logits: bits");
}

}  // namespace tq
