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
//    entry, also as two int8 slices; the slice products are accumulated
//    exactly in int32 and combined at the end.
//  * codebook term, b = 4: m16n8k16 fp16 MMAs on sign-magnitude codes (16
//    levels do not fit one 8-byte permute table), the query as fp16 hi + lo.
//  * sign term: m16n8k32 int8 MMAs.  The stored sign bits are spread to 0/1
//    bytes with one shift and mask per 4 bits; S q is quantized to 16-bit
//    integers z, and sum_i s_i z_i = sum_i z_i - 2 sum_i beta_i z_i.
// The MMA's N = 8 columns are the high and low slices of 4 queries.
//
// Two kernels per call, chained by programmatic dependent launch:
//  1. prep_queries_kernel: one thread-block cluster per (KV group, tile of 4
//     queries); each CTA computes 32 (or 64) rows of [Pi q ; S q] for the 4
//     queries, the CTAs exchange their partial maxima through distributed
//     shared memory, and each writes its rows as MMA B-fragment bytes.
//  2. logits_kernel: every warp owns a set of 16-key tiles and copies them
//     (as many as its ring holds) into shared memory with cp.async before it
//     waits for the query fragments, so the cache stream is in flight while
//     the queries are prepared.  Thread t of an MMA quad owns chunk t of every
//     record.
// HBM traffic is the packed records plus the logits.

#include "tq_internal.cuh"

namespace tqd {

// ---- query preparation ------------------------------------------------------
// Workspace: codebook fragments uint2 [gq][KC][32] (KC = E/8 int8 k-steps, or
// E/4 fp16 k-steps for b = 4), QJL fragments uint2 [gq][F/8][32]
// (gq = group x query tile), per-query scalars float4 [batch * n_q_heads] =
// {codebook scale, QJL step, 0, 0}.  Lane (2 * query + slice) * 4 + t of
// an int8 fragment holds the slice (0 high, 1 low) of chunk t's elements.

constexpr int kSliceMax = 32639;   // |z| bound: the high int8 slice stays in [-128, 127]
constexpr int kSliceMaxQ = 16319;  // |z| bound of S q: 2 z still splits into int8 slices
constexpr int kPrepThreads = 128;
constexpr int kMaxClusterCtas = 8;

struct PrepParams {
  const void* q;
  tq_dtype dtype;
  int d, d_pad, m_pad, E, F;   // E, F: coordinates / QJL rows per chunk
  int n_q_heads, n_kv_heads, G, qtiles;
  int cb_int8;           // codebook fragments as int8 slices (b <= 3) or fp16 hi/lo (b = 4)
  float cb_unscale;      // 2^-f: c16 * 2^f are the integer table entries
  const float* pi32;     // Pi [d_pad][d], rows >= d zero
  const float* s32;      // S  [m_pad][d], rows >= m zero
  uint2* frag;
  uint2* qfrag;
  float4* scal;
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// Stores v into the same shared variable of CTA `rank` of this cluster.
__device__ __forceinline__ void st_cluster(const void* local, uint32_t rank, float v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
}
__device__ __forceinline__ void st_cluster(const void* local, uint32_t rank, int v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
  asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(remote), "r"(v) : "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Sums 32 per-lane partial values across the warp so that lane l ends with
// the total of value l (a butterfly that halves the values each round).
__device__ __forceinline__ float reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = upper ? v[i] : v[i + o];
      const float keep = upper ? v[i + o] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return v[0];
}

// Rotates and sketches each query once (TQ §How it works: the query is
// pre-rotated once and reused over the whole context).
// grid: (nblk, groups * qtiles), cluster (nblk, 1, 1); CTA `rank` computes
// rows [rank * RB, rank * RB + RB) of [Pi q ; S q] for the 4 queries of its
// tile (RB = 4 * RPW rows; d_pad is a multiple of RB, so a block never
// straddles Pi q / S q).  The block's RB x d matrix rows are copied into
// shared memory with every cp.async in flight while the queries load.  Warp
// w: rows w * RPW .. w * RPW + RPW - 1 of the block, lanes split the sum over
// k.  The CTAs of the cluster exchange their per-query maxima through
// distributed shared memory; every fragment byte of the tile is written
// (zeros for padding rows and for query slots past G), so the workspace
// needs no clearing.
// QJL fragments: in the MMA k-step of rows 8 kk .. 8 kk + 7 of a chunk, the
// slots of rows 8 kk .. 8 kk + 3 hold the slices of 2 z and those of rows
// 8 kk + 4 .. 8 kk + 7 the slices of z (|z| <= kSliceMaxQ), matching the key
// operand of the logits kernel, whose sign bytes there are 2^(2 kk) beta and
// 2^(2 kk + 1) beta.
template <int RPW>
__global__ void __launch_bounds__(kPrepThreads) prep_queries_kernel(PrepParams p) {
  asm volatile("griddepcontrol.launch_dependents;");
  cluster_arrive_relaxed();          // phase 1: every CTA of the cluster has started
  constexpr int RB = 4 * RPW;        // rows per CTA
  extern __shared__ __align__(16) float mrows[];   // [RB][d]
  __shared__ float qs[4][256];
  __shared__ float qnorm2[4];
  __shared__ float wred[4][4];
  __shared__ float pmax[kMaxClusterCtas][4];   // partial maxima pushed by each rank
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = blockIdx.x, nblk = gridDim.x;
  const int gq = blockIdx.y;
  const int gi = gq / p.qtiles, qt = gq % p.qtiles;
  const int b = gi / p.n_kv_heads, kv = gi % p.n_kv_heads;
  const int d = p.d;
  const int64_t qbase = (int64_t)b * p.n_q_heads + kv * p.G + qt * 4;   // first query row of the tile
  const int nq = min(4, p.G - qt * 4);

  const int row0 = rank * RB;
  const bool sk = row0 >= p.d_pad;                 // this block holds S q rows
  const int prow0 = sk ? row0 - p.d_pad : row0;    // first row within its part
  {
    const float4* src = reinterpret_cast<const float4*>((sk ? p.s32 : p.pi32) + (size_t)prow0 * d);
    const uint32_t dst = smem_addr(mrows);
    for (int c = threadIdx.x; c < RB * d / 4; c += kPrepThreads)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + 16 * c), "l"(src + c) : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  // the 4 queries of the tile (zeros for slots past G) and their squared norms
  {
    float s2 = 0.0f;
    for (int k = lane; k < d; k += 32) {
      const float x = warp < nq ? load_elem(p.q, (qbase + warp) * d + k, p.dtype) : 0.0f;
      qs[warp][k] = x;
      s2 = fmaf(x, x, s2);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    if (lane == 0) qnorm2[warp] = s2;
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  // val[h]: lane l holds row prow0 + w * RPW + 8 h + l / 4 of query slot l % 4
  float val[RPW / 8];
#pragma unroll
  for (int h = 0; h < RPW / 8; ++h) {
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
    const float* Mh = mrows + (warp * RPW + 8 * h) * d;
    for (int k = lane; k < d; k += 32) {
      const float x0 = qs[0][k], x1 = qs[1][k], x2 = qs[2][k], x3 = qs[3][k];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float m = Mh[j * d + k];
        acc[4 * j] = fmaf(m, x0, acc[4 * j]);
        acc[4 * j + 1] = fmaf(m, x1, acc[4 * j + 1]);
        acc[4 * j + 2] = fmaf(m, x2, acc[4 * j + 2]);
        acc[4 * j + 3] = fmaf(m, x3, acc[4 * j + 3]);
      }
    }
    val[h] = reduce_scatter32(acc, lane);
  }
  const int qi = lane & 3;           // this lane's query slot

  // partial max |v| of this block per query slot
  float mx = 0.0f;
#pragma unroll
  for (int h = 0; h < RPW / 8; ++h) mx = fmaxf(mx, fabsf(val[h]));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
  if (lane < 4) wred[warp][lane] = mx;
  __syncthreads();
  cluster_wait();                    // phase 1 complete: the peers' shared memory exists
  if (threadIdx.x < 4 * nblk) {
    const int dst = threadIdx.x >> 2, qq = threadIdx.x & 3;
    const float m4 = fmaxf(fmaxf(wred[0][qq], wred[1][qq]), fmaxf(wred[2][qq], wred[3][qq]));
    st_cluster(&pmax[rank][qq], (uint32_t)dst, m4);
  }
  cluster_sync();                    // phase 2: every partial maximum delivered; no remote access after this

  const int nb_pi = p.d_pad / RB;    // ranks [0, nb_pi) hold Pi q rows
  float mpi = 0.0f, msk = 0.0f;
  for (int r = 0; r < nblk; ++r) {
    if (r < nb_pi) mpi = fmaxf(mpi, pmax[r][qi]);
    else msk = fmaxf(msk, pmax[r][qi]);
  }
  int e2 = 0;                        // b = 4: 2^(14 - e2) puts |(Pi q)_j| <= ||q|| below 2^14
  {
    const float qn = sqrtf(qnorm2[qi]);
    if (qn > 0.0f) frexpf(qn, &e2);
  }
  const float step = sk ? (msk > 0.0f ? msk / (float)kSliceMaxQ : 0.0f)
                        : (mpi > 0.0f ? mpi / (float)kSliceMax : 0.0f);
#pragma unroll
  for (int h = 0; h < RPW / 8; ++h) {
    const int l = prow0 + warp * RPW + 8 * h + (lane >> 2);   // row within its part
    const float v = val[h];
    if (!sk && !p.cb_int8) {
      const float vs = v * ldexpf(1.0f, 14 - e2);
      const __half hi = __float2half_rn(vs);
      const __half lo = __float2half_rn(vs - __half2float(hi));
      const int t = l / p.E, e4 = l % p.E;
      __half* fr = reinterpret_cast<__half*>(p.frag + ((int64_t)gq * (p.E / 4) + e4 / 4) * 32);
      const int half_idx = ((e4 >> 1) & 1) * 2 + (e4 & 1);
      fr[((2 * qi) * 4 + t) * 4 + half_idx] = hi;
      fr[((2 * qi + 1) * 4 + t) * 4 + half_idx] = lo;
      continue;
    }
    const int Ep = sk ? p.F : p.E;
    const int t = l / Ep, e = l % Ep;
    const int kk = e / 8, hreg = (e >> 2) & 1, by = e & 3;
    const int zmax = sk ? kSliceMaxQ : kSliceMax;
    int z = 0;
    if (step > 0.0f) z = max(-zmax, min(zmax, __float2int_rn(v / step)));
    if (sk && hreg == 0) z *= 2;              // rows 8 kk .. 8 kk + 3: 2 z
    const int zh = (z + 128) >> 8;            // floor((z + 128) / 256)
    const int zl = z - 256 * zh;              // in [-128, 127]
    int8_t* fr = reinterpret_cast<int8_t*>((sk ? p.qfrag : p.frag) + ((int64_t)gq * (Ep / 8) + kk) * 32);
    fr[((2 * qi) * 4 + t) * 8 + hreg * 4 + by] = (int8_t)zh;
    fr[((2 * qi + 1) * 4 + t) * 8 + hreg * 4 + by] = (int8_t)zl;
  }
  if (rank == 0 && threadIdx.x < nq) {
    const int qq = threadIdx.x;
    float m0 = 0.0f, m1 = 0.0f;
    for (int r = 0; r < nblk; ++r) {
      if (r < nb_pi) m0 = fmaxf(m0, pmax[r][qq]);
      else m1 = fmaxf(m1, pmax[r][qq]);
    }
    float c0;
    if (p.cb_int8) {
      c0 = (m0 > 0.0f ? m0 / (float)kSliceMax : 0.0f) * p.cb_unscale;
    } else {
      int e = 0;
      const float qn = sqrtf(qnorm2[qq]);
      if (qn > 0.0f) frexpf(qn, &e);
      c0 = ldexpf(1.0f, e - 14);
    }
    const float zstep = m1 > 0.0f ? m1 / (float)kSliceMaxQ : 0.0f;
    p.scal[qbase + qq] = make_float4(c0, zstep, 0.0f, 0.0f);
  }
}

// ---- logits ---------------------------------------------------------------------

constexpr int kLogitsWarps = 4;     // warps per CTA
constexpr int kLogitsMinBlocks = 6; // CTAs resident per SM (registers <= 80 per thread)
constexpr int kCtaPages = 64;       // block-table entries staged per CTA

// Per-warp shared-memory ring: a stage holds one 32-key unit, two 16-key
// tiles of 16 consecutive records each (16 * 16W bytes, contiguous in its
// page), then the two tiles' 16 norm slots (16 * NB <= 64 bytes each).
template <int W>
struct RingShape {
  static constexpr int kTileCode = 256 * W;
  static constexpr int kStageBytes = 2 * 256 * W + 128;
  static constexpr int kStages = kStageBytes <= 2304 ? 4 : 2;   // a power of two
};

struct LogitsParams {
  tq::CacheView cv;
  int page_shift;            // log2(page_tokens)
  const int32_t* ctx_len;
  int n_kv_heads, n_q_heads, G, qtiles;
  int keys_per_cta;          // a multiple of 32
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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

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

// grid: (chunks of keys, batch * n_kv_heads, query tiles of 4); block 128;
// dynamic smem kLogitsWarps * S * stage bytes.
// Warp w of a CTA takes the CTA's 32-key units w, w + 4, w + 8, ...; unit i of
// the warp goes to ring stage i % S.  The block-table entries of the CTA's
// key range are staged first (loaded together with ctx_len; page_tokens is
// a power of two, so page and slot are a shift and a mask); then each warp
// puts its first S units in flight (one cp.async group per unit, empty groups
// keep the count uniform) and only then waits for the query preparation
// kernel (griddepcontrol.wait).  A unit's copy and its reads are by the same
// warp: wait_group + __syncwarp order them, and a __syncwarp after the reads
// precedes the copy that reuses the stage.  The two tiles of a unit are read
// before either is computed, so their MMA chains interleave; a tile whose
// page is bad or that lies past the context computes on stale bytes and
// stores nothing.
// Sign term: k-step kk of a QJL word uses bit planes 2 kk and 2 kk + 1 in
// place (one mask per operand register), weighted 2^(2 kk + 1) after the
// query side's 2 z / z slots; a Horner step (x 4) between k-steps brings
// every k-step of a word to weight 2^(2 n - 1) (n k-steps in the word), and
// words are scaled to the common weight 128.
template <int BITS, int E, int F>
__global__ void __launch_bounds__(kLogitsWarps * 32, E >= 48 ? 4 : BITS == 4 ? 5 : kLogitsMinBlocks) logits_kernel(LogitsParams p) {
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
  __shared__ int64_t page_base[kCtaPages];   // byte offset of this head's block, -1 if bad

  const int gi = blockIdx.y;
  const int b = gi / p.n_kv_heads, h = gi % p.n_kv_heads;
  const int qt = blockIdx.z;
  const int k0 = blockIdx.x * p.keys_per_cta;          // < max_ctx
  const int kend = min(k0 + p.keys_per_cta, p.max_ctx);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int ps = p.page_shift;
  const int P = 1 << ps;
  const int first_page = k0 >> ps;
  const int ctx = min(p.ctx_len[b], p.max_ctx);
  {
    const int n_pg = ((kend - 1) >> ps) - first_page + 1;
    for (int j = threadIdx.x; j < n_pg; j += blockDim.x) {
      const int64_t page = p.cv.block_table[(int64_t)b * p.cv.max_pages + first_page + j];
      page_base[j] = (page >= 0 && page < p.cv.n_pages)
                         ? page * p.cv.page_bytes + (int64_t)h * p.cv.head_block_bytes : -1;
    }
  }
  if (k0 >= ctx) return;
  const int k1 = min(kend, ctx);
  __syncthreads();

  const int n_units = (k1 - k0 + 31) >> 5;
  const int n_my = warp < n_units ? (n_units - warp + kLogitsWarps - 1) / kLogitsWarps : 0;
  const uint8_t* ring = ring_smem + warp * S * STAGE;
  const uint32_t ring_s = smem_addr(ring);
  const int64_t norm_off = (int64_t)P * (16 * W);   // norm slots follow the P records

  // copies unit i of this warp (2 x (16 records + 16 norm slots)) into stage i % S
  auto issue = [&](int i) {
    const uint32_t dst = ring_s + (i & (S - 1)) * STAGE;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int base = k0 + 32 * (warp + kLogitsWarps * i) + 16 * hf;
      if (base >= k1) break;
      const int64_t off = page_base[(base >> ps) - first_page];
      if (off < 0) {
        report(p.cv.err, TQ_DEV_ERR_PAGE);
        continue;
      }
      const int slot = base & (P - 1);
      const uint8_t* hb = p.cv.pages + off;
      const uint8_t* src = hb + (int64_t)slot * (16 * W);
#pragma unroll
      for (int j = 0; j < (16 * W + 31) / 32; ++j) {
        const int c = lane + 32 * j;
        if (c < 16 * W) cp_async16(dst + hf * TILE + 16 * c, src + 16 * c);
      }
      if (lane < NB) cp_async16(dst + 2 * TILE + 64 * hf + 16 * lane, hb + norm_off + slot * NB + 16 * lane);
    }
  };

#pragma unroll
  for (int s = 0; s < S; ++s) {
    if (s < n_my) issue(s);
    cp_async_commit();
  }

  // the query fragments come from the preparation kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int gq = gi * p.qtiles + qt;
  uint2 bq[KC];
  const uint2* fsrc = p.frag + (int64_t)gq * KC * 32 + lane;
#pragma unroll
  for (int kk = 0; kk < KC; ++kk) bq[kk] = fsrc[kk * 32];
  uint2 bz[KQ > 0 ? KQ : 1];
  float zsumf = 0.0f;
  if constexpr (KQ > 0) {
    const uint2* qsrc = p.qfrag + (int64_t)gq * KQ * 32 + lane;
#pragma unroll
    for (int kk = 0; kk < KQ; ++kk) bz[kk] = qsrc[kk * 32];
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
  const float4 sc = p.scal[(int64_t)b * p.n_q_heads + hq];
  const float c0 = sc.x;
  const float c1 = F > 0 ? p.qjl_scale * sc.y : 0.0f;
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
        constexpr int rows_full = 32;
        const int nk = min(4, (F - rows_full * w) / 8);   // k-steps of this word (4, or 2 for a half word)
        int acc[4] = {0, 0, 0, 0};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (k < nk) {
            if (k > 0) {
#pragma unroll
              for (int r = 0; r < 4; ++r) acc[r] *= 4;
            }
            const uint32_t m0 = 0x01010101u << (2 * k), m1 = m0 << 1;
            mma_u8s8(acc, wa[q0 + w] & m0, wb[q0 + w] & m0, wa[q0 + w] & m1, wb[q0 + w] & m1, bz[4 * w + k]);
          }
        }
        const int sh = 6 - 2 * (nk - 1);           // weight 2^(2 nk - 1) -> 128
#pragma unroll
        for (int r = 0; r < 4; ++r) qa[r] += acc[r] << sh;
      }
      // sum_i s_i z_i = sum z - 2 sum beta z
      const float ta = fmaf(-1.0f / 64.0f, (float)(256 * qa[0] + qa[1]), zsumf);
      const float tb = fmaf(-1.0f / 64.0f, (float)(256 * qa[2] + qa[3]), zsumf);
      la = lo_half(na) * fmaf(c1 * hi_half(na), ta, c0 * cba);
      lb = lo_half(nb) * fmaf(c1 * hi_half(nb), tb, c0 * cbb);
    } else {
      la = lo_half(na) * (c0 * cba);
      lb = lo_half(nb) * (c0 * cbb);
    }
  };

  for (int i = 0; i < n_my; ++i) {
    cp_async_wait<S - 1>();
    __syncwarp();
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
      na1 = *reinterpret_cast<const unsigned short*>(nsl + 64 + 2 * g);
      nb1 = *reinterpret_cast<const unsigned short*>(nsl + 64 + 2 * (g + 8));
    }
    const bool ok0 = page_base[(ubase >> ps) - first_page] >= 0;
    const bool ok1 = ubase + 16 < k1 && page_base[((ubase + 16) >> ps) - first_page] >= 0;
    __syncwarp();                    // every read of this stage precedes its reuse
    if (i + S < n_my) issue(i + S);
    cp_async_commit();
    float la0, lb0, la1, lb1;
    tile(wa0, wb0, na0, nb0, la0, lb0);
    tile(wa1, wb1, na1, nb1, la1, lb1);
    if (qvalid) {
      const int r = ubase + g;
      if (ok0 && r < k1) __stcs(orow + r, la0);
      if (ok0 && r + 8 < k1) __stcs(orow + r + 8, lb0);
      if (ok1 && r + 16 < k1) __stcs(orow + r + 16, la1);
      if (ok1 && r + 24 < k1) __stcs(orow + r + 24, lb1);
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
static cudaError_t run_logits(const tqd::LogitsParams& p, dim3 grid, cudaStream_t st) {
  constexpr int q0 = BITS == 1 ? (E + 31) / 32 : BITS == 2 ? E / 16
                   : BITS == 3 ? 3 * (E / 32) + 2 * ((E % 32) / 16) : E / 8;
  constexpr int W = q0 + (F + 31) / 32;
  using RS = tqd::RingShape<W>;
  const int smem = tqd::kLogitsWarps * RS::kStages * RS::kStageBytes;
  static bool attr = false;            // per template instance
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(tqd::logits_kernel<BITS, E, F>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(tqd::kLogitsWarps * 32);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tqd::logits_kernel<BITS, E, F>, p);
}

template <int BITS>
static bool dispatch_logits(const Layout& L, const tqd::LogitsParams& p, dim3 grid, cudaStream_t st,
                            cudaError_t& err) {
  if (L.E == 32 && L.F == 32) return err = run_logits<BITS, 32, 32>(p, grid, st), true;
  if (L.E == 32 && L.F == 0) return err = run_logits<BITS, 32, 0>(p, grid, st), true;
  if (L.E == 16 && L.F == 16) return err = run_logits<BITS, 16, 16>(p, grid, st), true;
  if (L.E == 16 && L.F == 0) return err = run_logits<BITS, 16, 0>(p, grid, st), true;
  if (L.E == 64 && L.F == 64) return err = run_logits<BITS, 64, 64>(p, grid, st), true;
  if (L.E == 64 && L.F == 0) return err = run_logits<BITS, 64, 0>(p, grid, st), true;
  if (L.E == 48 && L.F == 48) return err = run_logits<BITS, 48, 48>(p, grid, st), true;
  if (L.E == 48 && L.F == 0) return err = run_logits<BITS, 48, 0>(p, grid, st), true;
  return false;
}

template <int RPW>
static cudaError_t run_prep(const tqd::PrepParams& pp, int nblk, int64_t units, cudaStream_t st) {
  const int smem = 4 * RPW * pp.d * (int)sizeof(float);   // the block's matrix rows
  static bool attr = false;            // per template instance
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(tqd::prep_queries_kernel<RPW>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 4 * RPW * 256 * 4);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)nblk, (unsigned)units);
  cfg.blockDim = dim3(tqd::kPrepThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = (unsigned)nblk;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tqd::prep_queries_kernel<RPW>, pp);
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
  if (groups * qtiles > 65535) return fail(TQ_EINVAL, "tq_logits: batch * n_kv_heads * query tiles > 65535");
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
  pp.pi32 = cb->pi32;
  pp.s32 = cb->s32;
  pp.frag = frag;
  pp.qfrag = qfrag;
  pp.scal = scal;
  // rows of [Pi q ; S q] per CTA: 32, or 64 when that keeps the cluster at
  // most kMaxClusterCtas CTAs (d_pad and m_pad are multiples of 64)
  const int rows = L.d_pad + L.m_pad;
  const int rb = rows <= 32 * tqd::kMaxClusterCtas ? 32 : 64;
  const int nblk = rows / rb;
  cudaError_t e = rb == 32 ? run_prep<8>(pp, nblk, groups * qtiles, st)
                           : run_prep<16>(pp, nblk, groups * qtiles, st);
  if (e != cudaSuccess) return cuda_fail(e, "tq_logits: query preparation launch");

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
  // Split the context so that the grid fills every CTA slot of the GPU once
  // (148 SMs x kLogitsMinBlocks), each CTA a whole number of 32-key units.
  const int64_t units = groups * qtiles;
  const int64_t slots = 148LL * tqd::kLogitsMinBlocks;
  const int64_t chunks = (slots + units - 1) / units;
  int64_t kpc = (max_ctx + chunks - 1) / chunks;
  kpc = ((kpc + 31) / 32) * 32;
  if (kpc < 32 * tqd::kLogitsWarps) kpc = 32 * tqd::kLogitsWarps;
  // a CTA stages at most kCtaPages block-table entries (its range may start
  // inside a page, hence the 2 spare entries)
  const int64_t kpc_cap = ((int64_t)(tqd::kCtaPages - 2) * cv.page_tokens / 32) * 32;
  if (kpc > kpc_cap) kpc = kpc_cap;
  const int64_t n_chunks = (max_ctx + kpc - 1) / kpc;
  if (n_chunks > 0x7fffffffLL) return fail(TQ_EINVAL, "tq_logits: context too long");
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
  dim3 grid((unsigned)n_chunks, (unsigned)groups, (unsigned)qtiles);
  bool ok = false;
  cudaError_t le = cudaSuccess;
  switch (L.bits) {
    case 1: ok = dispatch_logits<1>(L, lp, grid, st, le); break;
    case 2: ok = dispatch_logits<2>(L, lp, grid, st, le); break;
    case 3: ok = dispatch_logits<3>(L, lp, grid, st, le); break;
    case 4: ok = dispatch_logits<4>(L, lp, grid, st, le); break;
  }
  if (!ok) return fail(TQ_EUNSUPPORTED, "tq_logits: no kernel for this (d, m)");
  if (le != cudaSuccess) return cuda_fail(le, "tq_logits launch");
  return cuda_fail(cudaGetLastError(), "tq_logits launch");
}

}  // namespace tq
