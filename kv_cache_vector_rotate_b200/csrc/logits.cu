// Fused attention logits straight from the packed keys.
//
// "TurboQuant explained" (a2a-mcp.org), §Stage 2 and §How it works: the
// query is rotated once (Pi q) and sketched once (S q); every logit is then
//   L = ||k|| ( sum_j (Pi q)_j c[idx_j] + sqrt(pi/2)/m ||r|| sum_i (S q)_i s_i )
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
//  * logits_kernel, which pulls the cache into L2 while the queries are
//    prepared and then streams it through shared memory.
//
// The key side: every CTA owns a contiguous share of 32-key units; its
// warps run them through the tensor cores with the key operand built in
// registers:
//  - codebook term, b <= 3: m16n8k32 int8 MMAs.  The reconstruction levels
//    are k 2^-f with k an 8-bit integer, so a key element is one signed
//    byte; eight stored codes form one byte-permute selector after a single
//    mask, and one permute of the 8-byte level table gives four elements.
//    (Pi q) is quantized to 16-bit integers as two int8 slices; the products
//    are accumulated exactly in int32 and combined at the end.
//  - codebook term, b = 4: m16n8k16 fp16 MMAs on sign-magnitude codes (16
//    levels do not fit one 8-byte permute table), the query as fp16 hi + lo.
//  - sign term: m16n8k32 int8 MMAs.  The stored sign bits enter in place as
//    0 / 2^p bytes (one mask per operand register); S q is quantized to
//    integers z, and sum_i s_i z_i = sum_i z_i - 2 sum_i beta_i z_i.
// The MMA's N = 8 columns are the high and low slices of 4 queries.
// HBM traffic is the packed records plus the logits.

#include "key_tile.cuh"

namespace tqd {

constexpr int kSliceMax = 32639;   // |z| bound of Pi q: the high int8 slice stays in [-128, 127]
constexpr int kSliceMaxQ = 16319;  // |z| bound of S q: 2 z still splits into int8 slices
constexpr int kPrepThreads = 128;  // threads of a preparation CTA
constexpr int kPartRows = 32;      // rows of [Pi q ; S q] per preparation part



struct PrepParams {
  const void* q;             // [batch][n_q_heads][d]
  tq_dtype dtype;
  int d;
  int n_q_heads, n_kv_heads, G, qtiles;
  float cb_unscale;          // 2^-f
  float qjl_scale;           // sqrt(pi/2) / m
  float s_rowmax;            // >= max_i ||S_i||
  const uint4* qprep;        // [Pi ; S] bf16 hi + lo A fragments (tq_codebook::qprep_frag)
  uint2* frag;
  uint2* qfrag;
  float2* scal;
};


// ---- query preparation -----------------------------------------------------------
//
// Fragment bytes: codebook fragments uint2 [KC][32] per query tile (KC = E/8
// int8 k-steps, or E/4 fp16 k-steps for b = 4), QJL fragments uint2
// [F/8][32], per-query scales float2 {c0, c1}.  Lane (2 q + s) * 4 + t of a
// fragment holds slice s (0 high, 1 low) of query slot q for chunk t; byte
// e % 8 (half e % 4 for fp16) of it is row e of the k-step.  In the QJL part
// rows 8 kk .. 8 kk + 3 of a k-step hold the slices of 2 z, rows 8 kk + 4 ..
// 8 kk + 7 those of z (|z| <= kSliceMaxQ), matching the key operand of the
// tile (sign bytes 2^(2 kk) beta and 2^(2 kk + 1) beta).

// What the quantization of a prepared row needs of the codebook.
struct PrepConsts {
  float cb_unscale;          // 2^-f
  float qjl_scale;           // sqrt(pi/2) / m
  float s_rowmax;            // >= max_i ||S_i||
};

// Quantizes v = row `row` of [Pi q ; S q] for query slot `qs` (norm qn) into
// its fragment bytes: codebook fragments `fr` ([KC][32] uint2 of this query
// tile; int8 slices for b <= 3, fp16 hi / lo for b = 4), sign-term
// fragments `fz` ([F/8][32]).  Global or shared memory.
template <int E, int F, bool INT8>
__device__ __forceinline__ void put_prepared(float v, int row, int qs, float qn, const PrepConsts& pc, uint2* fr,
                                             uint2* fz) {
  const bool sk = row >= 4 * E;                 // an S q row
  const int l = sk ? row - 4 * E : row;         // row within its half
  int tc, e;                                    // chunk, row within the chunk
  if (sk) {
    tc = l / (F > 0 ? F : 1);
    e = l - tc * F;
  } else {
    tc = l / E;
    e = l - tc * E;
  }
  if (!sk && !INT8) {
    int e2 = 0;                                 // ||q|| in [2^(e2-1), 2^e2)
    if (qn > 0.0f) frexpf(qn, &e2);
    const float vs = v * ldexpf(1.0f, 14 - e2);
    const __half hi = __float2half_rn(vs);
    const __half lo = __float2half_rn(vs - __half2float(hi));
    __half* h = reinterpret_cast<__half*>(fr + (e / 4) * 32);
    h[((2 * qs) * 4 + tc) * 4 + (e & 3)] = hi;
    h[((2 * qs + 1) * 4 + tc) * 4 + (e & 3)] = lo;
    return;
  }
  const int zmax = sk ? kSliceMaxQ : kSliceMax;
  const float bound = sk ? pc.s_rowmax * qn : qn;
  const float scale = bound > 0.0f ? (float)zmax * __frcp_rn(bound) : 0.0f;
  int z = max(-zmax, min(zmax, __float2int_rn(v * scale)));
  if (sk && (e & 7) < 4) z *= 2;                // rows 8 kk .. 8 kk + 3 of a QJL k-step: 2 z
  const int zh = (z + 128) >> 8;                // floor((z + 128) / 256)
  const int zl = z - 256 * zh;                  // in [-128, 127]
  int8_t* b8 = reinterpret_cast<int8_t*>((sk ? fz : fr) + (e / 8) * 32);
  b8[((2 * qs) * 4 + tc) * 8 + (e & 7)] = (int8_t)zh;
  b8[((2 * qs + 1) * 4 + tc) * 8 + (e & 7)] = (int8_t)zl;
}

// Per-query scales {c0, c1} of a query with norm qn: c0 undoes the codebook
// fragments' scale (and 2^f of the int8 tables), c1 = sqrt(pi/2)/m times the
// sketch fragments' scale.
template <bool INT8>
__device__ __forceinline__ float2 prep_scales(float qn, const PrepConsts& pc) {
  int e = 0;
  if (!INT8 && qn > 0.0f) frexpf(qn, &e);
  const float c0 = INT8 ? qn * (1.0f / (float)kSliceMax) * pc.cb_unscale : ldexpf(1.0f, e - 14);
  const float c1 = pc.qjl_scale * (pc.s_rowmax * qn) * (1.0f / (float)kSliceMaxQ);
  return make_float2(c0, c1);
}

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
template <int E, int F, bool INT8>
__device__ __forceinline__ void prep_part(const PrepParams& p, int gq, int r, PrepSmem& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int gi = gq / p.qtiles, qt = gq % p.qtiles;
  const int b = gi / p.n_kv_heads, kv = gi % p.n_kv_heads;
  const int64_t qbase = (int64_t)b * p.n_q_heads + kv * p.G + qt * 4;   // first query row of the tile
  const int nq = min(4, p.G - qt * 4);
  const int d = p.d, d16 = (d + 15) >> 4;
  PrepConsts pc;
  pc.cb_unscale = p.cb_unscale;
  pc.qjl_scale = p.qjl_scale;
  pc.s_rowmax = p.s_rowmax;

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
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (lane + 32 * i < d) x[i] = load_elem(p.q, qoff + lane + 32 * i, p.dtype);
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
  if (warp < 2) {
    const float4 o = sm.ksum[mt][lane];
    const float va = acc[0] + acc[1] + o.x + o.y, vb = acc[2] + acc[3] + o.z + o.w;
    constexpr int kcs = INT8 ? E / 8 : E / 4;
    uint2* fr = p.frag + (int64_t)gq * kcs * 32;
    uint2* fz = p.qfrag + (int64_t)gq * (F / 8) * 32;
    put_prepared<E, F, INT8>(va, r * kPartRows + 16 * mt + g, t, qn, pc, fr, fz);
    put_prepared<E, F, INT8>(vb, r * kPartRows + 16 * mt + g + 8, t, qn, pc, fr, fz);
  }
  if (r == 0 && (int)threadIdx.x < nq) p.scal[qbase + threadIdx.x] = prep_scales<INT8>(sqrtf(sm.qn2[threadIdx.x]), pc);
  __syncthreads();                  // the shared buffers may be reused
}

// Two-launch form: grid (parts, groups * qtiles), block 128; the logits
// kernel follows by programmatic dependent launch.
template <int E, int F, bool INT8>
__global__ void __launch_bounds__(kPrepThreads) prep_queries_kernel(PrepParams p) {
  __shared__ PrepSmem sm;
  // launched as a programmatic dependent of the previous kernel on the
  // stream: the queries (and the workspace, which the previous logits call
  // may still read) are touched only after that kernel has completed, and
  // the logits kernel is released only then
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  prep_part<E, F, INT8>(p, blockIdx.y, blockIdx.x, sm);
}

// ---- logits ------------------------------------------------------------------------
//
// grid: n_cta CTAs, at least one per line, usually one per SM; a CTA is NC
// consumer warps (15; 8 for d > 128; 4 when every CTA gets few units) and
// one producer warp (at most 16 warps: a fifth warp on one of the SM's four
// schedulers would not get its registers).  The 64-key units of all lines
// (sequence, KV head, query tile; U units each) are numbered line by line;
// CTA c owns a contiguous share of them (at most U, so at most two lines)
// and consumer warp w takes the share's units w, w + NC, ...  Warp w has a
// ring of S copy slots, each holding one unit (64 records, then their 64
// norm slots) with a "full" mbarrier (completed by the unit's bulk copies)
// and an "empty" one (completed when warp w has read the slot).  The
// producer's lanes put the units in flight in consumption order, in waves
// of up to 32 units, refilling a slot once it is empty.  A bulk copy stalls the issuing thread while the memory system
// is saturated, and one thread issues only a few per microsecond, so the
// copies are spread over the producer's 32 lanes, kept few (one per unit
// when a 64-token page's head block is the unit: its records and norms are
// contiguous), and never issued by a consumer warp.
//
// Two ways to get the query fragments:
//  * PREP (d <= 128, one launch per call): the CTA prepares its own queries.
//    Before its programmatic-dependent-launch wait it only loads the
//    codebook's [Pi ; S] fragments (constants) into registers -- consumer
//    warp w holds 16-row tile w; a 16th tile goes to shared memory, for
//    consumer 0.  After the wait it loads its lines' context lengths,
//    block-table entries and queries; then the producer starts the stream
//    while the consumers compute tile w of [Pi q ; S q] for the CTA's 8 query
//    slots (4 per line) on the tensor cores and quantize it into fragment
//    bytes in shared memory.
//  * otherwise (two launches per call): prep_queries_kernel writes the
//    fragments to the workspace.  It is a programmatic dependent of the
//    previous kernel on the stream but releases this kernel only after its
//    own wait, so every earlier kernel has finished when this kernel starts
//    and it may read the cache before its wait: the producer puts one unit
//    per consumer warp in flight, the consumers wait and fetch their lines'
//    fragments, and the producer goes on once they have them (fragment
//    loads issued behind a full stream of copies would wait for it).  On a
//    short context this form is the faster one: in-CTA preparation loads
//    the whole [Pi ; S] table into every CTA.
// Every mbarrier wait is bounded; a CTA where one gives up reports
// TQ_DEV_ERR_TIMEOUT and lets every copy it issued land before it exits.

constexpr int kLogitsPages = 512;    // block-table entries staged per CTA
constexpr int kLogitsMaxSlots = 64;

__host__ __device__ constexpr int logits_max_consumers(int E) { return E >= 48 ? 8 : 15; }
// registers per thread: the two-launch form with d <= 128 stays at 112 so
// that a preparation CTA (128 threads x 64 registers) fits beside its 16
// warps
__host__ __device__ constexpr int logits_regs(int E, bool prep) { return prep || E >= 48 ? 128 : 112; }


struct LogitsParams {
  tq::CacheView cv;
  int page_shift;            // log2(page_tokens)
  const int32_t* ctx_len;
  int n_kv_heads, n_q_heads, G, qtiles;
  int units;                 // U: 64-key units per line
  int max_ctx;               // ctx_len values are clamped to [0, max_ctx]
  int per_cta, extra;        // CTA c owns per_cta units, + 1 when c < extra (lines * U < 2^31)
  FastDiv div_u, div_qtiles, div_kv;   // / U, / qtiles, / n_kv_heads
  int nc;                    // consumer warps
  FastDiv div_nc;
  int ring_shift;            // S = 1 << ring_shift copy slots per consumer warp
  int fixed_off;
  int n_cta;
  // PREP: queries and the preparation table
  const void* q;
  tq_dtype dtype;
  int d, d16;
  const uint4* table;        // [Pi ; S] bf16 hi + lo A fragments (tq_codebook::qprep_frag)
  int prep_tiles;            // 16-row tiles of [Pi ; S]
  PrepConsts pc;
  // two launches: the preparation kernel's output
  const uint2* frag;
  const uint2* qfrag;
  const float2* scal;
  float* out;
  int64_t out_stride;
  KeyTables kt;
};

// The fixed part of a CTA's shared memory (after the slots).
template <int KC, int KQ>
struct LogitsFixed {
  uint64_t full_bar[kLogitsMaxSlots];
  uint64_t empty_bar[kLogitsMaxSlots];
  int64_t page_base[kLogitsPages];         // byte offset of the head block, -1 if the page is bad
  uint2 fr[2][KC * 32];                    // codebook fragments of the two lines
  uint2 fz[2][(KQ > 0 ? KQ : 1) * 32];     // sign-term fragments
  float2 scal[8];                          // {c0, c1} of query slot 4 line + q
  float qn2[8];                            // PREP: ||q||^2 of the 8 query slots
  uint64_t xtab_bar;                       // PREP: the extra table tile has landed
  int flags;                               // bit 0: a wait gave up
  int slot_last[kLogitsMaxSlots];          // last unit issued into each slot
  uint16_t qs[2][8][128 + 8];              // PREP: bf16 hi / lo of the 8 query slots
  uint4 xtab[8 * 2 * 32];                  // PREP: A fragments of table tile NC (a 16th tile)
};

template <int BITS, int E, int F>
size_t logits_fixed_bytes() {
  using TS = TileShape<BITS, E, F>;
  return sizeof(LogitsFixed<TS::KC, TS::KQ>);
}


template <int BITS, int E, int F, bool PREP>
__global__ void __maxnreg__(logits_regs(E, PREP)) logits_kernel(LogitsParams p) {
  using TS = TileShape<BITS, E, F>;
  constexpr int KC = TS::KC, KQ = TS::KQ, W = TS::W, NB = TS::NB;
  using SS = SlotShape<W, NB>;
  constexpr int REC = SS::kRecBytes, NOFF = SS::kNormOff, STAGE = SS::kBytes;
  static_assert(!PREP || 4 * E <= 128, "the CTAs prepare at most 128 coordinates");
  extern __shared__ __align__(128) uint8_t smem[];
  auto& fx = *reinterpret_cast<LogitsFixed<KC, KQ>*>(smem + p.fixed_off);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NT = blockDim.x;
  const int NC = p.nc;                       // consumer warps; warp NC is the producer
  const bool producer = warp == NC;
  const int g = lane >> 2, t = lane & 3;
  const int c = blockIdx.x;
  const int i0 = c * p.per_cta + min(c, p.extra);
  const int n_units = p.per_cta + (c < p.extra ? 1 : 0);
  const int U = p.units;
  const int line0 = (int)fdiv((uint32_t)i0, p.div_u);
  const int n_lines = n_units > 0 ? (int)fdiv((uint32_t)(i0 + n_units - 1), p.div_u) - line0 + 1 : 0;   // 0, 1 or 2
  const int ua0 = i0 - line0 * U;                                          // first unit within line 0
  const int split = n_lines > 1 ? (line0 + 1) * U - i0 : n_units;          // units of line 0
  const int ps = p.page_shift, P = 1 << ps;
  const int S = 1 << p.ring_shift;

  if (tid < NC * S) {
    mbar_init(&fx.full_bar[tid], 1);
    mbar_init(&fx.empty_bar[tid], 1);
    fx.slot_last[tid] = -1;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (tid == 0) fx.flags = 0;
  // PREP: the preparation table is a constant of the codebook, loaded
  // before the wait (consumer warp w: A fragments of 16-row tile w of [Pi ; S])
  uint4 af[PREP ? 8 : 1][2];
  if constexpr (PREP) {
    if (producer && lane == 0 && p.prep_tiles > NC) {
      // tile NC of the table into shared memory for consumer 0
      mbar_init(&fx.xtab_bar, 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      const uint32_t bytes = (uint32_t)p.d16 * 64 * 16;
      mbar_arrive_tx(&fx.xtab_bar, bytes);
      bulk_copy_plain(smem_addr(fx.xtab), p.table + (size_t)NC * p.d16 * 64, bytes, &fx.xtab_bar);
    }
    if (warp < p.prep_tiles && warp < NC) {
      // volatile loads: issued here, ahead of the wait, not where they are used
      const uint4* tab = p.table + (size_t)warp * p.d16 * 64 + lane;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < p.d16) {
          af[j][0] = ldg_early(tab + (2 * j) * 32);
          af[j][1] = ldg_early(tab + (2 * j + 1) * 32);
        }
    }
    // everything below reads the caller's data, which the previous kernel on
    // the stream may have written
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
  }

  auto make_line = [&](int s) {
    LineView L;
    const int ln = line0 + s;
    const int gi = (int)fdiv((uint32_t)ln, p.div_qtiles);
    L.qt = ln - gi * p.qtiles;
    L.b = (int)fdiv((uint32_t)gi, p.div_kv);
    L.h = gi - L.b * p.n_kv_heads;
    const int ua = s == 0 ? ua0 : 0;
    const int ub = s == 0 ? ua0 + split : n_units - split;
    L.klo = 64 * ua;
    L.khi = min(64 * ub, p.max_ctx);
    L.first = L.klo >> ps;
    L.npg = s < n_lines && L.klo < L.khi ? ((L.khi - 1) >> ps) - L.first + 1 : 0;   // L0.npg + L1.npg <= kLogitsPages
    L.k1 = 0;
    L.ebase = 0;
    return L;
  };
  LineView L0 = make_line(0), L1 = make_line(1);
  L1.ebase = L0.npg;
  const int ctx0 = L0.npg > 0 ? p.ctx_len[L0.b] : 0;   // independent of the block-table loads
  const int ctx1 = L1.npg > 0 ? p.ctx_len[L1.b] : 0;
  int64_t pgv[4] = {0, 0, 0, 0};                      // kLogitsPages <= 4 * NT for NT >= 128
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int j = tid + k * NT;
    if (j < L0.npg + L1.npg) {
      const LineView& L = j < L0.npg ? L0 : L1;
      pgv[k] = p.cv.block_table[(int64_t)L.b * p.cv.max_pages + L.first + j - L.ebase];
    }
  }
  // PREP, warps 0-7: query slot n = warp (line n / 4, query n % 4 of its
  // tile) as bf16 hi + lo, and ||q||^2
  if constexpr (PREP) {
    if (warp < 8) {
      const LineView& L = warp < 4 ? L0 : L1;
      const int qi = L.qt * 4 + (warp & 3);
      const bool valid = (warp >> 2) < n_lines && qi < p.G;
      float x[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      if (valid) {
        const int64_t qoff = ((int64_t)L.b * p.n_q_heads + (int64_t)L.h * p.G + qi) * p.d;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (lane + 32 * i < p.d) x[i] = load_elem(p.q, qoff + lane + 32 * i, p.dtype);
      }
      float s2 = 0.0f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int k = lane + 32 * i;
        if (k < 16 * p.d16) {
          const uint16_t hb = bf16_bits(x[i]);
          fx.qs[0][warp][k] = hb;
          fx.qs[1][warp][k] = bf16_bits(x[i] - __bfloat162float(__ushort_as_bfloat16(hb)));
        }
        s2 = fmaf(x[i], x[i], s2);
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
      if (lane == 0) fx.qn2[warp] = s2;
    }
  }
  L0.k1 = min(L0.khi, max(0, min(ctx0, p.max_ctx)));
  L1.k1 = min(L1.khi, max(0, min(ctx1, p.max_ctx)));
  bool bad = false;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int j = tid + k * NT;
    if (j < L0.npg + L1.npg) {
      const LineView& L = j < L0.npg ? L0 : L1;
      const int pidx = L.first + j - L.ebase;
      const bool valid = pgv[k] >= 0 && pgv[k] < p.cv.n_pages;
      fx.page_base[j] = valid ? pgv[k] * p.cv.page_bytes + (int64_t)L.h * p.cv.head_block_bytes : -1;
      // pages past the context are not read: an invalid entry there is no error
      if (!valid && L.k1 > L.klo && pidx <= ((L.k1 - 1) >> ps)) {
        bad = true;
        report(p.cv.err, TQ_DEV_ERR_PAGE);
      }
    }
  }
  // fast path: every used page valid
  const bool fast = !__syncthreads_or(bad);   // also publishes the barriers' init

  if (producer) {
    // ---------------------------------------------------------- producer
    const int64_t norm_off = (int64_t)P * (16 * W);   // norm slots follow the P records
    const uint64_t pol = evict_first_policy();        // the cache is streamed once per call
    // the copies of unit i (consumer warp i % NC, its unit i / NC); false
    // when the wait for the slot gave up
    auto issue = [&](int i) -> bool {
      const int j = (int)fdiv((uint32_t)i, p.div_nc), w = i - j * NC;
      const int slot = w * S + (j & (S - 1));
      if (j >= S && !mbar_wait_sleep(&fx.empty_bar[slot], (uint32_t)((j >> p.ring_shift) - 1) & 1u)) return false;
      fx.slot_last[slot] = i;
      uint64_t* bar = &fx.full_bar[slot];
      const uint32_t dst = smem_addr(smem) + slot * STAGE;
      const bool in1 = i >= split;
      const int pos = 64 * (in1 ? i - split : ua0 + i);
      const LineView& L = in1 ? L1 : L0;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the consumer's reads of the slot first
      const int eb = L.ebase - L.first;
      if (fast && P == 64 && pos < L.k1) {
        // the unit is one page's head block: records and norms in one copy
        // (records past the context are read and not used)
        mbar_arrive_tx(bar, 64 * (16 * W + NB));
        bulk_copy(dst, p.cv.pages + fx.page_base[eb + (pos >> ps)], 64 * (16 * W + NB), bar, pol);
        return true;
      }
      // pieces of min(P, 64) keys (16 on a cache with a bad page) from
      // their pages: records, then norms
      const int piece = fast ? min(P, 64) : 16;
      uint32_t bytes = 0;
      for (int k = pos; k < pos + 64; k += piece)
        if (k < L.k1 && fx.page_base[eb + (k >> ps)] >= 0) bytes += piece * (16 * W + NB);
      mbar_arrive_tx(bar, bytes);          // 0 bytes: the phase completes on the arrival alone
      for (int k = pos; k < pos + 64; k += piece) {
        if (k >= L.k1) break;
        const int64_t off = fx.page_base[eb + (k >> ps)];
        if (off < 0) continue;
        const int sl = k & (P - 1);
        const uint8_t* hb = p.cv.pages + off;
        bulk_copy(dst + (k - pos) * (16 * W), hb + (int64_t)sl * (16 * W), piece * (16 * W), bar, pol);
        bulk_copy(dst + NOFF + (k - pos) * NB, hb + norm_off + sl * NB, piece * NB, bar, pol);
      }
      return true;
    };
    // Units go out in waves of `wave` consecutive units, lane k of a wave
    // taking unit base + k; a wave holds no two units of one slot and the
    // waves are ordered, so the uses of a slot are issued in order and a
    // lane that waits for a slot's release is at most one phase ahead of it
    // (a parity wait further ahead would return at once).
    const int wave = min(32, NC * S);
    bool ok = true;
    int base = 0;
    if constexpr (!PREP) {
      // one unit per consumer warp before the fragments are fetched
      if (lane < min(n_units, NC)) ok = issue(lane);
      base = min(n_units, NC);
      asm volatile("barrier.sync 1, %0;" ::"r"(NT) : "memory");   // the consumers have the fragments
    }
    for (; base < n_units; base += wave) {
      if (lane < wave && base + lane < n_units && ok) ok = issue(base + lane);
      if (!__all_sync(0xffffffffu, ok)) break;
    }
    if (!__all_sync(0xffffffffu, ok) && lane == 0) {
      atomicOr(&fx.flags, 1);
      report(p.cv.err, TQ_DEV_ERR_TIMEOUT);
    }
  } else {
    // ---------------------------------------------------------- consumers
    if constexpr (PREP) {
      // tile w of [Pi q ; S q] for the 8 query slots, from the table
      // fragments, while the first units arrive; consumer 0 also does tile NC
      // (from the table tile in shared memory) when there are NC + 1 tiles
      auto prep_tile = [&](int tile, bool from_smem) {
        const bool two = p.dtype != TQ_BF16;          // bf16 queries are exact in one bf16 term
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j < p.d16) {
            const uint4 a0 = from_smem ? fx.xtab[(2 * j) * 32 + lane] : af[j][0];
            const uint4 a1 = from_smem ? fx.xtab[(2 * j + 1) * 32 + lane] : af[j][1];
            const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&fx.qs[0][g][16 * j + 2 * t]);
            const uint32_t b1 = *reinterpret_cast<const uint32_t*>(&fx.qs[0][g][16 * j + 2 * t + 8]);
            mma_bf16(acc, a0, b0, b1);
            mma_bf16(acc, a1, b0, b1);
            if (two) {
              const uint32_t c0 = *reinterpret_cast<const uint32_t*>(&fx.qs[1][g][16 * j + 2 * t]);
              const uint32_t c1 = *reinterpret_cast<const uint32_t*>(&fx.qs[1][g][16 * j + 2 * t + 8]);
              mma_bf16(acc, a0, c0, c1);
              mma_bf16(acc, a1, c0, c1);
            }
          }
        }
        // acc: rows g (0, 1) and g + 8 (2, 3) of the tile, query slots 2t (0, 2) and 2t + 1 (1, 3)
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int n = 2 * t + (x & 1);
          const int row = 16 * tile + g + 8 * (x >> 1);
          put_prepared<E, F, TS::kInt8>(acc[x], row, n & 3, sqrtf(fx.qn2[n]), p.pc, fx.fr[n >> 2], fx.fz[n >> 2]);
        }
      };
      if (warp < p.prep_tiles) prep_tile(warp, false);
      if (warp == 0 && p.prep_tiles > NC) {
        if (mbar_wait_sleep(&fx.xtab_bar, 0u)) {
          prep_tile(NC, true);
        } else if (lane == 0) {
          atomicOr(&fx.flags, 1);
          report(p.cv.err, TQ_DEV_ERR_TIMEOUT);
        }
      }
      if (tid < 8) fx.scal[tid] = prep_scales<TS::kInt8>(sqrtf(fx.qn2[tid]), p.pc);
      asm volatile("barrier.sync 2, %0;" ::"r"(NC * 32) : "memory");   // fragments ready (consumers only)
    } else {
      // the query fragments and scales come from the preparation kernel;
      // the next call's preparation kernel may be scheduled from here on (it
      // waits for this grid to complete before it touches anything)
      asm volatile("griddepcontrol.wait;" ::: "memory");
      asm volatile("griddepcontrol.launch_dependents;");
      constexpr int FL = (KC + KQ) * 32;         // fragment words (uint2) per line
      for (int j = tid; j < n_lines * FL; j += NC * 32) {
        const int s = j / FL, r = j % FL;
        const int64_t gq = line0 + s;
        if (r < KC * 32) fx.fr[s][r] = ld_cg(p.frag + gq * (KC * 32) + r);
        else if constexpr (KQ > 0) fx.fz[s][r - KC * 32] = ld_cg(p.qfrag + gq * (KQ * 32) + (r - KC * 32));
      }
      if (tid < 4 * n_lines) {
        const LineView& L = tid < 4 ? L0 : L1;
        const int qi = L.qt * 4 + (tid & 3);
        fx.scal[tid] = qi < p.G ? ld_cg(p.scal + (int64_t)L.b * p.n_q_heads + (int64_t)L.h * p.G + qi)
                                : make_float2(0.0f, 0.0f);
      }
      asm volatile("barrier.sync 1, %0;" ::"r"(NT) : "memory");   // with the producer
    }

    const int n_my = warp < n_units ? (int)fdiv((uint32_t)(n_units - warp - 1), p.div_nc) + 1 : 0;   // units of this warp
    uint64_t* fbars = fx.full_bar + warp * S;
    uint64_t* ebars = fx.empty_bar + warp * S;
    const uint8_t* ring = smem + warp * S * STAGE;
    int cur = -1;
    QueryFrags<KC, KQ> qf;
    bool qvalid = false;
    float* orow = p.out;
    int k1 = 0, eb = 0;
    for (int j = 0; j < n_my; ++j) {
      if (!mbar_wait_sleep(&fbars[j & (S - 1)], (uint32_t)(j >> p.ring_shift) & 1u)) {
        if (lane == 0) {
          atomicOr(&fx.flags, 1);
          report(p.cv.err, TQ_DEV_ERR_TIMEOUT);
        }
        break;
      }
      const int i = warp + j * NC;
      const bool in1 = i >= split;
      const int pos0 = 64 * (in1 ? i - split : ua0 + i);
      const int s = in1 ? 1 : 0;
      if (s != cur) {
        cur = s;
        const LineView& L = in1 ? L1 : L0;
#pragma unroll
        for (int kk = 0; kk < KC; ++kk) qf.bq[kk] = fx.fr[s][kk * 32 + lane];
#pragma unroll
        for (int kk = 0; kk < KQ; ++kk) qf.bz[kk] = fx.fz[s][kk * 32 + lane];
        qf.zsum = query_zsum<KQ>(qf.bz);
        const float2 sc = fx.scal[4 * s + t];
        qf.c0 = sc.x;
        qf.c1 = F > 0 ? sc.y : 0.0f;
        const int qidx = L.qt * 4 + t;
        qvalid = qidx < p.G;
        orow = p.out + ((int64_t)L.b * p.n_q_heads + (int64_t)L.h * p.G + (qvalid ? qidx : 0)) * p.out_stride;
        k1 = L.k1;
        eb = L.ebase - L.first;
      }
      const uint8_t* stg = ring + (j & (S - 1)) * STAGE;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {          // two 32-key halves of the unit
        const int pos = pos0 + 32 * hf;
        const uint8_t* st = stg + hf * 32 * REC;
        uint32_t wa0[W], wb0[W], wa1[W], wb1[W];
        lds_chunk<W>(st + g * REC + t * (4 * W), wa0);
        lds_chunk<W>(st + (g + 8) * REC + t * (4 * W), wb0);
        lds_chunk<W>(st + (16 + g) * REC + t * (4 * W), wa1);
        lds_chunk<W>(st + (24 + g) * REC + t * (4 * W), wb1);
        uint32_t na0, nb0, na1, nb1;
        unit_norms<NB>(stg + NOFF + hf * 32 * NB, g, na0, nb0, na1, nb1);
        if (hf == 1) {
          __syncwarp();                  // every read of this slot precedes its release
          if (lane == 0) mbar_arrive(&ebars[j & (S - 1)]);
        }
        if (pos >= k1) continue;         // past the context: nothing to store
        bool ok0 = true, ok1 = pos + 16 < k1;
        if (!fast) {
          ok0 = fx.page_base[eb + (pos >> ps)] >= 0;
          ok1 = ok1 && fx.page_base[eb + ((pos + 16) >> ps)] >= 0;
        }
        float la0, lb0, la1, lb1;
        tile_logits<BITS, E, F>(wa0, wb0, na0, nb0, qf, p.kt, la0, lb0);
        tile_logits<BITS, E, F>(wa1, wb1, na1, nb1, qf, p.kt, la1, lb1);
        if (qvalid) {
          const int r = pos + g;
          if (fast && pos + 32 <= k1) {
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
    }
  }
  // every thread of the CTA meets here; after a wait that gave up, the
  // copies already issued land (each wait bounded) before shared memory is
  // released
  __syncthreads();
  if (fx.flags & 1) {
    for (int k = tid; k < NC * S; k += NT)
      if (fx.slot_last[k] >= 0)
        mbar_wait(&fx.full_bar[k], (uint32_t)((int)fdiv((uint32_t)fx.slot_last[k], p.div_nc) >> p.ring_shift) & 1u);
    if (PREP && tid == 0 && p.prep_tiles > NC) mbar_wait(&fx.xtab_bar, 0u);
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

// One launch when every CTA gets at least this many units.
constexpr int64_t kPrepMinUnits = 64;

size_t logits_workspace(const tq_codebook* cb, int64_t groups, int G) {
  return logits_ws_layout(cb, groups, G, groups * G).total;
}

// Shared-memory plan of a logits launch: NW warps x S copy slots (S a power
// of two, 2 or 4: S = 4 when a warp has more than 2 units and the slots
// fit), then the fixed part; the two-launch form leaves room for a
// preparation CTA on the same SM.
struct LogitsPlan {
  int nw, ring_shift, fixed_off, smem, smem_max;
};

template <int BITS, int E, int F>
static bool logits_plan(int64_t units_per_cta, bool prep, LogitsPlan* pl) {
  using TS = tqd::TileShape<BITS, E, F>;
  const int stage = tqd::SlotShape<TS::W, TS::NB>::kBytes;
  static int optin[64] = {};
  const int dev = current_device();
  int smax = dev >= 0 && dev < 64 ? optin[dev] : 0;
  if (smax == 0) {
    if (cudaDeviceGetAttribute(&smax, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
    if (dev >= 0 && dev < 64) optin[dev] = smax;
  }
  const int budget = prep ? smax : smax - 8 * 1024;
  const int fixed = (int)((tqd::logits_fixed_bytes<BITS, E, F>() + 15) / 16 * 16);
  pl->nw = prep ? 15 : units_per_cta >= 16 ? tqd::logits_max_consumers(E) : 4;
  const int64_t per_warp = (units_per_cta + pl->nw - 1) / pl->nw;
  int S = per_warp > 2 ? 4 : 2;
  while (S > 2 && fixed + pl->nw * S * stage > budget) S /= 2;
  if (fixed + pl->nw * S * stage > budget) return false;
  pl->ring_shift = S == 4 ? 2 : 1;
  pl->fixed_off = pl->nw * S * stage;
  pl->smem = pl->fixed_off + fixed;
  // the kernel attribute (set once per instance) covers the largest plan
  const int nw_max = prep ? 15 : tqd::logits_max_consumers(E);
  pl->smem_max = std::max(pl->smem, fixed + nw_max * 4 * stage <= budget ? fixed + nw_max * 4 * stage
                                                                         : fixed + nw_max * 2 * stage);
  return true;
}

template <int BITS, int E, int F, bool PREP>
static tq_status launch_logits_kernel(tqd::LogitsParams p, const LogitsPlan& pl, cudaStream_t st) {
  static PerDeviceOnce attr;           // per template instance
  if (const int dev_ = current_device(); attr.need(dev_)) {
    cudaError_t e = cudaFuncSetAttribute(tqd::logits_kernel<BITS, E, F, PREP>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem_max);
    if (e != cudaSuccess) return cuda_fail(e, "tq_logits: smem attribute");
    attr.mark(dev_);
  }
  p.ring_shift = pl.ring_shift;
  p.nc = pl.nw;
  p.div_nc = tqd::make_fastdiv((uint32_t)pl.nw);
  p.fixed_off = pl.fixed_off;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.n_cta);
  cfg.blockDim = dim3((pl.nw + 1) * 32);   // consumers + the producer warp
  cfg.dynamicSmemBytes = (size_t)pl.smem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, tqd::logits_kernel<BITS, E, F, PREP>, p);
  if (e != cudaSuccess) return cuda_fail(e, "tq_logits launch");
  return TQ_OK;
}

// The preparation kernel for (E, F), a programmatic dependent of the
// previous kernel on the stream.
template <int E, int F, bool kInt8>
static tq_status launch_prep(const tqd::PrepParams& pp, int parts, int64_t tiles, cudaStream_t st) {
  static PerDeviceOnce attr;
  if (const int dev_ = current_device(); attr.need(dev_)) {
    // the preparation kernel asks for the logits kernel's shared-memory
    // split, or its CTAs would keep logits CTAs off their SMs
    cudaError_t e = cudaFuncSetAttribute(tqd::prep_queries_kernel<E, F, kInt8>,
                                         cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return cuda_fail(e, "tq_logits: carveout attribute");
    attr.mark(dev_);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)parts, (unsigned)tiles);
  cfg.blockDim = dim3(tqd::kPrepThreads);
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, tqd::prep_queries_kernel<E, F, kInt8>, pp);
  if (e != cudaSuccess) return cuda_fail(e, "tq_logits: query preparation launch");
  return TQ_OK;
}

// One launch (the CTAs prepare their queries) when `prep` and d <= 128;
// otherwise the preparation kernel, then the logits kernel.
template <int BITS, int E, int F>
static tq_status run_logits(tqd::LogitsParams p, const tqd::PrepParams& pp, int parts, int64_t tiles,
                            int64_t units_per_cta, bool prep, cudaStream_t st) {
  LogitsPlan pl;
  if constexpr (E <= 32) {
    if (prep && logits_plan<BITS, E, F>(units_per_cta, true, &pl))
      return launch_logits_kernel<BITS, E, F, true>(p, pl, st);
  }
  if (!logits_plan<BITS, E, F>(units_per_cta, false, &pl))
    return fail(TQ_EUNSUPPORTED, "tq_logits: shared-memory plan");
  tq_status sp = launch_prep<E, F, BITS <= 3>(pp, parts, tiles, st);
  if (sp != TQ_OK) return sp;
  return launch_logits_kernel<BITS, E, F, false>(p, pl, st);
}

template <int BITS>
static tq_status dispatch_logits(const Layout& L, const tqd::LogitsParams& p, const tqd::PrepParams& pp,
                                 int parts, int64_t tiles, int64_t upc, bool prep, cudaStream_t st) {
  if (L.E == 32 && L.F == 32) return run_logits<BITS, 32, 32>(p, pp, parts, tiles, upc, prep, st);
  if (L.E == 32 && L.F == 0) return run_logits<BITS, 32, 0>(p, pp, parts, tiles, upc, prep, st);
  if (L.E == 16 && L.F == 16) return run_logits<BITS, 16, 16>(p, pp, parts, tiles, upc, prep, st);
  if (L.E == 16 && L.F == 0) return run_logits<BITS, 16, 0>(p, pp, parts, tiles, upc, prep, st);
  if (L.E == 64 && L.F == 64) return run_logits<BITS, 64, 64>(p, pp, parts, tiles, upc, prep, st);
  if (L.E == 64 && L.F == 0) return run_logits<BITS, 64, 0>(p, pp, parts, tiles, upc, prep, st);
  if (L.E == 48 && L.F == 48) return run_logits<BITS, 48, 48>(p, pp, parts, tiles, upc, prep, st);
  if (L.E == 48 && L.F == 0) return run_logits<BITS, 48, 0>(p, pp, parts, tiles, upc, prep, st);
  return fail(TQ_EUNSUPPORTED, "tq_logits: no kernel for this (d, m)");
}

// Byte-permute tables of the key codebook's reconstruction levels.
tqd::KeyTables key_tables(const tq_codebook* cb) {
  tqd::KeyTables kt;
  kt.t0 = cb->int8_levels[0];
  kt.t1 = cb->int8_levels[1];
  const uint16_t* M = cb->mag16;
  kt.lo0 = kt.lo1 = kt.hi0 = kt.hi1 = 0u;
  if (cb->lay.bits == 4) {
    for (int i = 0; i < 4; ++i) {
      kt.lo0 |= (uint32_t)(M[i] & 0xFF) << (8 * i);
      kt.lo1 |= (uint32_t)(M[4 + i] & 0xFF) << (8 * i);
      kt.hi0 |= (uint32_t)(M[i] >> 8) << (8 * i);
      kt.hi1 |= (uint32_t)(M[4 + i] >> 8) << (8 * i);
    }
  }
  return kt;
}

// Parameters of the preparation kernel writing into workspace `ws`.
static tqd::PrepParams prep_params(const tq_codebook* cb, const void* q, tq_dtype dt, int n_q_heads,
                                   int n_kv_heads, void* ws, const LogitsWs& wl) {
  const Layout& L = cb->lay;
  const int G = n_q_heads / n_kv_heads;
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  tqd::PrepParams pp;
  pp.q = q;
  pp.dtype = dt;
  pp.d = L.d;
  pp.n_q_heads = n_q_heads;
  pp.n_kv_heads = n_kv_heads;
  pp.G = G;
  pp.qtiles = (G + 3) / 4;
  pp.cb_unscale = std::ldexp(1.0f, -cb->table_exp);
  pp.qjl_scale = (float)cb->qjl_scale;
  // |(S q)_i| <= ||S_i|| ||q||: the float bound is rounded up
  pp.s_rowmax = (float)(cb->s_row_norm_max * (1.0 + 1e-6));
  pp.qprep = cb->qprep_frag;
  pp.frag = reinterpret_cast<uint2*>(wsb);
  pp.qfrag = reinterpret_cast<uint2*>(wsb + wl.frag);
  pp.scal = reinterpret_cast<float2*>(wsb + wl.frag + wl.qfrag);
  return pp;
}

size_t query_prep_workspace(const tq_codebook* cb, int64_t batch, int n_kv_heads, int n_q_heads) {
  return logits_ws_layout(cb, batch * n_kv_heads, n_q_heads / n_kv_heads, batch * n_q_heads).total;
}

tq_status launch_query_prep(const tq_codebook* cb, const void* q, tq_dtype dt, int64_t batch, int n_kv_heads,
                            int n_q_heads, void* ws, PreparedQueries* pq, cudaStream_t st) {
  const Layout& L = cb->lay;
  const int G = n_q_heads / n_kv_heads;
  const int64_t groups = batch * n_kv_heads;
  const int64_t tiles = groups * ((G + 3) / 4);
  if (groups > 65535 || tiles > 65535) return fail(TQ_EINVAL, "batch * n_kv_heads too large");
  const LogitsWs wl = logits_ws_layout(cb, groups, G, batch * n_q_heads);
  const tqd::PrepParams pp = prep_params(cb, q, dt, n_q_heads, n_kv_heads, ws, wl);
  pq->frag = pp.frag;
  pq->qfrag = pp.qfrag;
  pq->scal = pp.scal;
  const int parts = (L.d_pad + L.m_pad) / tqd::kPartRows;
  const bool i8 = L.bits <= 3;
  if (L.E == 32 && L.F == 32) return i8 ? launch_prep<32, 32, true>(pp, parts, tiles, st) : launch_prep<32, 32, false>(pp, parts, tiles, st);
  if (L.E == 32 && L.F == 0) return i8 ? launch_prep<32, 0, true>(pp, parts, tiles, st) : launch_prep<32, 0, false>(pp, parts, tiles, st);
  if (L.E == 16 && L.F == 16) return i8 ? launch_prep<16, 16, true>(pp, parts, tiles, st) : launch_prep<16, 16, false>(pp, parts, tiles, st);
  if (L.E == 16 && L.F == 0) return i8 ? launch_prep<16, 0, true>(pp, parts, tiles, st) : launch_prep<16, 0, false>(pp, parts, tiles, st);
  return fail(TQ_EUNSUPPORTED, "query preparation: no kernel for this (d, m)");
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
  const tqd::PrepParams pp = prep_params(cb, q, dt, n_q_heads, cv.n_kv_heads, ws, wl);
  uint2* frag = pp.frag;
  uint2* qfrag = pp.qfrag;
  float2* scal = pp.scal;
  int ps = 0;
  while ((1 << ps) < cv.page_tokens) ++ps;
  const int64_t units = (max_ctx + 63) / 64;
  const int parts = (L.d_pad + L.m_pad) / tqd::kPartRows;

  tqd::LogitsParams lp;
  lp.cv = cv;
  lp.page_shift = ps;
  lp.ctx_len = ctx_len;
  lp.n_kv_heads = cv.n_kv_heads;
  lp.n_q_heads = n_q_heads;
  lp.G = G;
  lp.qtiles = qtiles;
  lp.units = (int)units;
  lp.max_ctx = (int)max_ctx;
  // CTAs: one per SM, at least one per line (so a CTA spans at most two
  // lines) and enough that a CTA's block-table entries fit its staging
  // array; when every CTA would get fewer than 16 units (of 64 keys), four
  // times as many CTAs of 4 consumer warps (several per SM).
  const int64_t lines = groups * qtiles;
  const int64_t items = lines * units;
  const int64_t max_upc = (int64_t)(tqd::kLogitsPages - 4) * cv.page_tokens / 64;
  const int64_t n_sm = device_sm_count();
  int64_t n_cta = std::max(n_sm, lines);
  if ((items + n_cta - 1) / n_cta < 16) n_cta = std::max(4 * n_sm, lines);
  n_cta = std::max(n_cta, (items + max_upc - 1) / max_upc);
  n_cta = std::min(n_cta, items);
  if (n_cta > 0x7fffffffLL) return fail(TQ_EINVAL, "tq_logits: context too long");
  const int64_t upc = (items + n_cta - 1) / n_cta;
  if (items > 0x7fffffffLL) return fail(TQ_EINVAL, "tq_logits: batch * heads * context too large");
  lp.n_cta = (int)n_cta;
  lp.per_cta = (int)(items / n_cta);
  lp.extra = (int)(items % n_cta);
  lp.div_u = tqd::make_fastdiv((uint32_t)units);
  lp.div_qtiles = tqd::make_fastdiv((uint32_t)qtiles);
  lp.div_kv = tqd::make_fastdiv((uint32_t)cv.n_kv_heads);
  lp.q = q;
  lp.dtype = dt;
  lp.d = L.d;
  lp.d16 = (L.d + 15) / 16;
  lp.table = cb->qprep_frag;
  lp.prep_tiles = (L.d_pad + L.m_pad) / 16;
  lp.pc.cb_unscale = pp.cb_unscale;
  lp.pc.qjl_scale = pp.qjl_scale;
  lp.pc.s_rowmax = pp.s_rowmax;
  // the CTAs prepare their own queries when each gets enough units to
  // amortize loading the [Pi ; S] table (d <= 128)
  const bool prep = L.E <= 32 && upc >= kPrepMinUnits;
  lp.frag = frag;
  lp.qfrag = qfrag;
  lp.scal = scal;
  lp.out = out;
  lp.out_stride = out_stride;
  lp.kt = key_tables(cb);
  switch (L.bits) {
    case 1: return dispatch_logits<1>(L, lp, pp, parts, lines, upc, prep, st);
    case 2: return dispatch_logits<2>(L, lp, pp, parts, lines, upc, prep, st);
    case 3: return dispatch_logits<3>(L, lp, pp, parts, lines, upc, prep, st);
    case 4: return dispatch_logits<4>(L, lp, pp, parts, lines, upc, prep, st);
  }
  return fail(TQ_EUNSUPPORTED, "tq_logits: bits");
}

}  // namespace tq
