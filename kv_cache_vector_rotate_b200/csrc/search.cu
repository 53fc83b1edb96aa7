// Many-query scoring with a fused top-k: for every query head, the k largest
// estimated logits over a sequence's cached keys.
//
// "TurboQuant explained" (a2a-mcp.org), §Benchmarks (nearest-neighbour search
// scored from the codes, top-k recall) and §Stage 2 (the logit estimate).  The
// logit of query q against key n is the tq_logits estimate
//   L = ||k_n|| ( sum_j (Pi q)_j c[idx_nj] + sqrt(pi/2)/m ||r_n|| sum_i (S q)_i s_ni ).
// With many queries per key head this is a GEMM over the decoded codes, run on
// the tcgen05 tensor cores:
//  * A (M = 128 keys x K): each key's codes decoded into fp16 -- the
//    reconstruction levels (exact in fp16 at every width) and the signs +-1 --
//    by one thread per key, written straight into tensor memory
//    (tcgen05.st), one record chunk (E coordinates or sketch rows) at a time.
//    The MMAs read A from tensor memory, so the decoded operand never touches
//    shared memory.
//  * B (K x N): the queries of a 64-query tile, resident in shared memory in
//    the K-major 128-byte-swizzle layout: Pi q as fp16 hi + lo (N = 128: the
//    1e-3 logit tolerance needs more than fp16's 11 bits there) and
//    sqrt(pi/2)/m S q as fp16 (N = 64: the sketch term's rounding stays two
//    orders below the tolerance); each part is scaled by a power of two
//    (fp16 range) that the epilogue undoes.
//  * D (fp32, tensor memory, double-buffered): codebook sums [128 x 128] and
//    sketch sums [128 x 64]; L = ||k|| (c0 (D_hi + D_lo) + c1 ||r|| D_s).
// The epilogue keeps, per query, the k best (L, position) seen by the CTA
// (ties to the lower position): a row is appended to the query's candidate
// buffer when it reaches the query's threshold (the k-th best at the last
// cut), and a warp sorts a buffer and cuts it to the k best whenever it is
// half full, which raises the threshold.  A last kernel merges the CTAs'
// lists.
//
// Warp roles (18 warps): 0-7 decode (thread = key row, the tensor-memory
// lanes of warp w % 4; warps 0-3 the even A chunks of a tile, 4-7 the odd
// ones), 8-15 epilogue (thread = key row, lanes of warp w % 4; warps 8-11
// take the tile's queries 0-31, warps 12-15 queries 32-63), 16 copies the
// records of 128-key tiles into a ring (bulk copies, no multicast), 17
// issues the MMAs and owns the tensor memory.  Every wait is bounded; a CTA where one gives
// up reports TQ_DEV_ERR_TIMEOUT, lets its copies and MMAs finish, frees its
// tensor memory and returns.

#include <algorithm>
#include <cmath>

#include "pack.cuh"
#include "stream.cuh"
#include "value_tile.cuh"

namespace tqd {

constexpr int kSrQ = 64;           // queries per tile (line)
constexpr int kSrRows = 128;       // keys per tile
constexpr int kSrMaxK = 32;        // largest k
constexpr int kSrBuf = 64;         // candidate buffer per query (sorted and cut to k when half full)
constexpr int kSrRing = 2;         // record-ring slots
constexpr int kSrAbuf = 4;         // A chunk buffers in tensor memory
constexpr int kSrThreads = 576;    // 8 decoders, 8 epilogue, producer, MMA issuer
constexpr int kSrDecoders = 8;     // warps 0-7: two per tensor-memory quadrant (even / odd chunks)
constexpr int kSrEpi0 = 8;         // warps 8-15: epilogue
constexpr int kSrProducer = 16, kSrIssuer = 17;   // warp indices
constexpr float kSrNone = -INFINITY;
constexpr int kSrNoIdx = 0x7fffffff;

struct SearchParams {
  tq::CacheView cv;
  int page_shift;
  const int32_t* ctx_len;
  int n_kv_heads, n_q_heads, G, qtiles;   // qtiles = ceil(G / 64)
  int max_ctx;
  int row_tiles;                          // RT = ceil(max_ctx / 128)
  int64_t n_items;                        // lines * RT
  int per_cta, extra;                     // CTA c owns per_cta items, + 1 when c < extra
  int k;                                  // top-k
  // query preparation
  const void* q;
  tq_dtype dtype;
  int d;
  const float* pit32;                     // Pi^T [d][d_pad]
  const float* st32;                      // S^T [d][m_pad]
  float qjl_scale;
  float s_rowmax;
  // operands and results
  uint8_t* bimg;                          // [lines][image bytes]: the B operand, shared-memory image
  float2* scal;                           // [lines][64]: c0, c1
  float2* part;                           // [n_cta][2][64][k]: (score, position as float bits)
  uint32_t tlo0, tlo1, thi0, thi1;        // fp16 level bytes (b <= 3: levels; b = 4: magnitudes)
  float* out_score;                       // [batch][n_q_heads][k]
  int32_t* out_idx;
};

// Byte sizes for E coordinates / F sketch rows per chunk and W record words per chunk.
template <int E, int F, int W>
struct SrShape {
  static constexpr int kMseAtoms = E / 16;                 // 64-column K atoms of Pi q (4E columns)
  static constexpr int kQjlAtoms = F / 16;
  static constexpr int kMseAtomBytes = 2 * kSrQ * 128;     // 128 rows (hi, lo) x 128 bytes
  static constexpr int kQjlAtomBytes = kSrQ * 128;         // 64 rows x 128 bytes
  static constexpr int kImage = kMseAtoms * kMseAtomBytes + kQjlAtoms * kQjlAtomBytes;
  static constexpr int kRec = 16 * W;
  static constexpr int kNb = F > 0 ? 4 : 2;
  static constexpr int kHalf = (64 * (kRec + kNb) + 15) / 16 * 16;   // 64 keys: records then norms
  static constexpr int kSlot = 2 * kHalf;
  static constexpr int kChunks = F > 0 ? 8 : 4;            // A chunks per tile
  static constexpr int kCols = E / 2;                      // tensor-memory columns per chunk
  static constexpr int kSteps = E / 16;                    // K = 16 MMAs per chunk
};

struct SrMeta {
  int k1;          // keys of the tile inside the context
  uint32_t bad;    // bit j: keys 16 j .. 16 j + 15 are on a bad page
};

struct SrEntry {
  float s;
  int i;
};

struct SrState {
  uint64_t rec_full[kSrRing], rec_empty[kSrRing];
  uint64_t a_full[kSrAbuf], a_empty[kSrAbuf];
  uint64_t d_full[2], d_empty[2];
  uint64_t b_ready, mma_done;
  uint32_t tmem_base;
  int fail;

  SrMeta meta[kSrRing];
  float2 rowscale[4][kSrRows];              // ||k||, ||k|| ||r|| (x = -inf: the key does not count)
  int cnt[kSrQ];
  float4 qp[kSrQ];                          // c0, c1, the k-th entry's score and position (int bits)
  SrEntry buf[kSrQ][kSrBuf + 1];            // entries 0 .. cnt - 1 (+ 1: distinct banks per query)
};

// (a.s, a.i) ranks before (b.s, b.i): higher score, then lower position.
__device__ __forceinline__ bool sr_before(float as, int ai, float bs, int bi) {
  return as > bs || (as == bs && ai < bi);
}

// Instruction descriptor, kind::f16 with fp16 A and B (K-major), fp32 D, M = 128.
__host__ __device__ constexpr uint32_t sr_idesc(int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ uint64_t sr_desc(uint32_t smem_byte_addr) {
  // K-major, 128-byte swizzle: start >> 4, LBO 1 (unused), SBO 1024 >> 4, version 1, layout 2
  return (uint64_t)((smem_byte_addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// D (tensor memory) += A (tensor memory) B (shared memory descriptor).
__device__ __forceinline__ void sr_mma(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}"
      ::"r"(d), "r"(a), "l"(bdesc), "r"(idesc), "r"(acc) : "memory");
}
__device__ __forceinline__ void sr_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void sr_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void sr_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 8 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void sr_st8(uint32_t taddr, const uint32_t* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
               ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
// 16 consecutive 32-bit columns of this thread's lane (the caller waits).
__device__ __forceinline__ void sr_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t* u = reinterpret_cast<uint32_t*>(v);
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7])
               : "r"(taddr) : "memory");
}
__device__ __forceinline__ void sr_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t* u = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
        "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
      : "r"(taddr) : "memory");
}
// 32 consecutive 32-bit columns of this thread's lane (the caller waits).
__device__ __forceinline__ void sr_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t* u = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
        "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15]),
        "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]),
        "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
      : "r"(taddr) : "memory");
}

// Byte offset of B element (row n, column k) in a part whose atoms hold `rows` rows.
__device__ __forceinline__ uint32_t sr_bofs(int n, int k, int rows) {
  return (uint32_t)((k >> 6) * rows * 128 + n * 128 + ((((k & 63) >> 3) ^ (n & 7)) << 4) + (k & 7) * 2);
}

// ---- query preparation: one CTA (128 threads) per query slot of a line ----------
// grid: (64, lines).  Rows j < 4E of Pi q and i < 4F of S q in fp32 (Pi^T and
// S^T stored coalesced), each part scaled by 2^(14 - e) (2^(e-1) <= its bound
// < 2^e: |Pi q|_j <= ||q||, |c S q|_i <= c max_i ||S_i|| ||q||); slots past G
// get zeros.
template <int E, int F>
__global__ void __launch_bounds__(128) search_prep_kernel(SearchParams p) {
  using SH = SrShape<E, F, 1>;
  __shared__ float qs[256];
  __shared__ float red[4];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  const int qn = blockIdx.x, ln = blockIdx.y;
  const int gi = ln / p.qtiles, qt = ln % p.qtiles;
  const int b = gi / p.n_kv_heads, h = gi % p.n_kv_heads;
  const int hql = qt * kSrQ + qn;
  const bool valid = hql < p.G;
  const int d = p.d;
  const int64_t qoff = ((int64_t)b * p.n_q_heads + (int64_t)h * p.G + (valid ? hql : 0)) * d;
  float s2 = 0.0f;
  for (int k = threadIdx.x; k < d; k += 128) {
    const float x = valid ? load_elem(p.q, qoff + k, p.dtype) : 0.0f;
    qs[k] = x;
    s2 = fmaf(x, x, s2);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s2;
  __syncthreads();
  const float qn2 = (red[0] + red[1]) + (red[2] + red[3]);
  const float qnorm = sqrtf(qn2);
  int e0 = 0, e1 = 0;
  if (qnorm > 0.0f) frexpf(qnorm, &e0);
  const float sbound = p.qjl_scale * p.s_rowmax * qnorm;
  if (sbound > 0.0f) frexpf(sbound, &e1);
  const float up0 = ldexpf(1.0f, 14 - e0), up1 = ldexpf(1.0f, 14 - e1);
  uint8_t* img = p.bimg + (int64_t)ln * SH::kImage;
  constexpr int DP = 4 * E, MP = 4 * F;
  const int dpad = DP, mpad = MP;
  for (int j = threadIdx.x; j < DP; j += 128) {
    float v = 0.0f;
    if (j < d)
      for (int k = 0; k < d; ++k) v = fmaf(qs[k], p.pit32[(size_t)k * dpad + j], v);
    v *= up0;
    const __half hi = __float2half_rn(v);
    const __half lo = __float2half_rn(v - __half2float(hi));
    *reinterpret_cast<__half*>(img + sr_bofs(qn, j, 2 * kSrQ)) = hi;
    *reinterpret_cast<__half*>(img + sr_bofs(kSrQ + qn, j, 2 * kSrQ)) = lo;
  }
  if constexpr (F > 0) {
    uint8_t* qimg = img + SH::kMseAtoms * SH::kMseAtomBytes;
    for (int i = threadIdx.x; i < MP; i += 128) {
      float v = 0.0f;
      for (int k = 0; k < d; ++k) v = fmaf(qs[k], p.st32[(size_t)k * mpad + i], v);
      *reinterpret_cast<__half*>(qimg + sr_bofs(qn, i, kSrQ)) = __float2half_rn(v * p.qjl_scale * up1);
    }
  }
  if (threadIdx.x == 0) p.scal[(int64_t)ln * kSrQ + qn] = make_float2(ldexpf(1.0f, e0 - 14), ldexpf(1.0f, e1 - 14));
}

// ---- the scoring kernel -------------------------------------------------------------
// grid: n_cta CTAs (at least one per line: a CTA's items span at most two
// lines); CTA c takes items i0 .. i0 + n - 1 (item = line * RT + row tile).
template <int BITS, int E, int F>
__global__ void __launch_bounds__(kSrThreads, 1) search_kernel(SearchParams p) {
  using CW = ChunkWords<BITS, E, F>;
  constexpr int W = CW::W, NIDX = CW::q0;
  using SH = SrShape<E, F, W>;
  constexpr int REC = SH::kRec, NB = SH::kNb, HALF = SH::kHalf, NCH = SH::kChunks, NCOL = SH::kCols;
  constexpr uint32_t kColD = 192;                      // per accumulator buffer: codebook 128 + sketch 64
  constexpr uint32_t kColA = 384;                      // A chunk buffers
  extern __shared__ __align__(1024) uint8_t ssm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base_s = smem_addr(ssm);
  if (base_s & 1023u) {
    if (tid == 0) report(p.cv.err, TQ_DEV_ERR_CONFIG);
    return;
  }
  uint8_t* bsm = ssm;                                  // B image
  uint8_t* ring = ssm + SH::kImage;                    // record ring
  SrState& st = *reinterpret_cast<SrState*>(ring + kSrRing * SH::kSlot);
  const int c = blockIdx.x;
  const int64_t i0 = (int64_t)c * p.per_cta + min(c, p.extra);
  const int n_my = p.per_cta + (c < p.extra ? 1 : 0);
  const int RT = p.row_tiles;
  const int K = p.k;
  const int line0 = (int)(i0 / RT);

  if (tid == 0) {
    for (int s = 0; s < kSrRing; ++s) {
      mbar_init(&st.rec_full[s], 1);
      mbar_init(&st.rec_empty[s], kSrDecoders);
    }
    for (int s = 0; s < kSrAbuf; ++s) {
      mbar_init(&st.a_full[s], 4);
      mbar_init(&st.a_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&st.d_full[s], 1);
      mbar_init(&st.d_empty[s], 8);
    }
    mbar_init(&st.b_ready, 1);
    mbar_init(&st.mma_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    st.fail = 0;

  }
  if (warp == kSrIssuer) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_addr(&st.tmem_base)), "r"(512) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid < kSrQ) st.cnt[tid] = 0;
  sr_fence_before();
  __syncthreads();
  sr_fence_after();
  asm volatile("griddepcontrol.wait;" ::: "memory");   // the query operands come from the preparation kernel
  const uint32_t tmem = st.tmem_base;
  auto fail_now = [&]() {
    atomicOr(&st.fail, 1);
    report(p.cv.err, TQ_DEV_ERR_TIMEOUT);
  };
  auto item_line = [&](int t) { return (int)((i0 + t) / RT); };
  auto item_rt = [&](int t) { return (int)((i0 + t) % RT); };

  if (warp == kSrProducer) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = evict_first_policy();
      const int ps = p.page_shift, P = 1 << ps;
      int issued = 0;
      for (int t = 0; t < n_my; ++t) {
        const int slot = t % kSrRing;
        if (t >= kSrRing && !mbar_wait_backoff(&st.rec_empty[slot], (uint32_t)((t / kSrRing) - 1) & 1u)) {
          fail_now();
          break;
        }
        if (st.fail) break;
        const int ln = item_line(t), rt = item_rt(t);
        const int gi = ln / p.qtiles;
        const int b = gi / p.n_kv_heads, h = gi % p.n_kv_heads;
        const int r0 = rt * kSrRows;
        const int ctx = min(max(p.ctx_len[b], 0), p.max_ctx);
        const int k1 = max(0, min(kSrRows, ctx - r0));
        // pages of the tile's 16-key pieces (a piece never straddles a page)
        uint32_t bad = 0u, bytes = 0u;
        int64_t off[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          off[j] = -1;
          if (16 * j < k1) {
            const int pos = r0 + 16 * j;
            const int64_t pg = p.cv.block_table[(int64_t)b * p.cv.max_pages + (pos >> ps)];
            if (pg < 0 || pg >= p.cv.n_pages) {
              bad |= 1u << j;
              report(p.cv.err, TQ_DEV_ERR_PAGE);
            } else {
              off[j] = pg * p.cv.page_bytes + (int64_t)h * p.cv.head_block_bytes;
            }
          }
        }
        // a 64-key half inside the context on good pages of >= 64 keys goes
        // in one copy (64-key pages: the head block is records then norms,
        // as the slot) or two (records, norms)
        bool whole[2];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          whole[hf] = P >= 64 && 64 * hf + 64 <= k1 && ((bad >> (4 * hf)) & 15u) == 0u;
          if (whole[hf]) bytes += P == 64 ? (uint32_t)HALF : 64u * (REC + NB);
          else
            for (int j = 4 * hf; j < 4 * hf + 4; ++j)
              if (off[j] >= 0) bytes += 16 * (REC + NB);
        }
        st.meta[slot].k1 = k1;
        st.meta[slot].bad = bad;
        uint64_t* bar = &st.rec_full[slot];
        const uint32_t dst = smem_addr(ring + slot * SH::kSlot);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive_tx(bar, bytes);
        for (int hf = 0; hf < 2; ++hf) {
          if (!whole[hf]) continue;
          const int pos = r0 + 64 * hf, sl = pos & (P - 1);
          const uint8_t* hb = p.cv.pages + off[4 * hf];
          if (P == 64) {
            bulk_copy(dst + hf * HALF, hb, HALF, bar, pol);
          } else {
            bulk_copy(dst + hf * HALF, hb + (int64_t)sl * REC, 64 * REC, bar, pol);
            bulk_copy(dst + hf * HALF + 64 * REC, hb + (int64_t)P * REC + sl * NB, 64 * NB, bar, pol);
          }
        }
        for (int j = 0; j < 8; ++j) {
          if (off[j] < 0 || whole[j >> 2]) continue;
          const int pos = r0 + 16 * j, sl = pos & (P - 1);
          const int hf = j >> 2, w16 = (j & 3) * 16;    // half of the slot, key within the half
          const uint8_t* hb = p.cv.pages + off[j];
          bulk_copy(dst + hf * HALF + w16 * REC, hb + (int64_t)sl * REC, 16 * REC, bar, pol);
          bulk_copy(dst + hf * HALF + 64 * REC + w16 * NB, hb + (int64_t)P * REC + sl * NB, 16 * NB, bar, pol);
        }
        issued = t + 1;
      }
      // the copies issued land before the CTA exits
      for (int t = max(0, issued - kSrRing); t < issued; ++t)
        mbar_wait(&st.rec_full[t % kSrRing], (uint32_t)(t / kSrRing) & 1u);
    }
  } else if (warp == kSrIssuer) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_cb = sr_idesc(2 * kSrQ), id_s = sr_idesc(kSrQ);
      int cur_line = -1, b_phase = 0, a_cnt = 0, md_phase = 0;
      bool ok = true;
      for (int t = 0; t < n_my && ok; ++t) {
        const int ln = item_line(t);
        if (ln != cur_line) {
          // a new line: every MMA of the previous one is done with B, then B
          // is replaced
          if (cur_line >= 0) {
            sr_commit(&st.mma_done);
            if (!mbar_wait(&st.mma_done, (uint32_t)md_phase & 1u)) { ok = false; fail_now(); break; }
            ++md_phase;
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          mbar_arrive_tx(&st.b_ready, SH::kImage);
          bulk_copy_plain(base_s, p.bimg + (int64_t)ln * SH::kImage, SH::kImage, &st.b_ready);
          if (!mbar_wait(&st.b_ready, (uint32_t)b_phase & 1u)) { ok = false; fail_now(); break; }
          ++b_phase;
          cur_line = ln;
        }
        const int db = t & 1;
        if (t >= 2 && !mbar_wait_backoff(&st.d_empty[db], (uint32_t)((t >> 1) - 1) & 1u, 64u)) { ok = false; fail_now(); break; }
        sr_fence_after();
        const uint32_t dcb = tmem + db * kColD, ds = dcb + 2 * kSrQ;
        for (int ch = 0; ch < NCH; ++ch, ++a_cnt) {
          const int ab = a_cnt % kSrAbuf;
          if (!mbar_wait_backoff(&st.a_full[ab], (uint32_t)(a_cnt / kSrAbuf) & 1u, 64u)) { ok = false; fail_now(); break; }
          sr_fence_after();
          const uint32_t abase = tmem + kColA + ab * NCOL;
          const bool sk = ch >= 4;
#pragma unroll
          for (int ks = 0; ks < SH::kSteps; ++ks) {
            const int kg = (sk ? ch - 4 : ch) * SH::kSteps + ks;   // K step within the part
            const uint32_t boff = sk ? SH::kMseAtoms * SH::kMseAtomBytes + (kg >> 2) * SH::kQjlAtomBytes + (kg & 3) * 32
                                     : (kg >> 2) * SH::kMseAtomBytes + (kg & 3) * 32;
            sr_mma(sk ? ds : dcb, abase + 8 * ks, sr_desc(base_s + boff), sk ? id_s : id_cb,
                   (kg > 0) ? 1u : 0u);
          }
          sr_commit(&st.a_empty[ab]);
        }
        if (!ok) break;
        sr_commit(&st.d_full[db]);
      }
      // every MMA issued is complete before the tensor memory is freed
      sr_commit(&st.mma_done);
      mbar_wait(&st.mma_done, (uint32_t)md_phase & 1u);
    }
  } else if (warp < kSrDecoders) {
    // ------------------------------------------------------------ decoders
    const int r = tid & 127;                        // key row of the tile = tensor-memory lane
    const int parity = warp >> 2;                   // this warp's chunks: parity, parity + 2, ...
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    for (int t = 0; t < n_my; ++t) {
      const int slot = t % kSrRing;
      // warp-uniform exits: the tensor-memory stores below are warp-wide
      if (!__all_sync(0xffffffffu, mbar_wait_backoff(&st.rec_full[slot], (uint32_t)(t / kSrRing) & 1u))) {
        if (lane == 0) fail_now();
        break;
      }
      if (__any_sync(0xffffffffu, st.fail != 0)) break;
      const SrMeta mt = st.meta[slot];
      const bool valid = r < mt.k1 && !((mt.bad >> (r >> 4)) & 1u);
      const uint8_t* hb = ring + slot * SH::kSlot + (r >> 6) * HALF;
      const uint8_t* rec = hb + (r & 63) * REC;
      float2 rs = make_float2(kSrNone, 0.0f);
      if (valid) {
        if constexpr (F > 0) {
          const uint32_t nw = *reinterpret_cast<const uint32_t*>(hb + 64 * REC + (r & 63) * 4);
          const float nk = __half2float(__ushort_as_half((unsigned short)(nw & 0xFFFFu)));
          const float nr = __half2float(__ushort_as_half((unsigned short)(nw >> 16)));
          rs = make_float2(nk, nk * nr);
        } else {
          rs = make_float2(__half2float(*reinterpret_cast<const __half*>(hb + 64 * REC + (r & 63) * 2)), 0.0f);
        }
      }
      if (parity == 0) st.rowscale[t & 3][r] = rs;
      bool ok = true;
      for (int ch = parity; ch < NCH; ch += 2) {
        const int a_cnt = t * NCH + ch;             // the chunk's place in the A-buffer sequence
        const int ab = a_cnt % kSrAbuf;
        if (a_cnt >= kSrAbuf &&
            !__all_sync(0xffffffffu, mbar_wait_backoff(&st.a_empty[ab], (uint32_t)((a_cnt / kSrAbuf) - 1) & 1u, 128u))) {
          ok = false;
          break;
        }
        uint32_t v[NCOL];
        const uint32_t* cw = reinterpret_cast<const uint32_t*>(rec + (ch & 3) * 4 * W);
        if (ch < 4) {
#pragma unroll
          for (int kk = 0; kk < E / 8; ++kk) {
            const uint4 q4 = decode8<BITS, E>(cw, kk, p);
            v[4 * kk] = q4.x; v[4 * kk + 1] = q4.y; v[4 * kk + 2] = q4.z; v[4 * kk + 3] = q4.w;
          }
        } else if constexpr (F > 0) {
          // sketch row l: word l / 32, bit 8 (l % 4) + (l % 32) / 4; rows 2j, 2j + 1 -> column j (+-1 as fp16)
#pragma unroll
          for (int wq = 0; wq < (F + 31) / 32; ++wq) {
            const uint32_t w = cw[NIDX + wq];
            const uint32_t x0 = prmt(w, 0u, 0x1404u);   // bytes 0, 1 -> 1, 3
            const uint32_t x1 = prmt(w, 0u, 0x3424u);   // bytes 2, 3 -> 1, 3
#pragma unroll
            for (int kq = 0; kq < 8; ++kq) {
              if (32 * wq + 4 * kq < F) {
                v[16 * wq + 2 * kq] = ((x0 << (7 - kq)) & 0x80008000u) | 0x3C003C00u;
                v[16 * wq + 2 * kq + 1] = ((x1 << (7 - kq)) & 0x80008000u) | 0x3C003C00u;
              }
            }
          }
        }
        const uint32_t ta = tmem + lane_base + kColA + ab * NCOL;
#pragma unroll
        for (int x = 0; x < NCOL / 8; ++x) sr_st8(ta + 8 * x, v + 8 * x);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        sr_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&st.a_full[ab]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&st.rec_empty[slot]);
      if (!ok) {
        if (lane == 0) fail_now();
        break;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // epilogue warp ew (0-7): tensor-memory quadrant ew % 4 (its rows r),
    // queries 32 (ew / 4) .. + 31 of the tile (8-query column groups G0 .. G0 + 3)
    const int er = tid - 32 * kSrEpi0;              // 0 .. 255
    const int ew = warp - kSrEpi0;
    const int r = er & 127;
    const int G0 = 4 * (ew >> 2);
    const uint32_t lane_base = (uint32_t)(32 * (ew & 3)) << 16;
    auto ebar = [&]() { asm volatile("barrier.sync 1, 256;" ::: "memory"); };
    // the same barrier, returning whether any epilogue thread passed `v`
    auto ebar_or = [&](bool v) -> bool {
      uint32_t any;
      asm volatile(
          "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n barrier.red.or.pred q, 1, 256, p;\n"
          " selp.u32 %0, 1, 0, q;\n}"
          : "=r"(any) : "r"(v ? 1u : 0u) : "memory");
      return any != 0u;
    };
    int cur_line = line0;
    // a line's query scales, and empty thresholds
    // (query slots past G never take a candidate: their threshold is +inf)
    auto load_scales = [&](int ln) {
      if (er < kSrQ) {
        const float2 sc = p.scal[(int64_t)ln * kSrQ + er];
        const bool real = (ln % p.qtiles) * kSrQ + er < p.G;
        st.qp[er] = make_float4(sc.x, sc.y, real ? kSrNone : INFINITY, __int_as_float(kSrNoIdx));
      }
      ebar();
    };
    load_scales(cur_line);
    // warp-wide: sort query q's buffer (best first, ties to the lower
    // position), keep the k best and raise the threshold
    auto cut = [&](int q) {
      const int n = min(st.cnt[q], kSrBuf);
      SrEntry a = lane < n ? st.buf[q][lane] : SrEntry{kSrNone, kSrNoIdx};
      SrEntry bb = lane + 32 < n ? st.buf[q][lane + 32] : SrEntry{kSrNone, kSrNoIdx};
      // bitonic sort of the 64 elements e = lane (a) and e = lane + 32 (bb)
#pragma unroll
      for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          if (stride == 32) {
            if (sr_before(bb.s, bb.i, a.s, a.i)) {
              const SrEntry tmp = a;
              a = bb;
              bb = tmp;
            }
          } else {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              SrEntry& v = half == 0 ? a : bb;
              const int e = lane + 32 * half;
              const float os = __shfl_xor_sync(0xffffffffu, v.s, stride);
              const int oi = __shfl_xor_sync(0xffffffffu, v.i, stride);
              const bool lower = (e & stride) == 0;
              const bool up = (e & size) == 0;           // best first where up
              const bool mine_first = sr_before(v.s, v.i, os, oi);
              if ((lower == up) != mine_first) {
                v.s = os;
                v.i = oi;
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane < K) st.buf[q][lane] = a;
      const float ks = __shfl_sync(0xffffffffu, a.s, K - 1);
      const int ki = __shfl_sync(0xffffffffu, a.i, K - 1);
      __syncwarp();
      if (lane == 0) {
        st.cnt[q] = min(n, K);
        if (n >= K) {
          st.qp[q].z = ks;
          st.qp[q].w = __int_as_float(ki);
        }
      }
      __syncwarp();
    };
    // the lists of the finished line go to the partials; the buffers restart
    auto flush = [&](int seg) {
      for (int qi = 0; qi < 8; ++qi) {
        const int q = 8 * ew + qi;
        if (st.cnt[q] > 0) cut(q);
      }
      ebar();
      for (int x = er; x < kSrQ * K; x += 256) {
        const int q = x / K, kk = x % K;
        const SrEntry e = kk < st.cnt[q] ? st.buf[q][kk] : SrEntry{kSrNone, kSrNoIdx};
        p.part[(((int64_t)c * 2 + seg) * kSrQ + q) * K + kk] = make_float2(e.s, __int_as_float(e.i));
      }
      ebar();
      if (er < kSrQ) st.cnt[er] = 0;
      ebar();
    };
    for (int t = 0; t < n_my; ++t) {
      const int ln = item_line(t);
      if (ln != cur_line) {
        flush(0);
        cur_line = ln;
        load_scales(ln);
      }
      const int db = t & 1;
      // the epilogue warps leave together (named barriers follow): one
      // barrier that also tells every warp whether any wait gave up
      const bool got = mbar_wait_backoff(&st.d_full[db], (uint32_t)(t >> 1) & 1u, 128u);
      if (ebar_or(!got)) {
        if (er == 0) fail_now();
        break;
      }
      sr_fence_after();
      const float2 rs = st.rowscale[t & 3][r];
      const int pos = item_rt(t) * kSrRows + r;
      const uint32_t dcb = tmem + lane_base + db * kColD, ds = dcb + 2 * kSrQ;
      uint32_t consider = rs.x == kSrNone ? 0u : 0xffffffffu;   // this warp's queries the row still competes for
      for (int round = 0; round < 64; ++round) {
        bool ovf = false;                            // a hit of this thread did not fit its buffer
        // 1. scores of this row for 8 queries at a time (their constants
        //    loaded first); those that reach the query's threshold are
        //    appended to its buffer, one shared-memory atomic per hit
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int G = G0 + g;                      // column group: queries 8 G .. 8 G + 7
          const uint32_t want = (consider >> (8 * g)) & 0xFFu;
          if (!__any_sync(0xffffffffu, want != 0u)) continue;   // warp-uniform
          float vh[8], vl[8], vs[8];
          sr_ld8(dcb + 8 * G, vh);
          sr_ld8(dcb + kSrQ + 8 * G, vl);
          if constexpr (F > 0) sr_ld8(ds + 8 * G, vs);
          float4 qv[8];
#pragma unroll
          for (int x = 0; x < 8; ++x) qv[x] = st.qp[8 * G + x];   // broadcast loads
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          uint32_t hit = 0u;
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            float sv = qv[x].x * (vh[x] + vl[x]);
            if constexpr (F > 0) sv = fmaf(qv[x].y * rs.y, vs[x], rs.x * sv);
            else sv = rs.x * sv;
            vh[x] = sv;
            // ranks before the threshold entry: higher, or equal at a lower position
            const bool beats = sv > qv[x].z || (sv == qv[x].z && pos < __float_as_int(qv[x].w));
            hit |= (beats ? 1u : 0u) << x;
          }
          hit &= want;
          uint32_t keep = 0u;                        // hits that did not fit (retried after the cut)
          // each lane appends its own hits, one shared-memory atomic per hit:
          // the lanes' atomics go out together, so a warp waits for about as
          // many round trips as its busiest lane has hits (usually 0 or 1)
          for (uint32_t h = hit; h != 0u; h &= h - 1u) {
            const int x = __ffs(h) - 1;
            const int q = 8 * G + x;
            const int slot = atomicAdd(&st.cnt[q], 1);
            float sv = 0.0f;
#pragma unroll
            for (int y = 0; y < 8; ++y)
              if (y == x) sv = vh[y];
            if (slot < kSrBuf) st.buf[q][slot] = {sv, pos};
            else keep |= 1u << x;
          }
          __syncwarp();
          if (keep) ovf = true;
          const uint32_t sh = 8 * g;
          consider = (consider & ~(0xFFu << sh)) | (keep << sh);
        }
        ebar();
        // 2. buffers half full (or full) are cut to the k best
        for (int qi = 0; qi < 8; ++qi) {
          const int q = 8 * ew + qi;
          if (st.cnt[q] >= kSrBuf / 2) cut(q);
        }
        // every cut is done; another round only if some hit did not fit
        if (!ebar_or(ovf)) break;
      }
      sr_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&st.d_empty[db]);
    }
    if (n_my > 0) flush(item_line(n_my - 1) != line0 ? 1 : 0);
  }

  // every role is done: the tensor memory is freed
  sr_fence_before();
  __syncthreads();
  sr_fence_after();
  if (warp == kSrIssuer)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
}

// ---- merge of the CTAs' lists: one warp per query ---------------------------------------
// grid: lines * 8 CTAs of 256 threads (8 query slots each).
__global__ void __launch_bounds__(256) search_finish_kernel(SearchParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int ln = blockIdx.x / 8, q = (blockIdx.x % 8) * 8 + (threadIdx.x >> 5);
  const int gi = ln / p.qtiles, qt = ln % p.qtiles;
  const int b = gi / p.n_kv_heads, h = gi % p.n_kv_heads;
  const int hql = qt * kSrQ + q;
  if (hql >= p.G) return;
  const int K = p.k;
  const int64_t x0 = (int64_t)ln * p.row_tiles, x1 = x0 + p.row_tiles - 1;
  const int64_t big = (int64_t)p.extra * (p.per_cta + 1);
  auto cta_of = [&](int64_t x) -> int {
    return (int)(x < big ? x / (p.per_cta + 1) : p.extra + (x - big) / max(p.per_cta, 1));
  };
  const int c_a = cta_of(x0), c_b = cta_of(x1);
  const int n_lists = c_b - c_a + 1;
  // lane l walks lists l, l + 32, ... with a head pointer each (at most 8 per lane)
  int head[8];
  const float2* src[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    head[j] = 0;
    src[j] = nullptr;
    const int li = lane + 32 * j;
    if (li < n_lists) {
      const int cc = c_a + li;
      const int64_t ci0 = (int64_t)cc * p.per_cta + min(cc, p.extra);
      const int seg = ln - (int)(ci0 / p.row_tiles);
      src[j] = p.part + (((int64_t)cc * 2 + seg) * kSrQ + q) * K;
    }
  }
  const int64_t obase = ((int64_t)b * p.n_q_heads + (int64_t)h * p.G + hql) * K;
  for (int kk = 0; kk < K; ++kk) {
    float bs = kSrNone;
    int bi = kSrNoIdx, bj = -1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (src[j] && head[j] < K) {
        const float2 e = src[j][head[j]];
        const int ei = __float_as_int(e.y);
        if (ei != kSrNoIdx && sr_before(e.x, ei, bs, bi)) {
          bs = e.x;
          bi = ei;
          bj = j;
        }
      }
    }
    // warp arg-best
    float ws = bs;
    int wi = bi, wl = lane;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, ws, o);
      const int oi = __shfl_xor_sync(0xffffffffu, wi, o);
      const int ol = __shfl_xor_sync(0xffffffffu, wl, o);
      if (sr_before(os, oi, ws, wi) || (os == ws && oi == wi && ol < wl)) {
        ws = os;
        wi = oi;
        wl = ol;
      }
    }
    if (lane == wl && bj >= 0) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j == bj) ++head[j];
    }
    if (lane == 0) {
      p.out_score[obase + kk] = wi == kSrNoIdx ? kSrNone : ws;
      p.out_idx[obase + kk] = wi == kSrNoIdx ? -1 : wi;
    }
  }
}

}  // namespace tqd

namespace tq {

struct SearchLayout {
  int64_t lines, row_tiles, items, n_cta;
  size_t img, scal, part, total;
};

static SearchLayout search_layout(const tq_codebook* cb, int64_t batch, int n_kv_heads, int n_q_heads,
                                  int64_t max_ctx, int k) {
  auto al = [](size_t n) { return (n + 255) / 256 * 256; };
  const Layout& L = cb->lay;
  SearchLayout s;
  const int G = n_q_heads / n_kv_heads;
  s.lines = batch * n_kv_heads * ((G + tqd::kSrQ - 1) / tqd::kSrQ);
  s.row_tiles = (max_ctx + tqd::kSrRows - 1) / tqd::kSrRows;
  s.items = s.lines * s.row_tiles;
  s.n_cta = std::min<int64_t>(s.items, std::max<int64_t>(device_sm_count(), s.lines));
  const size_t image = (size_t)(L.E / 16) * 2 * tqd::kSrQ * 128 + (size_t)(L.F / 16) * tqd::kSrQ * 128;
  s.img = al((size_t)s.lines * image);
  s.scal = al((size_t)s.lines * tqd::kSrQ * sizeof(float2));
  s.part = al((size_t)std::max<int64_t>(s.n_cta, 1) * 2 * tqd::kSrQ * k * sizeof(float2));
  s.total = s.img + s.scal + s.part;
  return s;
}

size_t search_workspace(const tq_codebook* cb, int64_t batch, int n_kv_heads, int n_q_heads, int64_t max_ctx, int k) {
  return search_layout(cb, batch, n_kv_heads, n_q_heads, max_ctx, k).total;
}

template <int BITS, int E, int F>
static tq_status launch_search_t(const tqd::SearchParams& p, int64_t lines, int64_t n_cta, cudaStream_t st) {
  using CW = tqd::ChunkWords<BITS, E, F>;
  using SH = tqd::SrShape<E, F, CW::W>;
  const size_t smem = (size_t)SH::kImage + tqd::kSrRing * SH::kSlot + sizeof(tqd::SrState) + 1024;
  static PerDeviceOnce attr;
  if (const int dev_ = current_device(); attr.need(dev_)) {
    cudaError_t e = cudaFuncSetAttribute(tqd::search_kernel<BITS, E, F>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "tq_logits_topk: smem attribute");
    attr.mark(dev_);
  }
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = st;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(tqd::kSrQ, (unsigned)lines);
  cfg.blockDim = dim3(128);
  cudaError_t e = cudaLaunchKernelEx(&cfg, tqd::search_prep_kernel<E, F>, p);
  if (e != cudaSuccess) return cuda_fail(e, "tq_logits_topk: query preparation launch");
  cfg.gridDim = dim3((unsigned)n_cta);
  cfg.blockDim = dim3(tqd::kSrThreads);
  cfg.dynamicSmemBytes = smem;
  e = cudaLaunchKernelEx(&cfg, tqd::search_kernel<BITS, E, F>, p);
  if (e != cudaSuccess) return cuda_fail(e, "tq_logits_topk: scoring launch");
  cfg.gridDim = dim3((unsigned)(lines * 8));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  e = cudaLaunchKernelEx(&cfg, tqd::search_finish_kernel, p);
  if (e != cudaSuccess) return cuda_fail(e, "tq_logits_topk: merge launch");
  return TQ_OK;
}

template <int BITS>
static tq_status dispatch_search(const Layout& L, const tqd::SearchParams& p, int64_t lines, int64_t n_cta,
                                 cudaStream_t st) {
  if (L.E == 64 && L.F == 64) return launch_search_t<BITS, 64, 64>(p, lines, n_cta, st);
  if (L.E == 64 && L.F == 0) return launch_search_t<BITS, 64, 0>(p, lines, n_cta, st);
  if (L.E == 48 && L.F == 48) return launch_search_t<BITS, 48, 48>(p, lines, n_cta, st);
  if (L.E == 48 && L.F == 0) return launch_search_t<BITS, 48, 0>(p, lines, n_cta, st);
  if (L.E == 32 && L.F == 32) return launch_search_t<BITS, 32, 32>(p, lines, n_cta, st);
  if (L.E == 32 && L.F == 0) return launch_search_t<BITS, 32, 0>(p, lines, n_cta, st);
  if (L.E == 16 && L.F == 16) return launch_search_t<BITS, 16, 16>(p, lines, n_cta, st);
  if (L.E == 16 && L.F == 0) return launch_search_t<BITS, 16, 0>(p, lines, n_cta, st);
  return fail(TQ_EUNSUPPORTED, "tq_logits_topk: no kernel for this (d, m)");
}

tq_status launch_search(const tq_codebook* cb, const CacheView& cv, const void* q, tq_dtype dt, int64_t batch,
                        int n_q_heads, const int32_t* ctx_len, int64_t max_ctx, int k, float* out_score,
                        int32_t* out_idx, void* ws, size_t ws_bytes, cudaStream_t st) {
  const Layout& L = cb->lay;
  const SearchLayout s = search_layout(cb, batch, cv.n_kv_heads, n_q_heads, max_ctx, k);
  if (!ws || ws_bytes < s.total) return fail(TQ_EINVAL, "tq_logits_topk: workspace too small");
  if (s.lines > 65535 || s.items > 0x7fffffffLL || s.lines * 8 > 0x7fffffffLL)
    return fail(TQ_EINVAL, "tq_logits_topk: batch * heads * context too large");
  tqd::SearchParams p;
  p.cv = cv;
  int ps = 0;
  while ((1 << ps) < cv.page_tokens) ++ps;
  p.page_shift = ps;
  p.ctx_len = ctx_len;
  p.n_kv_heads = cv.n_kv_heads;
  p.n_q_heads = n_q_heads;
  p.G = n_q_heads / cv.n_kv_heads;
  p.qtiles = (p.G + tqd::kSrQ - 1) / tqd::kSrQ;
  p.max_ctx = (int)max_ctx;
  p.row_tiles = (int)s.row_tiles;
  p.n_items = s.items;
  p.per_cta = (int)(s.items / s.n_cta);
  p.extra = (int)(s.items % s.n_cta);
  p.k = k;
  p.q = q;
  p.dtype = dt;
  p.d = L.d;
  p.pit32 = cb->pit32;
  p.st32 = cb->st32;
  p.qjl_scale = (float)cb->qjl_scale;
  p.s_rowmax = (float)(cb->s_row_norm_max * (1.0 + 1e-6));
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  p.bimg = base;
  p.scal = reinterpret_cast<float2*>(base + s.img);
  p.part = reinterpret_cast<float2*>(base + s.img + s.scal);
  const uint16_t* T = L.bits == 4 ? cb->mag16 : cb->cent16;   // 8 entries
  p.tlo0 = p.tlo1 = p.thi0 = p.thi1 = 0u;
  for (int i = 0; i < 4; ++i) {
    p.tlo0 |= (uint32_t)(T[i] & 0xFF) << (8 * i);
    p.tlo1 |= (uint32_t)(T[4 + i] & 0xFF) << (8 * i);
    p.thi0 |= (uint32_t)(T[i] >> 8) << (8 * i);
    p.thi1 |= (uint32_t)(T[4 + i] >> 8) << (8 * i);
  }
  p.out_score = out_score;
  p.out_idx = out_idx;
  switch (L.bits) {
    case 1: return dispatch_search<1>(L, p, s.lines, s.n_cta, st);
    case 2: return dispatch_search<2>(L, p, s.lines, s.n_cta, st);
    case 3: return dispatch_search<3>(L, p, s.lines, s.n_cta, st);
    case 4: return dispatch_search<4>(L, p, s.lines, s.n_cta, st);
  }
  return fail(TQ_EUNSUPPORTED, "tq_logits_topk: bits");
}

}  // namespace tq
