// Quantize-and-append on the tcgen05 tensor cores (head_dim 128, bf16 input).
//
// "TurboQuant explained" (a2a-mcp.org) §Stage 1: normalize, rotate by Pi,
// map each rotated coordinate to its Lloyd-Max cell; §Stage 2: signs of a
// Gaussian projection of the residual; §How to implement: quantize on every
// cache update.  For a tile of 128 vectors X (rows) both projections are
// dense contractions:
//    Y = X Pi^T          (128 x 128 x 128)
//    P = R S_rot^T       (128 x m x 128),  S_rot = S Pi^T, R the residuals
// run as tcgen05 MMAs (M = N = 128, K = 16, bf16 operands from shared memory,
// fp32 accumulators in tensor memory).  Pi and S_rot are split into bf16 hi +
// lo (the input is bf16, so X Pi^T = X Pi_hi + X Pi_lo to fp32 rounding); R
// is split as well, and P = R_hi S_hi + R_hi S_lo + R_lo S_hi.
//
// One persistent CTA of 16 warps per SM keeps Pi and S_rot resident (128 KB)
// and walks 128-vector tiles.  X tiles arrive by TMA (two boxes of 64
// columns, 128-byte swizzle) into one of two buffers; Y is double-buffered in
// tensor memory, so the rotation of the next tile runs while this tile's
// epilogue does.  Warp w reads rows 32 (w % 4) .. + 31 (its tensor-memory
// lanes) and chunk w / 4 (32 coordinates) of each: the thread quantizes its
// 32 coordinates, writes their residual into the operand tiles of the
// sketch (R hi over the spent X buffer, R lo in its own tile), later turns
// its 32 entries of P into sign bits, and stores its chunk of the record.
//
// Shared-memory operands use the K-major 128-byte-swizzle canonical layout:
// a 128 x 128 bf16 operand is two K-atoms of 128 rows x 128 bytes (16 KB,
// 1024-byte aligned); 16-byte chunk c of row r sits at chunk c ^ (r % 8),
// which is the layout a TMA box of 64 bf16 columns with 128-byte swizzle
// writes.

#include <cudaTypedefs.h>

#include "pack.cuh"
#include "stream.cuh"

namespace tqd {

constexpr int kQtcThreads = 512;                  // 16 warps: rows 32 (w % 4) .., chunk w / 4
constexpr int kOpBytes = 128 * 128 * 2;           // one 128 x 128 bf16 operand
constexpr int kAtomBytes = 128 * 128;             // one K-atom: 128 rows x 64 bf16

struct QuantizeTcParams {
  int64_t rows, n_new;       // rows = batch * n_kv_heads * n_new
  int n_kv_heads;
  const int32_t* start_pos;
  tq::CacheView cv;
  const __nv_bfloat16* pi_bf;    // [2][128][128]: hi, lo of Pi[j][k]
  const __nv_bfloat16* srot_bf;  // [2][128][128]: hi, lo of (S Pi^T)[i][j]
  const float* bound32;          // [2^b - 1]
  const float* cent32;           // [2^b] the reconstruction levels
  int64_t n_tiles;
};

// Byte offset of element (row r, k) in a K-major SW128 128 x 128 bf16 operand.
__device__ __forceinline__ uint32_t sw128_offset(int r, int k) {
  const int atom = k >> 6, c = (k & 63) >> 3;
  return (uint32_t)(atom * 16384 + r * 128 + ((c ^ (r & 7)) << 4) + (k & 7) * 2);
}

// Shared-memory matrix descriptor (sm_100): start address >> 4 in bits
// [0,14), leading-dimension byte offset >> 4 in [16,30) (1: unused by the
// swizzled K-major form), stride-dimension byte offset >> 4 in [32,46) (1024:
// the next group of 8 rows), version 1 in [46,48), layout 2 (128-byte
// swizzle) in [61,64).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_byte_addr) {
  return (uint64_t)((smem_byte_addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulator (bits [4,6) = 1), bf16
// A and B ([7,10) = 1, [10,13) = 1), both K-major, N >> 3 in [17,23), M >> 4
// in [24,29).
constexpr uint32_t kIdescBf16 = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %3, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p;\n}"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(accumulate), "r"(kIdescBf16) : "memory");
}
// Arrives on `bar` once every tcgen05 operation issued so far by this thread completes.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// 32 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr) : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// One 64-column x 128-row box of the bf16 input (a K-atom of the operand),
// no multicast, completing on `bar`.
__device__ __forceinline__ void tma_load_box(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)) : "memory");
}

// True when the stored code of local element e occupies consecutive bits of
// one chunk word (then it is ORed in with one shift).
template <int BITS, int E>
__host__ __device__ constexpr bool code_contiguous(int e) {
  for (int k = 1; k < (BITS == 4 ? 4 : BITS); ++k)
    if (code_word<BITS, E>(e, k) != code_word<BITS, E>(e, 0) || code_bit<BITS, E>(e, k) != code_bit<BITS, E>(e, 0) + k)
      return false;
  return true;
}

// bf16 pair (lo element first) and the bf16 pair of what it leaves of (a, b).
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Small shared state, after the operands in the dynamic shared memory.
struct QtcState {
  uint64_t bar_x, bar_y, bar_p[2];
  uint32_t tmem_base;
  int fail;
  float sb[16], sc[16];     // boundaries (sb[0] unused) and centroids
  float part_x[4][128];     // per-chunk sums of squares of a row (||x||^2)
};

__device__ __forceinline__ void tmem_st1(uint32_t taddr, float v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(__float_as_uint(v)) : "memory");
}
__device__ __forceinline__ float tmem_ld4_sum(uint32_t taddr) {
  uint32_t a, b, c, d;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "r"(taddr) : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  return (__uint_as_float(a) + __uint_as_float(b)) + (__uint_as_float(c) + __uint_as_float(d));
}

// grid: min(tiles, SMs) persistent CTAs; block 512; dynamic smem (1024-byte
// aligned): Pi hi/lo, (S_rot hi/lo,) the X tile, (R hi, R lo,) QtcState.
// CTA c takes the 128-row tiles c, c + gridDim.x, ...  Tensor memory: Y in
// columns 0..127; with a sketch, P of tile k in 128 + 128 (k % 2) .. + 127 and
// the four per-chunk ||r||^2 of each row in 384 + 4 (k % 2) .. + 3.
// Iteration k: ||x|| from X(k); the X tile is then free and the copy of
// X(k + 1) starts; the thread quantizes its chunk of Y(k) and, once the
// sketch of tile k - 1 is done with R, writes its residual to R; after a CTA
// barrier one thread issues the sketch of tile k and another the rotation of
// tile k + 1, while every thread turns P(k - 1) into sign bits and stores the
// records of tile k - 1.  Every wait on a copy or an MMA is bounded; a CTA
// whose wait gives up reports TQ_DEV_ERR_TIMEOUT, waits (bounded) for what it
// has in flight and frees its tensor memory.
template <int BITS, int F>
__global__ void __launch_bounds__(kQtcThreads, 1)
    quantize_tc_kernel(const __grid_constant__ CUtensorMap tmx, QuantizeTcParams p) {
  constexpr int E = 32;
  constexpr int K = 1 << BITS;
  using CW = ChunkWords<BITS, E, F>;
  constexpr int W = CW::W;
  constexpr bool kQjl = F > 0;
  constexpr uint32_t kCols = kQjl ? 512 : 128;   // tensor-memory columns (a power of two >= 32)
  constexpr uint32_t kColP = 128, kColR = 384;
  extern __shared__ __align__(1024) uint8_t qsm_raw[];
  constexpr int kRes = kQjl ? 4 : 2;             // resident operands
  constexpr int kOps = kRes + (kQjl ? 3 : 1);    // + X, R hi, R lo
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ch = warp >> 2;                      // chunk: coordinates 32 ch .. 32 ch + 31
  const int r = 32 * (warp & 3) + lane;          // row of the tile (tensor-memory lane)
  const uint32_t base_s = smem_addr(qsm_raw);
  if (base_s & 1023u) {                          // the SW128 atoms need 1024-byte alignment
    if (tid == 0) report(p.cv.err, TQ_DEV_ERR_CONFIG);
    return;
  }
  QtcState& st = *reinterpret_cast<QtcState*>(qsm_raw + kOps * kOpBytes);
  const uint32_t pi_s = base_s, sr_s = base_s + 2 * kOpBytes, x_s = base_s + kRes * kOpBytes,
                 rh_s = x_s + kOpBytes, rl_s = x_s + 2 * kOpBytes;
  uint8_t* const rh_g = qsm_raw + (kRes + 1) * kOpBytes;
  uint8_t* const rl_g = qsm_raw + (kRes + 2) * kOpBytes;
  const int64_t n_my = p.n_tiles > blockIdx.x ? (p.n_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

  if (tid == 0) {
    mbar_init(&st.bar_x, 1);
    mbar_init(&st.bar_y, 1);
    mbar_init(&st.bar_p[0], 1);
    mbar_init(&st.bar_p[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmx)) : "memory");
    st.fail = 0;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_addr(&st.tmem_base)), "r"(kCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid < K) st.sc[tid] = p.cent32[tid];
  if (tid < K - 1) st.sb[tid + 1] = p.bound32[tid];
  if (tid == 0) st.sb[0] = 0.0f;
  // resident operands: Pi hi / lo (and S_rot hi / lo) in the swizzled layout
  for (int q = tid; q < kRes * 128 * 16; q += kQtcThreads) {
    const int op = q / 2048, rr = (q / 16) % 128, c = q % 16;
    const __nv_bfloat16* src = (op < 2 ? p.pi_bf + (size_t)op * 16384 : p.srot_bf + (size_t)(op - 2) * 16384) +
                               (size_t)rr * 128 + 8 * c;
    const uint32_t dst = base_s + op * kOpBytes + sw128_offset(rr, 8 * c);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
  }
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the copies, visible to the MMAs
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = st.tmem_base;
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;   // this warp's tensor-memory lanes
  const float* const sb = st.sb;
  const float* const sc = st.sc;

  // Thread kIssueY (warp 4) issues the copies and the rotation MMAs, thread
  // kIssueP (warp 8) the sketch MMAs; each counts, per barrier it issues
  // to, the phases it started and the completions it has seen (the n-th
  // completion of a barrier has parity n % 2), so that a failed CTA can wait
  // out what is in flight.  Every thread knows the parities of the waits in
  // the loop from k.  Descriptors of consecutive K-steps differ only in the
  // start-address field (address >> 4, 14 bits, never carried out of).
  constexpr int kIssueY = 128, kIssueP = 256;
  int x_iss = 0, x_done = 0, y_iss = 0, y_done = 0, p_iss[2] = {0, 0}, p_done[2] = {0, 0};
  const uint64_t d_pih = sw128_desc(pi_s), d_pil = sw128_desc(pi_s + kOpBytes), d_x = sw128_desc(x_s);
  const uint64_t d_srh = sw128_desc(sr_s), d_srl = sw128_desc(sr_s + kOpBytes);
  const uint64_t d_rh = sw128_desc(rh_s), d_rl = sw128_desc(rl_s);
  auto issue_x = [&](int64_t k) {                // TMA of tile k (two 64-column boxes)
    const int y = (int)((blockIdx.x + k * gridDim.x) * 128);
    mbar_arrive_tx(&st.bar_x, kOpBytes);
    tma_load_box(x_s, &tmx, 0, y, &st.bar_x);
    tma_load_box(x_s + kAtomBytes, &tmx, 64, y, &st.bar_x);
    ++x_iss;
  };
  auto issue_y = [&]() -> bool {                 // Y = X Pi^T once the X tile has landed
    if (!mbar_wait(&st.bar_x, (uint32_t)(x_done & 1))) return false;
    ++x_done;
    tc_fence_after();
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t ko = ((ks >> 2) * kAtomBytes + (ks & 3) * 32) >> 4;
      tc_mma(tmem, d_x + ko, d_pih + ko, ks > 0);
      tc_mma(tmem, d_x + ko, d_pil + ko, 1);
    }
    tc_commit(&st.bar_y);
    ++y_iss;
    return true;
  };
  if (tid == kIssueY && n_my > 0) {
    issue_x(0);
    if (!issue_y()) st.fail = 1;
  }
  __syncthreads();                               // st.fail

  // the tile whose signs and record are still to be done (sketch form)
  uint32_t rec_prev[W];
  int64_t hb_prev = -1;
  int slot_prev = 0;
  float nrm_prev = 0.0f;
  bool aborted = false;

  // P(j) into sign bits, then the record of tile j (and its norm slot)
  auto finish = [&](int64_t j) {
    if constexpr (kQjl) {
      float pv[32];
      tmem_ld32(tmem + lane_base + kColP + 128 * (uint32_t)(j & 1) + 32 * ch, pv);
      uint32_t qw = 0u;
#pragma unroll
      for (int e = 0; e < 32; ++e) qw |= (__float_as_uint(pv[e]) >> 31) << qjl_bit(e);
      rec_prev[CW::q0] = qw;
    }
    float rn = 0.0f;
    if (kQjl && ch == 0) rn = sqrtf(tmem_ld4_sum(tmem + lane_base + kColR + 4 * (uint32_t)(j & 1)));
    if (hb_prev >= 0) {
      uint8_t* recp = p.cv.pages + hb_prev + (int64_t)slot_prev * 16 * W + ch * 4 * W;
      if constexpr (W % 4 == 0) {
#pragma unroll
        for (int i = 0; i < W / 4; ++i)
          reinterpret_cast<uint4*>(recp)[i] =
              make_uint4(rec_prev[4 * i], rec_prev[4 * i + 1], rec_prev[4 * i + 2], rec_prev[4 * i + 3]);
      } else if constexpr (W % 2 == 0) {
#pragma unroll
        for (int i = 0; i < W / 2; ++i) reinterpret_cast<uint2*>(recp)[i] = make_uint2(rec_prev[2 * i], rec_prev[2 * i + 1]);
      } else {
#pragma unroll
        for (int i = 0; i < W; ++i) reinterpret_cast<uint32_t*>(recp)[i] = rec_prev[i];
      }
      if (ch == 0) {
        const __half nh = __float2half_rn(nrm_prev);
        if (__hisinf(nh)) report(p.cv.err, TQ_DEV_ERR_RANGE);
        __half* ns = reinterpret_cast<__half*>(p.cv.pages + hb_prev + (int64_t)p.cv.page_tokens * 16 * W +
                                               (int64_t)slot_prev * (kQjl ? 4 : 2));
        ns[0] = nh;
        if constexpr (kQjl) ns[1] = __float2half_rn(rn);
      }
    }
  };

  for (int64_t k = 0; k < n_my; ++k) {
    const int64_t row0 = (blockIdx.x + k * gridDim.x) * 128;
    // where this row's record goes (the block-table read overlaps the waits)
    const int64_t row = row0 + r;
    int64_t hb = -1;
    int slot = 0;
    if (row < p.rows) {
      const int64_t per_seq = (int64_t)p.n_kv_heads * p.n_new;
      const int64_t b = row / per_seq;
      const int h = (int)((row / p.n_new) % p.n_kv_heads);
      const int64_t pos = p.start_pos[b] + row % p.n_new;
      hb = head_block_offset(p.cv, b, h, pos);
      slot = (int)(pos % p.cv.page_tokens);
    }
    // Y(k) is complete (so its MMAs are done reading X(k))
    bool ok = st.fail == 0 && mbar_wait(&st.bar_y, (uint32_t)(k & 1));
    if (ok && tid == kIssueY) ++y_done;
    tc_fence_after();
    // this thread's 32 coordinates of Y(k); ||x|| = ||Pi x|| from the row of Y
    // (Pi is orthogonal; Y carries the input to fp32 rounding)
    float y[32];
    tmem_ld32(tmem + lane_base + 32 * ch, y);
    float n2 = 0.0f;
#pragma unroll
    for (int e = 0; e < 32; ++e) n2 = fmaf(y[e], y[e], n2);
    st.part_x[ch][r] = n2;
    tc_fence_before();
    // the four warps of this row group (warps w % 4 equal) exchange their
    // partial norms; a failed wait is agreed on at the CTA barrier below
    asm volatile("barrier.sync %0, 128;" ::"r"(1 + (warp & 3)) : "memory");
    tc_fence_after();
    if (ok && tid == kIssueY && k + 1 < n_my) issue_x(k + 1);   // X(k) was read by Y(k) (this thread saw it)
    const float nrm = sqrtf((st.part_x[0][r] + st.part_x[1][r]) + (st.part_x[2][r] + st.part_x[3][r]));
    const float inv = nrm > 0.0f ? 1.0f / nrm : 0.0f;

    // quantize this chunk of Y(k): index bits and residual
    uint32_t rec[W];
#pragma unroll
    for (int i = 0; i < W; ++i) rec[i] = 0u;
    float rr2 = 0.0f;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float u = y[e] * inv;
      int idx = 0;
#pragma unroll
      for (int step = K / 2; step >= 1; step >>= 1)
        if (u >= sb[idx + step]) idx += step;
      const uint32_t code = stored_code<BITS>(idx);
      if (code_contiguous<BITS, E>(e)) {
        rec[code_word<BITS, E>(e, 0)] |= code << code_bit<BITS, E>(e, 0);
      } else {
#pragma unroll
        for (int kb = 0; kb < (BITS == 4 ? 4 : BITS); ++kb)
          rec[code_word<BITS, E>(e, kb)] |= ((code >> kb) & 1u) << code_bit<BITS, E>(e, kb);
      }
      y[e] = u - sc[idx];                       // residual, rotated space
      rr2 = fmaf(y[e], y[e], rr2);
    }
    bool ok2 = true;
    if constexpr (kQjl) {
      tmem_st1(tmem + lane_base + kColR + 4 * (uint32_t)(k & 1) + ch, rr2);
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      // R is free once the sketch of tile k - 1 is done (its P is read below)
      if (k > 0) {
        ok2 = mbar_wait(&st.bar_p[(k - 1) & 1], (uint32_t)(((k - 1) >> 1) & 1));
        if (ok2 && tid == kIssueP) ++p_done[(k - 1) & 1];
      }
      // residual as bf16 hi / lo, 8 values per 16-byte chunk
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) split_bf16x2(y[8 * c + 2 * e], y[8 * c + 2 * e + 1], hw[e], lw[e]);
        const uint32_t off = sw128_offset(r, 32 * ch + 8 * c);
        *reinterpret_cast<uint4*>(rh_g + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(rl_g + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // R, visible to the MMAs
    }
    tc_fence_before();
    if (__syncthreads_or(!ok || !ok2)) {         // R complete; every read of Y(k) done
      aborted = true;
      break;
    }
    tc_fence_after();
    if constexpr (kQjl) {
      if (tid == kIssueP) {
        // P(k) = R S_rot^T: R_hi S_hi + R_hi S_lo + R_lo S_hi
        const uint32_t dcol = tmem + kColP + 128 * (uint32_t)(k & 1);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t ko = ((ks >> 2) * kAtomBytes + (ks & 3) * 32) >> 4;
          tc_mma(dcol, d_rh + ko, d_srh + ko, ks > 0);
          tc_mma(dcol, d_rh + ko, d_srl + ko, 1);
          tc_mma(dcol, d_rl + ko, d_srh + ko, 1);
        }
        tc_commit(&st.bar_p[k & 1]);
        ++p_iss[k & 1];
      }
    }
    // the next tile's rotation (Y(k) has been read)
    if (tid == kIssueY && k + 1 < n_my && !issue_y()) st.fail = 1;
    if constexpr (kQjl) {
      if (k > 0) finish(k - 1);                  // P(k - 1) completed before R was written
      hb_prev = hb;
      slot_prev = slot;
      nrm_prev = nrm;
#pragma unroll
      for (int i = 0; i < W; ++i) rec_prev[i] = rec[i];
    } else {
      hb_prev = hb;
      slot_prev = slot;
      nrm_prev = nrm;
#pragma unroll
      for (int i = 0; i < W; ++i) rec_prev[i] = rec[i];
      finish(k);
    }
  }
  if constexpr (kQjl) {
    // the last tile's signs and record
    if (!aborted && n_my > 0) {
      const int64_t j = n_my - 1;
      const bool ok = mbar_wait(&st.bar_p[j & 1], (uint32_t)((j >> 1) & 1));
      if (ok && tid == kIssueP) ++p_done[j & 1];
      tc_fence_before();
      if (__syncthreads_or(!ok)) aborted = true;
      else {
        tc_fence_after();
        finish(j);
      }
    }
  }

  if (__syncthreads_or(st.fail != 0 || aborted)) {
    // a wait gave up: report, then wait (bounded) for every copy and MMA this
    // CTA put in flight before its shared and tensor memory are released
    if (tid == kIssueY) {
      report(p.cv.err, TQ_DEV_ERR_TIMEOUT);
      while (x_done < x_iss && mbar_wait(&st.bar_x, (uint32_t)(x_done & 1))) ++x_done;
      while (y_done < y_iss && mbar_wait(&st.bar_y, (uint32_t)(y_done & 1))) ++y_done;
    }
    if (tid == kIssueP)
      for (int bb = 0; bb < 2; ++bb)
        while (p_done[bb] < p_iss[bb] && mbar_wait(&st.bar_p[bb], (uint32_t)(p_done[bb] & 1))) ++p_done[bb];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols) : "memory");
}

}  // namespace tqd

namespace tq {

// cuTensorMapEncodeTiled from the driver, through the runtime (no link
// against libcuda).
static PFN_cuTensorMapEncodeTiled_v12000 encode_tiled_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool looked = false;
  if (!looked) {
    looked = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

template <int BITS, int F>
static tq_status run_quantize_tc(const CUtensorMap& map, const tqd::QuantizeTcParams& p, int sms,
                                 cudaStream_t st) {
  constexpr int ops = F > 0 ? 7 : 3;
  const int smem = ops * tqd::kOpBytes + (int)sizeof(tqd::QtcState);
  static PerDeviceOnce attr;           // per template instance
  if (const int dev_ = current_device(); attr.need(dev_)) {
    cudaError_t e = cudaFuncSetAttribute(tqd::quantize_tc_kernel<BITS, F>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "quantize_tc: smem attribute");
    attr.mark(dev_);
  }
  const int64_t grid = p.n_tiles < sms ? p.n_tiles : sms;
  tqd::quantize_tc_kernel<BITS, F><<<(unsigned)grid, tqd::kQtcThreads, smem, st>>>(map, p);
  return cuda_fail(cudaGetLastError(), "quantize_tc launch");
}

// The tensor-core path serves head_dim 128 (d_pad 128, m <= 128), bf16 input
// rows that are 16-byte aligned, and batches of at least kMinRows vectors
// (smaller appends are latency-bound and go to the CUDA-core kernel, which
// writes identical records).
tq_status launch_quantize_tc(const tq_codebook* cb, const void* x, tq_dtype dt, int64_t batch,
                             int n_kv_heads, int64_t n_new, const int32_t* start_pos,
                             const CacheView& cv, cudaStream_t st, bool* handled) {
  constexpr int64_t kMinRows = 512;
  const Layout& L = cb->lay;
  *handled = false;
  const int64_t rows = batch * n_kv_heads * n_new;
  if (dt != TQ_BF16 || L.d != 128 || L.d_pad != 128 || !(L.m_pad == 0 || L.m_pad == 128) ||
      rows < kMinRows || rows > 0x7fffff00LL || (reinterpret_cast<uintptr_t>(x) & 15u) != 0)
    return TQ_OK;
  const PFN_cuTensorMapEncodeTiled_v12000 encode = encode_tiled_fn();
  if (!encode) return TQ_OK;
  const int sms = device_sm_count();
  // X as a 2-D bf16 tensor [rows][128]; a box is 64 columns (128 bytes) x
  // 128 rows, written with the 128-byte swizzle; rows past the end read as 0
  CUtensorMap map;
  const cuuint64_t dims[2] = {128, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {128 * sizeof(__nv_bfloat16)};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return fail(TQ_ECUDA, "quantize_tc: cuTensorMapEncodeTiled");
  tqd::QuantizeTcParams p;
  p.rows = rows;
  p.n_new = n_new;
  p.n_kv_heads = n_kv_heads;
  p.start_pos = start_pos;
  p.cv = cv;
  p.pi_bf = cb->pi_bf;
  p.srot_bf = cb->srot_bf;
  p.bound32 = cb->bound32;
  p.cent32 = cb->cent32;
  p.n_tiles = (rows + 127) / 128;
  tq_status s = TQ_OK;
  const bool q = L.m_pad == 128;
  switch (L.bits) {
    case 1: s = q ? run_quantize_tc<1, 32>(map, p, sms, st) : run_quantize_tc<1, 0>(map, p, sms, st); break;
    case 2: s = q ? run_quantize_tc<2, 32>(map, p, sms, st) : run_quantize_tc<2, 0>(map, p, sms, st); break;
    case 3: s = q ? run_quantize_tc<3, 32>(map, p, sms, st) : run_quantize_tc<3, 0>(map, p, sms, st); break;
    case 4: s = q ? run_quantize_tc<4, 32>(map, p, sms, st) : run_quantize_tc<4, 0>(map, p, sms, st); break;
    default: return TQ_OK;
  }
  *handled = true;
  return s;
}

}  // namespace tq
