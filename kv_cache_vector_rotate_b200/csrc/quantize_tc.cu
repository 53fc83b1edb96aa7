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
// is split as well, and P = R_hi S_hi + R_hi S_lo + R_lo S_hi.  One CTA per SM
// keeps Pi and S_rot resident (128 KB) and walks 128-vector tiles; every
// thread owns one vector in the epilogues: it reads its row of Y from tensor
// memory, quantizes, forms the residual (written back as the next MMA's
// operand), reads its row of P, and assembles its whole record in registers.
//
// Shared-memory operands use the K-major 128-byte-swizzle canonical layout:
// a 128 x 128 bf16 operand is two K-atoms of 128 rows x 128 bytes (16 KB,
// 1024-byte aligned); 16-byte chunk c of row r sits at chunk c ^ (r % 8).

#include "pack.cuh"
#include "stream.cuh"

namespace tqd {

constexpr int kQtcThreads = 128;                  // 4 warps: warp w owns rows 32w .. 32w + 31
constexpr int kOpBytes = 128 * 128 * 2;           // one 128 x 128 bf16 operand

struct QuantizeTcParams {
  const __nv_bfloat16* x;    // [rows][128]
  int64_t rows, n_new;       // rows = batch * n_kv_heads * n_new
  int n_kv_heads;
  const int32_t* start_pos;
  tq::CacheView cv;
  const __nv_bfloat16* pi_bf;    // [2][128][128]: hi, lo of Pi[j][k]
  const __nv_bfloat16* srot_bf;  // [2][128][128]: hi, lo of (S Pi^T)[i][j]
  const float* bound32;          // [2^b - 1]
  const float* cent32;           // [2^b] float(c16)
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

// grid: min(tiles, SMs) persistent CTAs; block 128; dynamic smem
// (3 + 4 * has_qjl) operands + 1 KB alignment slack.  CTA k takes the
// 128-row tiles k, k + gridDim.x, ...; thread 32 w + l owns row 32 w + l of
// the tile, which lives in tensor-memory lane 32 w + l (columns 0..127: Y,
// 128..255: P).  One elected thread issues the MMAs; every wait on their
// completion is bounded.
template <int BITS, int F>
__global__ void __launch_bounds__(kQtcThreads, 1) quantize_tc_kernel(QuantizeTcParams p) {
  constexpr int E = 32;
  constexpr int K = 1 << BITS;
  using CW = ChunkWords<BITS, E, F>;
  constexpr int W = CW::W;
  constexpr bool kQjl = F > 0;
  constexpr uint32_t kCols = kQjl ? 256 : 128;   // tensor-memory columns (a power of two >= 32)
  extern __shared__ uint8_t qsm_raw[];
  __shared__ uint64_t bar_mma;
  __shared__ uint32_t tmem_base_s;
  __shared__ float sb[16], sc[16];
  __shared__ int abort_all;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base_s = (smem_addr(qsm_raw) + 1023u) & ~1023u;    // SW128 atoms: 1024-byte aligned
  uint8_t* const base_g = qsm_raw + (base_s - smem_addr(qsm_raw));
  const uint32_t pi_s = base_s, xt_s = base_s + 2 * kOpBytes, sr_s = base_s + 3 * kOpBytes,
                 rt_s = base_s + 5 * kOpBytes;
  uint8_t* const rt_g = base_g + 5 * kOpBytes;
  uint8_t* const xt_g = base_g + 2 * kOpBytes;

  if (tid == 0) {
    mbar_init(&bar_mma, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    abort_all = 0;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_addr(&tmem_base_s)), "r"(kCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid < K) sc[tid] = p.cent32[tid];
  if (tid < K - 1) sb[tid + 1] = p.bound32[tid];
  if (tid == 0) sb[0] = 0.0f;
  // resident operands: Pi hi / lo (and S_rot hi / lo) in the swizzled layout
  {
    const int n_ops = kQjl ? 4 : 2;
    for (int q = tid; q < n_ops * 128 * 16; q += kQtcThreads) {
      const int op = q / 2048, r = (q / 16) % 128, c = q % 16;
      const __nv_bfloat16* src = (op < 2 ? p.pi_bf + (size_t)op * 16384 : p.srot_bf + (size_t)(op - 2) * 16384) +
                                 (size_t)r * 128 + 8 * c;
      const uint32_t dst = (op < 2 ? pi_s + op * kOpBytes : sr_s + (op - 2) * kOpBytes) + sw128_offset(r, 8 * c);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  const uint32_t lane_base = (uint32_t)(32 * warp) << 16;     // this warp's tensor-memory lanes
  uint32_t phase = 0;

  for (int64_t tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x) {
    const int64_t row0 = tile * 128;
    // X tile: 128 rows x 16 chunks of 16 bytes, zero past the last row
    for (int q = tid; q < 128 * 16; q += kQtcThreads) {
      const int r = q >> 4, c = q & 15;
      const bool ok = row0 + r < p.rows;
      const __nv_bfloat16* src = p.x + (ok ? (row0 + r) * 128 + 8 * c : 0);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                   ::"r"(xt_s + sw128_offset(r, 8 * c)), "l"(src), "r"(ok ? 16 : 0) : "memory");
    }
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the copies, visible to the MMAs
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // Y = X Pi^T (X Pi_hi + X Pi_lo), 8 K-steps of 16
    if (tid == 0) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
        const uint64_t ad = sw128_desc(xt_s + koff);
        tc_mma(tmem, ad, sw128_desc(pi_s + koff), ks > 0);
        tc_mma(tmem, ad, sw128_desc(pi_s + kOpBytes + koff), 1);
      }
      tc_commit(&bar_mma);
    }
    // this thread's row: ||x|| from the tile (while the MMAs run)
    const int r = tid;
    float n2 = 0.0f;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const uint4 v = *reinterpret_cast<const uint4*>(xt_g + sw128_offset(r, 8 * c));
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = __uint_as_float(w4[e] << 16), b2 = __uint_as_float(w4[e] & 0xFFFF0000u);
        n2 = fmaf(a, a, fmaf(b2, b2, n2));
      }
    }
    const float nrm = sqrtf(n2);
    const float inv = nrm > 0.0f ? 1.0f / nrm : 0.0f;
    bool ok = mbar_wait(&bar_mma, phase);
    phase ^= 1u;
    if (__syncthreads_or(!ok)) {
      if (tid == 0) abort_all = 1;
      break;
    }
    tc_fence_after();

    // quantize: indices, residual (as the next MMA's operand), record words
    uint32_t rec[4 * W];
#pragma unroll
    for (int i = 0; i < 4 * W; ++i) rec[i] = 0u;
    float rr2 = 0.0f;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      float y[32];
      tmem_ld32(tmem + lane_base + 32 * t, y);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float u = y[e] * inv;
        int idx = 0;
#pragma unroll
        for (int step = K / 2; step >= 1; step >>= 1)
          if (u >= sb[idx + step]) idx += step;
        const uint32_t code = stored_code<BITS>(idx);
#pragma unroll
        for (int k = 0; k < (BITS == 4 ? 4 : BITS); ++k)
          rec[t * W + code_word<BITS, E>(e, k)] |= ((code >> k) & 1u) << code_bit<BITS, E>(e, k);
        y[e] = u - sc[idx];                       // residual, rotated space
        rr2 = fmaf(y[e], y[e], rr2);
      }
      if constexpr (kQjl) {
        // residual as bf16 hi / lo, 8 values per 16-byte chunk
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float a0 = y[8 * c + 2 * e], a1 = y[8 * c + 2 * e + 1];
            const __nv_bfloat16 h0 = __float2bfloat16_rn(a0), h1 = __float2bfloat16_rn(a1);
            const __nv_bfloat16 l0 = __float2bfloat16_rn(a0 - __bfloat162float(h0));
            const __nv_bfloat16 l1 = __float2bfloat16_rn(a1 - __bfloat162float(h1));
            hw[e] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
            lw[e] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
          }
          const uint32_t off = sw128_offset(r, 32 * t + 8 * c);
          *reinterpret_cast<uint4*>(rt_g + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(rt_g + kOpBytes + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
      }
    }
    const float rn = sqrtf(rr2);

    if constexpr (kQjl) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the residual tile, visible to the MMAs
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      // P = R S_rot^T: R_hi S_hi + R_hi S_lo + R_lo S_hi
      if (tid == 0) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint64_t rh = sw128_desc(rt_s + koff), rl = sw128_desc(rt_s + kOpBytes + koff);
          tc_mma(tmem + 128, rh, sw128_desc(sr_s + koff), ks > 0);
          tc_mma(tmem + 128, rh, sw128_desc(sr_s + kOpBytes + koff), 1);
          tc_mma(tmem + 128, rl, sw128_desc(sr_s + koff), 1);
        }
        tc_commit(&bar_mma);
      }
      ok = mbar_wait(&bar_mma, phase);
      phase ^= 1u;
      if (__syncthreads_or(!ok)) {
        if (tid == 0) abort_all = 1;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        float pv[32];
        tmem_ld32(tmem + 128 + lane_base + 32 * t, pv);
        uint32_t qw = 0u;
#pragma unroll
        for (int e = 0; e < 32; ++e) qw |= (pv[e] < 0.0f ? 1u : 0u) << qjl_bit(e);
        rec[t * W + CW::q0] = qw;
      }
    }

    // store the record and the norm slot
    const int64_t row = row0 + r;
    if (row < p.rows) {
      const int64_t per_seq = (int64_t)p.n_kv_heads * p.n_new;
      const int64_t b = row / per_seq;
      const int h = (int)((row / p.n_new) % p.n_kv_heads);
      const int64_t pos = p.start_pos[b] + row % p.n_new;
      const int64_t hb = head_block_offset(p.cv, b, h, pos);
      if (hb >= 0) {
        const int slot = (int)(pos % p.cv.page_tokens);
        uint8_t* recp = p.cv.pages + hb + (int64_t)slot * 16 * W;
        if constexpr (W % 4 == 0) {
#pragma unroll
          for (int i = 0; i < W; ++i)
            reinterpret_cast<uint4*>(recp)[i] =
                make_uint4(rec[4 * i], rec[4 * i + 1], rec[4 * i + 2], rec[4 * i + 3]);
        } else {
#pragma unroll
          for (int i = 0; i < 4 * W; ++i) reinterpret_cast<uint32_t*>(recp)[i] = rec[i];
        }
        const __half nh = __float2half_rn(nrm);
        if (__hisinf(nh)) report(p.cv.err, TQ_DEV_ERR_RANGE);
        __half* ns = reinterpret_cast<__half*>(p.cv.pages + hb + (int64_t)p.cv.page_tokens * 16 * W +
                                               (int64_t)slot * (kQjl ? 4 : 2));
        ns[0] = nh;
        if constexpr (kQjl) ns[1] = __float2half_rn(rn);
      }
    }
    tc_fence_before();
    __syncthreads();                               // tensor memory and the tiles are reused
    tc_fence_after();
  }

  if (abort_all) {
    // a completion wait gave up: report, wait (bounded) for the MMAs in flight
    if (tid == 0) report(p.cv.err, TQ_DEV_ERR_TIMEOUT);
    mbar_wait(&bar_mma, phase);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols) : "memory");
}

}  // namespace tqd

namespace tq {

template <int BITS, int F>
static tq_status run_quantize_tc(const tqd::QuantizeTcParams& p, int sms, cudaStream_t st) {
  const int smem = (F > 0 ? 7 : 3) * tqd::kOpBytes + 1024;
  static bool attr = false;            // per template instance
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(tqd::quantize_tc_kernel<BITS, F>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "quantize_tc: smem attribute");
    attr = true;
  }
  const int64_t grid = p.n_tiles < sms ? p.n_tiles : sms;
  tqd::quantize_tc_kernel<BITS, F><<<(unsigned)grid, tqd::kQtcThreads, smem, st>>>(p);
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
      rows < kMinRows || (reinterpret_cast<uintptr_t>(x) & 15u) != 0)
    return TQ_OK;
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 148;
  }
  tqd::QuantizeTcParams p;
  p.x = reinterpret_cast<const __nv_bfloat16*>(x);
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
    case 1: s = q ? run_quantize_tc<1, 32>(p, sms, st) : run_quantize_tc<1, 0>(p, sms, st); break;
    case 2: s = q ? run_quantize_tc<2, 32>(p, sms, st) : run_quantize_tc<2, 0>(p, sms, st); break;
    case 3: s = q ? run_quantize_tc<3, 32>(p, sms, st) : run_quantize_tc<3, 0>(p, sms, st); break;
    case 4: s = q ? run_quantize_tc<4, 32>(p, sms, st) : run_quantize_tc<4, 0>(p, sms, st); break;
    default: return TQ_OK;
  }
  *handled = true;
  return s;
}

}  // namespace tq
