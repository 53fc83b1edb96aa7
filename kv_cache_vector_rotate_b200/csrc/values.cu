// Value path from packed records: v_hat = ||v|| Pi^T c[idx] (c: the reconstruction levels).
//
// "TurboQuant explained" (a2a-mcp.org), §Stage 1: the MSE stage alone codes
// the values; reconstruction is the centroid vector rotated back.
//  * mode A writes v_hat for every token;
//  * mode B forms o_h = sum_t w_{h,t} v_hat_t for the query heads of a KV head.
//    The sum is accumulated in the rotated space (acc_h = sum_t w_{h,t}
//    ||v_t|| c[idx_t]) and rotated back once per head (o_h = Pi^T acc_h).
//    Per KV group that is ACC^T = C^T (w ||v||)^T, a contraction over the
//    tokens, run on the tensor cores: each warp streams 32-token units of
//    records into a shared-memory ring with bulk copies, each lane decodes
//    one token's coordinates into fp16 level values of a [token][coordinate]
//    tile, ldmatrix.trans turns the tile into MMA A fragments (coordinates x
//    tokens), and the weights times the norms, split into fp16 hi + lo, are
//    the B columns (4 query heads x 2).  Partial sums of context chunks go to
//    the workspace; a second kernel adds them and applies Pi^T.

#include "pack.cuh"
#include "stream.cuh"
#include "value_tile.cuh"

namespace tqd {

struct ValuesParams {
  tq::CacheView cv;
  const int32_t* ctx_len;
  int n_kv_heads, n_q_heads, G;
  int d;
  const float* pi32;        // [d_pad][d]
  const float* cent32;      // [2^b]
  const float* w;           // mode B weights
  int64_t w_stride;
  void* out;
  tq_dtype odt;
  int64_t out_stride;
  int max_ctx;              // ctx_len values are clamped to [0, max_ctx]
};

// Level index of local element l of a chunk (layout version 3).
template <int BITS, int E>
__device__ __forceinline__ int unpack_index(const uint32_t* w, int l) {
  uint32_t code = 0u;
  if (BITS == 3 && l / 32 < E / 32 && l % 32 >= 24) {
#pragma unroll
    for (int k = 0; k < 3; ++k) code |= ((w[code_word<BITS, E>(l, k)] >> code_bit<BITS, E>(l, k)) & 1u) << k;
  } else {
    code = (w[code_word<BITS, E>(l, 0)] >> code_bit<BITS, E>(l, 0)) & ((1u << BITS) - 1u);
  }
  return level_index<BITS>(code);
}

// Stages 16 tokens: cs[tok][j] = ||v|| c[idx_j] (0 past the context or for
// an unusable page).  128 threads: 8 threads per token, each decoding every
// 8th coordinate.
template <int BITS, int E>
__device__ __forceinline__ void stage_tokens(const ValuesParams& p, int b, int h, int base, int ctx,
                                             float (*cs)[4 * E + 1], const float* sc) {
  constexpr int W = ChunkWords<BITS, E, 0>::W;
  constexpr int CB = 16 * W;
  const int tok = threadIdx.x >> 3, sub = threadIdx.x & 7;
  const int pos = base + tok;
  bool ok = pos < ctx;
  const uint8_t* hb = nullptr;
  if (ok) {
    const int64_t page = p.cv.block_table[(int64_t)b * p.cv.max_pages + pos / p.cv.page_tokens];
    if (page < 0 || page >= p.cv.n_pages) {
      if (sub == 0) report(p.cv.err, TQ_DEV_ERR_PAGE);
      ok = false;
    } else {
      hb = p.cv.pages + page * p.cv.page_bytes + (int64_t)h * p.cv.head_block_bytes;
    }
  }
  const int slot = pos % p.cv.page_tokens;
  float nrm = 0.0f;
  if (ok) nrm = __half2float(*reinterpret_cast<const __half*>(hb + (int64_t)p.cv.page_tokens * CB + slot * 2));
  for (int j = sub; j < 4 * E; j += 8) {
    float v = 0.0f;
    if (ok && j < p.d) {
      const uint32_t* cw = reinterpret_cast<const uint32_t*>(hb + (int64_t)slot * CB) + (j / E) * W;
      v = nrm * sc[unpack_index<BITS, E>(cw, j % E)];
    }
    cs[tok][j] = v;
  }
}

// Mode A.  grid: (ceil(max_ctx / 16), batch * n_kv_heads); block 128.
template <int BITS, int E>
__global__ void __launch_bounds__(128) dequant_kernel(ValuesParams p) {
  constexpr int DP = 4 * E;
  __shared__ float cs[16][DP + 1];
  __shared__ float sc[16];
  const int gi = blockIdx.y, b = gi / p.n_kv_heads, h = gi % p.n_kv_heads;
  const int ctx = min(p.ctx_len[b], p.max_ctx);
  const int base = blockIdx.x * 16;
  if (base >= ctx) return;
  if (threadIdx.x < (1 << BITS)) sc[threadIdx.x] = p.cent32[threadIdx.x];
  __syncthreads();
  stage_tokens<BITS, E>(p, b, h, base, ctx, cs, sc);
  __syncthreads();
  const int d = p.d;
  for (int k = threadIdx.x; k < d; k += 128) {
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
    for (int j = 0; j < d; ++j) {
      const float pk = __ldg(p.pi32 + (size_t)j * d + k);   // (Pi^T)_{k j}
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = fmaf(pk, cs[i][j], acc[i]);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int pos = base + i;
      if (pos >= ctx) break;
      const int64_t o = (((int64_t)gi) * p.out_stride + pos) * d + k;
      if (p.odt == TQ_F32) reinterpret_cast<float*>(p.out)[o] = acc[i];
      else if (p.odt == TQ_BF16) reinterpret_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(acc[i]);
      else reinterpret_cast<__half*>(p.out)[o] = __float2half_rn(acc[i]);
    }
  }
}

// ---- mode B on the tensor cores ----------------------------------------------------

// Warps per CTA of the accumulate kernel: 16 for d <= 128 (one CTA per SM,
// so a line has few partials for the finish to sum), 4 above (the tiles of
// 16 warps would not fit in shared memory; 2-3 CTAs per SM).
template <int E>
__host__ __device__ constexpr int val_warps() { return E <= 32 ? 16 : 4; }
constexpr int kValCtaPages = 64;   // block-table entries staged per CTA
constexpr int kValStages = 2;      // ring stages per warp (a power of two: slot i & (S - 1), phase i / S)
static_assert((kValStages & (kValStages - 1)) == 0, "the ring indexes its slots with i & (S - 1)");

struct ValuesTcParams {
  tq::CacheView cv;
  int page_shift;                  // log2(page_tokens)
  const int32_t* ctx_len;
  int n_kv_heads, n_q_heads, G, qtiles;
  int n_chunks;                    // CTAs per (group, query tile) along the tokens
  int units;                       // 32-token units of max_ctx
  int max_ctx;                     // ctx_len values are clamped to [0, max_ctx]
  int d;
  const float* w;                  // [batch][n_q_heads][w_stride]
  int64_t w_stride;
  float* partial;                  // [n_chunks][groups * qtiles][4][4E]
  const float* pi32;               // [d_pad][d]
  float* out;                      // [batch][n_q_heads][d]
  uint32_t tlo0, tlo1, thi0, thi1; // low / high bytes of the fp16 levels (b <= 3: levels 0..7; b = 4: magnitudes)
};

template <int W, int E>
struct ValShape {
  static constexpr int kRec = 16 * W;                  // bytes per record
  static constexpr int kStage = 32 * kRec + 64;        // 32 records + 32 fp16 norms
  static constexpr int kTile = 32 * 4 * E * 2;         // fp16 [32 tokens][4E coordinates]
  static constexpr int kWarpBytes = kValStages * kStage + kTile + 8 * kBRow * 2;   // + the B rows
};

// 2^s as a float for s in [-126, 127] (built from the exponent field).
__device__ __forceinline__ float pow2i(int s) { return __int_as_float((s + 127) << 23); }

// Mode B, pass 1.  grid: (n_chunks, batch * n_kv_heads, query tiles of 4);
// block val_warps * 32; dynamic smem val_warps * ValShape::kWarpBytes.
// CTA x of a (group, query tile) owns the 32-token units [x U / n_chunks,
// (x + 1) U / n_chunks) (U = ceil(max_ctx / 32)); warp w takes its units w,
// w + val_warps, ...; lane 0 bulk-copies a unit (32 records, 32 norms) into ring
// stage i % 2 (mbarrier, bounded wait).  Lane l decodes token l into row l
// of the warp's fp16 tile (16-byte pieces XOR-swizzled by row: conflict-free
// stores and ldmatrix reads) and forms w ||v|| for the 4 query slots; then
// per 16 tokens and 16 coordinates one ldmatrix.x4.trans and one
// m16n8k16 MMA.  Column pair (2q, 2q + 1) of the accumulators is the hi / lo
// part of query slot q.  Tokens past the context, on a bad page, or query
// slots past G get weight 0, and such tokens norm 0 (the tile then holds
// finite table values, and nothing read from those slots reaches the sums).  The
// warps' sums meet in shared memory; the CTA writes one partial.
template <int BITS, int E>
__global__ void __launch_bounds__(val_warps<E>() * 32) values_acc_kernel(ValuesTcParams p) {
  constexpr int kValWarps = val_warps<E>();
  constexpr int W = ChunkWords<BITS, E, 0>::W;
  using VS = ValShape<W, E>;
  constexpr int REC = VS::kRec, STAGE = VS::kStage, S = kValStages;
  constexpr int DP = 4 * E;        // padded coordinates
  constexpr int MT = DP / 16;      // 16-coordinate tiles
  extern __shared__ __align__(16) uint8_t vsm[];
  __shared__ int64_t page_base[kValCtaPages];
  __shared__ uint64_t bars[kValWarps][S];

  // a programmatic dependent of the previous kernel (nothing is read before it
  // finishes); the finish kernel may start now: it prefetches Pi and then
  // waits for this grid
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
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
  const int n_pgx = k0 < kend ? ((kend - 1) >> ps) - first_page + 1 : 0;   // <= kValCtaPages
  const int ctx = min(p.ctx_len[b], p.max_ctx);
  const int jt = threadIdx.x;
  static_assert(kValCtaPages <= kValWarps * 32, "one block-table entry per thread");
  const int64_t pg = jt < n_pgx ? p.cv.block_table[(int64_t)b * p.cv.max_pages + first_page + jt] : 0;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < S; ++s) mbar_init(&bars[warp][s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  const int k1 = min(kend, ctx);
  const bool has_keys = k0 < k1;
  bool bad = false;
  if (jt < n_pgx) {
    const bool valid = pg >= 0 && pg < p.cv.n_pages;
    page_base[jt] = valid ? pg * p.cv.page_bytes + (int64_t)h * p.cv.head_block_bytes : -1;
    if (!valid && has_keys && jt <= ((k1 - 1) >> ps) - first_page) {
      bad = true;
      report(p.cv.err, TQ_DEV_ERR_PAGE);
    }
  }
  const bool fast = !__syncthreads_or(bad) && P >= 32;

  const int n_units = has_keys ? (k1 - k0 + 31) >> 5 : 0;
  const int n_my = warp < n_units ? (n_units - warp + kValWarps - 1) / kValWarps : 0;
  uint8_t* wbase = vsm + warp * VS::kWarpBytes;
  const uint32_t ring_s = smem_addr(wbase);
  uint8_t* tile = wbase + S * STAGE;
  unsigned short* wh = reinterpret_cast<unsigned short*>(tile + VS::kTile);   // [8][kBRow] fp16 B rows
  const int64_t norm_off = (int64_t)P * REC;
  const uint64_t pol = evict_first_policy();

  auto issue = [&](int i) {
    if (lane != 0) return;
    uint64_t* bar = &bars[warp][i & (S - 1)];
    const uint32_t dst = ring_s + (i & (S - 1)) * STAGE;
    const int ubase = k0 + 32 * (warp + kValWarps * i);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (fast) {
      const int slot = ubase & (P - 1);
      const uint8_t* hb = p.cv.pages + page_base[(ubase >> ps) - first_page];
      mbar_arrive_tx(bar, 32 * REC + 64);
      bulk_copy(dst, hb + (int64_t)slot * REC, 32 * REC, bar, pol);
      bulk_copy(dst + 32 * REC, hb + norm_off + slot * 2, 64, bar, pol);
      return;
    }
    uint32_t bytes = 0;
    int64_t off[2] = {-1, -1};
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int base = ubase + 16 * hf;
      if (base < k1) off[hf] = page_base[(base >> ps) - first_page];
      if (off[hf] >= 0) bytes += 16 * REC + 32;
    }
    mbar_arrive_tx(bar, bytes);
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      if (off[hf] < 0) continue;
      const int slot = (ubase + 16 * hf) & (P - 1);
      const uint8_t* hb = p.cv.pages + off[hf];
      bulk_copy(dst + hf * 16 * REC, hb + (int64_t)slot * REC, 16 * REC, bar, pol);
      bulk_copy(dst + 32 * REC + 32 * hf, hb + norm_off + slot * 2, 32, bar, pol);
    }
  };
#pragma unroll
  for (int s = 0; s < S; ++s)
    if (s < n_my) issue(s);

  const int64_t wrow0 = ((int64_t)b * p.n_q_heads + h * p.G + qt * 4) * p.w_stride;
  const int nq = min(4, p.G - qt * 4);
  float acc[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.0f;
  // per query slot, the power of two 2^sc that the B values carry: set by
  // the largest |w ||v||| seen so far (below 2^14), so that fp16 hi + lo keep
  // their 22 bits whatever the scale of the weights and norms; when a unit
  // needs a smaller one the accumulators are scaled down exactly
  int sc[4] = {0, 0, 0, 0};
  bool has[4] = {false, false, false, false};
  bool timed_out = false;
  int issued = min(S, n_my);
  // the weights of unit i (this lane's token, 4 query slots), loaded one unit ahead
  auto load_w = [&](int i, float (&wv)[4]) {
    const int pos = k0 + 32 * (warp + kValWarps * i) + lane;
    bool tok_ok = i < n_my && pos < k1;
    if (tok_ok && !fast) tok_ok = page_base[(pos >> ps) - first_page] >= 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) wv[q] = (tok_ok && q < nq) ? __ldg(p.w + wrow0 + q * p.w_stride + pos) : 0.0f;
  };
  float wnext[4];
  load_w(0, wnext);
  for (int i = 0; i < n_my; ++i) {
    float wv[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) wv[q] = wnext[q];
    load_w(i + 1, wnext);
    if (!mbar_wait(&bars[warp][i & (S - 1)], (uint32_t)(i / S) & 1u)) {
      timed_out = true;
      break;
    }
    // decode token `lane` into row `lane` of the tile
    const uint8_t* stg = wbase + (i & (S - 1)) * STAGE;
    uint32_t rec[4 * W];
#pragma unroll
    for (int x = 0; x < W; ++x) {
      const uint4 v = reinterpret_cast<const uint4*>(stg + lane * REC)[x];
      rec[4 * x] = v.x; rec[4 * x + 1] = v.y; rec[4 * x + 2] = v.z; rec[4 * x + 3] = v.w;
    }
    // a slot past the context or on a bad page may hold any bytes (a NaN
    // norm times a zero weight would still poison the sums): its norm is 0
    const int pos = k0 + 32 * (warp + kValWarps * i) + lane;
    bool tok_ok = pos < k1;
    if (tok_ok && !fast) tok_ok = page_base[(pos >> ps) - first_page] >= 0;
    const float nrm = tok_ok ? __half2float(reinterpret_cast<const __half*>(stg + 32 * REC)[lane]) : 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int kk = 0; kk < E / 8; ++kk) {
        const int piece = c * (E / 8) + kk;     // coordinates 8 piece .. 8 piece + 7
        reinterpret_cast<uint4*>(tile + lane * (DP * 2))[piece ^ (lane & 7)] =
            decode8<BITS, E>(rec + c * W, kk, p);
      }
    float wq[4] = {wv[0] * nrm, wv[1] * nrm, wv[2] * nrm, wv[3] * nrm};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      // non-negative floats order as their bit patterns; the exponent field
      // gives 2^(e - 1) <= max < 2^e
      const uint32_t mx = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(wq[q])));
      if (mx != 0u) {                               // warp-uniform
        const int e = (int)((mx >> 23) & 0xFFu) - 126;
        const int s_new = min(120, 14 - e);
        if (!has[q] || s_new < sc[q]) {
          if (has[q] && t == q) {
            const float f = pow2i(max(-126, s_new - sc[q]));
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              acc[mt][0] *= f; acc[mt][1] *= f; acc[mt][2] *= f; acc[mt][3] *= f;
            }
          }
          sc[q] = s_new;
          has[q] = true;
        }
      }
      wq[q] *= pow2i(sc[q]);                        // 0 stays 0 while nothing was seen
    }
    // token `lane`'s B values: w ||v|| 2^sc split into fp16 hi + lo, once per
    // token and query slot
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __half hi = __float2half_rn(wq[q]);
      const __half lo = __float2half_rn(wq[q] - __half2float(hi));
      wh[(2 * q) * kBRow + lane] = __half_as_ushort(hi);
      wh[(2 * q + 1) * kBRow + lane] = __half_as_ushort(lo);
    }
    __syncwarp();                                 // the tile, the B rows, and every read of the stage
    if (i + S < n_my) {
      issue(i + S);
      issued = i + S + 1;
    }
    // 2 k-steps of 16 tokens: B column g = row g (slice g & 1 of query slot
    // g >> 1), tokens tk and tk + 1 in one word
    const uint32_t* whw = reinterpret_cast<const uint32_t*>(wh);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      uint32_t bw[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int tk = 16 * j + 2 * t + 8 * r;
        bw[r] = whw[(g * kBRow + tk) / 2];
      }
      const int mi = lane >> 3, rr = lane & 7;
      const int row = 16 * j + 8 * (mi >> 1) + rr;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int piece = 2 * mt + (mi & 1);
        uint32_t a0, a1, a2, a3;
        ldsm_x4_trans(smem_addr(tile + row * (DP * 2) + 16 * (piece ^ rr)), a0, a1, a2, a3);
        mma_f16(acc[mt], a0, a1, a2, a3, make_uint2(bw[0], bw[1]));
      }
    }
    __syncwarp();                                 // the tile is rewritten by the next unit
  }
  if (timed_out) {
    if (lane == 0) report(p.cv.err, TQ_DEV_ERR_TIMEOUT);
    for (int u = max(0, issued - S); u < issued; ++u) mbar_wait(&bars[warp][u & (S - 1)], (uint32_t)(u / S) & 1u);
  }
  // the warps' sums meet in shared memory (the rings are free now)
  __syncthreads();
  // [kValWarps][4][RSV]: rows padded by 8 floats, so that the 4 query slots'
  // lanes (t) of one store fall in different banks
  constexpr int RSV = DP + 8;
  static_assert(kValWarps * 4 * RSV * 4 <= kValWarps * VS::kWarpBytes, "the merge rows fit the rings");
  float* red = reinterpret_cast<float*>(vsm);
  float unsc = 1.0f;                               // undo query slot t's scale
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (q == t && has[q]) unsc = pow2i(-sc[q]);
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    red[(warp * 4 + t) * RSV + 16 * mt + g] = (acc[mt][0] + acc[mt][1]) * unsc;
    red[(warp * 4 + t) * RSV + 16 * mt + g + 8] = (acc[mt][2] + acc[mt][3]) * unsc;
  }
  __syncthreads();
  const int gq = gi * p.qtiles + qt;
  float* dst = p.partial + ((int64_t)blockIdx.x * gridDim.y * gridDim.z + gq) * 4 * DP;
  for (int i = threadIdx.x; i < 4 * DP; i += kValWarps * 32) {
    float s = 0.0f;
#pragma unroll
    for (int w2 = 0; w2 < kValWarps; ++w2) s += red[(w2 * 4 + i / DP) * RSV + i % DP];
    dst[i] = s;
  }
}

// Mode B, pass 2: o = Pi^T sum_chunks partial, one CTA per (query tile,
// query slot < G); CL x DP threads (CL = 1024 / DP chunk lanes).  Thread
// (cl, k) loads its entries Pi[j][k] (j = cl, cl + CL, ...) before it waits
// for pass 1 (programmatic dependent launch; pass 1 lets it start early), then
// sums its chunks of the partials with independent accumulators.
template <int E>
__global__ void __launch_bounds__(1024) values_finish_kernel(ValuesTcParams p) {
  constexpr int DP = 4 * E;
  constexpr int CL = 1024 / DP;    // chunk lanes
  constexpr int JN = (DP + CL - 1) / CL;   // rows of Pi per thread
  __shared__ float red[CL][DP];
  __shared__ float a[DP];
  const int gq = blockIdx.x / 4, q = blockIdx.x % 4;
  const int gi = gq / p.qtiles, qt = gq % p.qtiles;
  const int hql = qt * 4 + q;                     // query within the group
  const int b = gi / p.n_kv_heads, h = gi % p.n_kv_heads;
  const int k = threadIdx.x % DP, cl = threadIdx.x / DP;
  const int d = p.d;
  constexpr bool kPre = JN <= 16;              // Pi entries held in registers across the wait
  float pij[kPre ? JN : 1];
  if constexpr (kPre) {
#pragma unroll
    for (int n = 0; n < JN; ++n) {
      const int j = cl + CL * n;
      pij[n] = (k < d && j < d) ? __ldg(p.pi32 + (size_t)j * d + k) : 0.0f;
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");   // the next kernel may be scheduled (it waits for this one)
  if (hql >= p.G) return;
  const int nq = gridDim.x;                       // groups * qtiles * 4
  const float* src = p.partial + ((int64_t)gq * 4 + q) * DP + k;
  const int64_t cs = (int64_t)nq * DP;            // stride between chunks
  float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
  int c = cl;
  for (; c + 3 * CL < p.n_chunks; c += 4 * CL) {
    s0 += src[(int64_t)c * cs];
    s1 += src[(int64_t)(c + CL) * cs];
    s2 += src[(int64_t)(c + 2 * CL) * cs];
    s3 += src[(int64_t)(c + 3 * CL) * cs];
  }
  for (; c < p.n_chunks; c += CL) s0 += src[(int64_t)c * cs];
  red[cl][k] = (s0 + s1) + (s2 + s3);
  __syncthreads();
  if (cl == 0) {
    float t2 = 0.0f;
#pragma unroll
    for (int x = 0; x < CL; ++x) t2 += red[x][k];
    a[k] = t2;
  }
  __syncthreads();
  // o_k = sum_j Pi[j][k] a_j over this lane's rows j
  float o = 0.0f;
  if constexpr (kPre) {
#pragma unroll
    for (int n = 0; n < JN; ++n) {
      const int j = cl + CL * n;
      if (j < DP) o = fmaf(pij[n], a[j], o);
    }
  } else {
    for (int j = cl; j < d; j += CL)
      if (k < d) o = fmaf(__ldg(p.pi32 + (size_t)j * d + k), a[j], o);
  }
  __syncthreads();
  red[cl][k] = o;
  __syncthreads();
  if (cl == 0 && k < d) {
    float t2 = 0.0f;
#pragma unroll
    for (int x = 0; x < CL; ++x) t2 += red[x][k];
    p.out[((int64_t)b * p.n_q_heads + h * p.G + hql) * d + k] = t2;
  }
}

}  // namespace tqd

namespace tq {

// Mode B chunking: every CTA slot of the GPU (SMs x 4) gets one CTA, each
// an equal share (to one 32-token unit) of a sequence; more CTAs when a share
// would need more than kValCtaPages - 2 block-table entries.
// CTAs of the accumulate kernel per (group, query tile): one wave of the
// CTAs that fit per SM (ctas_per_sm, at most 4), more when a CTA's share
// would not fit its staged block-table entries.
static int64_t values_chunks(int64_t units_gq, int64_t max_ctx, int page_tokens, int ctas_per_sm) {
  const int64_t units = (max_ctx + 31) / 32;
  int64_t n = std::max<int64_t>(1, (int64_t)device_sm_count() * ctas_per_sm / std::max<int64_t>(1, units_gq));
  const int64_t max_units_cta = (int64_t)(tqd::kValCtaPages - 2) * page_tokens / 32;
  n = std::max<int64_t>(n, (units + max_units_cta - 1) / max_units_cta);
  return std::min<int64_t>(n, units);
}

// The workspace is sized for the smallest page (16 tokens), so it covers
// every cache of these sizes.
size_t values_workspace(const tq_codebook* cb, int64_t batch, int n_kv_heads, int n_q_heads,
                        int64_t max_ctx) {
  if (n_kv_heads <= 0 || n_q_heads <= 0 || max_ctx <= 0) return 0;
  const int G = n_q_heads / n_kv_heads;
  const int64_t gq = batch * n_kv_heads * ((G + 3) / 4);
  const int64_t chunks = values_chunks(gq, max_ctx, 16, 4);   // 4: the most CTAs per SM the grid assumes
  return (size_t)chunks * gq * 4 * cb->lay.d_pad * sizeof(float);
}

// CTAs of the accumulate kernel that fit per SM (registers, shared memory), at
// most 4; per device, per instance.  Sets the kernel's shared-memory limit.
template <int BITS, int E>
static int values_occupancy_t() {
  constexpr int W = tqd::ChunkWords<BITS, E, 0>::W;
  constexpr int NW = tqd::val_warps<E>();
  const int smem = NW * tqd::ValShape<W, E>::kWarpBytes;
  static int cache[64] = {};
  const int dev = current_device();
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int occ = 0;
  if (cudaFuncSetAttribute(tqd::values_acc_kernel<BITS, E>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, tqd::values_acc_kernel<BITS, E>, NW * 32,
                                                    smem) != cudaSuccess) {
    (void)cudaGetLastError();
    occ = 1;
  }
  occ = std::max(1, std::min(occ, 4));
  if (dev >= 0 && dev < 64) cache[dev] = occ;
  return occ;
}

template <int BITS>
static int values_occupancy_b(int E) {
  switch (E) {
    case 16: return values_occupancy_t<BITS, 16>();
    case 32: return values_occupancy_t<BITS, 32>();
    case 48: return values_occupancy_t<BITS, 48>();
    default: return values_occupancy_t<BITS, 64>();
  }
}

static int values_occupancy(const Layout& L) {
  switch (L.bits) {
    case 1: return values_occupancy_b<1>(L.E);
    case 2: return values_occupancy_b<2>(L.E);
    case 3: return values_occupancy_b<3>(L.E);
    default: return values_occupancy_b<4>(L.E);
  }
}

template <int BITS, int E>
static tq_status run_values(tqd::ValuesParams p, const tqd::ValuesTcParams& tp, int64_t batch,
                            int64_t max_ctx, bool mode_b, cudaStream_t st) {
  const int64_t groups = batch * p.n_kv_heads;
  if (!mode_b) {
    dim3 grid((unsigned)((max_ctx + 15) / 16), (unsigned)groups);
    tqd::dequant_kernel<BITS, E><<<grid, 128, 0, st>>>(p);
    return TQ_OK;
  }
  constexpr int W = tqd::ChunkWords<BITS, E, 0>::W;
  constexpr int NW = tqd::val_warps<E>();
  const int smem = NW * tqd::ValShape<W, E>::kWarpBytes;
  static PerDeviceOnce attr;           // per template instance
  if (const int dev_ = current_device(); attr.need(dev_)) {
    cudaError_t e = cudaFuncSetAttribute(tqd::values_acc_kernel<BITS, E>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "values: smem attribute");
    attr.mark(dev_);
  }
  dim3 grid((unsigned)tp.n_chunks, (unsigned)groups, (unsigned)tp.qtiles);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = dim3(NW * 32);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  cudaError_t ea = cudaLaunchKernelEx(&cfg, tqd::values_acc_kernel<BITS, E>, tp);
  if (ea != cudaSuccess) return cuda_fail(ea, "values: accumulate launch");
  cfg = {};
  cfg.gridDim = dim3((unsigned)(groups * tp.qtiles * 4));
  cfg.blockDim = dim3((1024 / (4 * E)) * (4 * E));   // whole chunk lanes of 4E coordinates
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, tqd::values_finish_kernel<E>, tp);
  if (e != cudaSuccess) return cuda_fail(e, "values: finish launch");
  return TQ_OK;
}

template <int BITS>
static int dispatch_values(const Layout& L, const tqd::ValuesParams& p, const tqd::ValuesTcParams& tp,
                           int64_t batch, int64_t max_ctx, bool mode_b, cudaStream_t st, tq_status* s) {
  switch (L.E) {
    case 16: *s = run_values<BITS, 16>(p, tp, batch, max_ctx, mode_b, st); return 1;
    case 32: *s = run_values<BITS, 32>(p, tp, batch, max_ctx, mode_b, st); return 1;
    case 48: *s = run_values<BITS, 48>(p, tp, batch, max_ctx, mode_b, st); return 1;
    case 64: *s = run_values<BITS, 64>(p, tp, batch, max_ctx, mode_b, st); return 1;
  }
  return 0;
}

tq_status launch_values(const tq_codebook* cb, const CacheView& cv, const float* w,
                        int64_t w_stride, int64_t batch, int n_q_heads, const int32_t* ctx_len,
                        int64_t max_ctx, void* out, tq_dtype odt, int64_t out_stride, void* ws,
                        size_t ws_bytes, cudaStream_t st) {
  const Layout& L = cb->lay;
  if (L.m != 0) return fail(TQ_EUNSUPPORTED, "tq_dequant_values: values codebooks have m = 0");
  const bool mode_b = w != nullptr;
  if (max_ctx == 0 || batch == 0) return TQ_OK;
  tqd::ValuesParams p;
  p.cv = cv;
  p.ctx_len = ctx_len;
  p.n_kv_heads = cv.n_kv_heads;
  p.n_q_heads = n_q_heads;
  p.G = mode_b ? n_q_heads / cv.n_kv_heads : 1;
  p.d = L.d;
  p.pi32 = cb->pi32;
  p.cent32 = cb->cent32;
  p.w = w;
  p.w_stride = w_stride;
  p.out = out;
  p.odt = odt;
  p.out_stride = out_stride;
  p.max_ctx = (int)max_ctx;
  tqd::ValuesTcParams tp;
  tp.cv = cv;
  int ps = 0;
  while ((1 << ps) < cv.page_tokens) ++ps;
  tp.page_shift = ps;
  tp.ctx_len = ctx_len;
  tp.n_kv_heads = cv.n_kv_heads;
  tp.n_q_heads = n_q_heads;
  tp.G = n_q_heads / cv.n_kv_heads;
  tp.qtiles = (tp.G + 3) / 4;
  const int64_t gq = batch * cv.n_kv_heads * tp.qtiles;
  if (mode_b && (batch * cv.n_kv_heads > 65535 || tp.qtiles > 65535 || gq * 4 > 0x7fffffffLL))
    return fail(TQ_EINVAL, "tq_dequant_values: batch * n_kv_heads too large");
  tp.n_chunks = (int)values_chunks(gq, max_ctx, cv.page_tokens, mode_b ? values_occupancy(L) : 4);
  tp.units = (int)((max_ctx + 31) / 32);
  tp.max_ctx = (int)max_ctx;
  tp.d = L.d;
  tp.w = w;
  tp.w_stride = w_stride;
  tp.partial = reinterpret_cast<float*>(ws);
  tp.pi32 = cb->pi32;
  tp.out = reinterpret_cast<float*>(out);
  tp.tlo0 = tp.tlo1 = tp.thi0 = tp.thi1 = 0u;
  {
    const uint16_t* T = L.bits == 4 ? cb->mag16 : cb->cent16;   // 8 entries
    for (int i = 0; i < 4; ++i) {
      tp.tlo0 |= (uint32_t)(T[i] & 0xFF) << (8 * i);
      tp.tlo1 |= (uint32_t)(T[4 + i] & 0xFF) << (8 * i);
      tp.thi0 |= (uint32_t)(T[i] >> 8) << (8 * i);
      tp.thi1 |= (uint32_t)(T[4 + i] >> 8) << (8 * i);
    }
  }
  if (mode_b && ws_bytes < (size_t)tp.n_chunks * gq * 4 * L.d_pad * sizeof(float))
    return fail(TQ_EINVAL, "tq_dequant_values: workspace too small");
  tq_status s = TQ_OK;
  int ok = 0;
  switch (L.bits) {
    case 1: ok = dispatch_values<1>(L, p, tp, batch, max_ctx, mode_b, st, &s); break;
    case 2: ok = dispatch_values<2>(L, p, tp, batch, max_ctx, mode_b, st, &s); break;
    case 3: ok = dispatch_values<3>(L, p, tp, batch, max_ctx, mode_b, st, &s); break;
    case 4: ok = dispatch_values<4>(L, p, tp, batch, max_ctx, mode_b, st, &s); break;
  }
  if (!ok) return fail(TQ_EUNSUPPORTED, "tq_dequant_values: no kernel for this d");
  if (s != TQ_OK) return s;
  return cuda_fail(cudaGetLastError(), "tq_dequant_values launch");
}

}  // namespace tq
