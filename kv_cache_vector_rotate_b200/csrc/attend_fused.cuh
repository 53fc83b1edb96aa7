// Fused split-K decode attention straight from the two packed caches.
//
// "TurboQuant explained" (a2a-mcp.org), §How it works: the attention logits
// come from the compressed keys without dequantizing them; §Stage 1: the
// values are the MSE stage's reconstructions ||v|| Pi_v^T c[idx].  One pass
// over the caches does, for each 64-token unit of a line (sequence b, KV
// head h, tile of 4 query heads):
//  1. the logits of the unit's keys for the 4 query slots -- the logits
//     kernel's 16-key tiles, key operand built in registers;
//  2. an online softmax update per query slot: running maximum m and sum l
//     of 2^(s - m), s = scale log2(e) L (the base-2 form of exp(scale L));
//  3. acc += p_t ||v_t|| c[idx_t] in the value codebook's rotated space, on
//     the tensor cores: the value codes of 16 tokens are decoded into an fp16
//     [token][coordinate] tile, ldmatrix.trans turns it into A fragments
//     (coordinates x tokens), and p_t ||v_t|| (fp16 hi + lo, 4 query slots x
//     2) are the B columns -- the value pass's tile;
// with acc scaled by 2^(m_old - m_new) whenever a maximum grows.
//
// Work split: the lines' 64-token units are numbered line by line and every
// CTA takes a contiguous share (at most two lines; its consumer warps are
// divided between the lines in proportion to their units).  A producer
// warp's lane w feeds consumer warp w: per unit one bulk copy of the key
// head block and one of the value head block (64-token pages; pieces
// otherwise) into the warp's ring slot, both completing one mbarrier.  The
// CTA merges its warps' (m, l, acc) per line and writes one partial per line
// and query slot; attend_finish_kernel merges the partials of a line,
// divides by l and applies Pi_v^T.  HBM traffic: the two caches' records
// once, plus a few KB of partials.
//
// A token counts only if its key and value pages are valid; a bad page is
// reported and its tokens leave the softmax.  Every wait is bounded: a CTA
// where one gives up reports TQ_DEV_ERR_TIMEOUT and lets its copies land
// before it exits.
#pragma once

#include <cmath>

#include "key_tile.cuh"
#include "pack.cuh"
#include "value_tile.cuh"

namespace tqd {

constexpr int kAttPages = 512;      // block-table entries staged per CTA and cache
constexpr int kAttMaxWarps = 11;    // consumer warps (+ 1 producer: 12 warps, 168 registers)
constexpr int kAttMaxSlots = 2 * kAttMaxWarps;

struct AttendParams {
  tq::CacheView kcv, vcv;
  int page_shift;            // log2(page_tokens), the same for both caches
  const int32_t* ctx_len;
  int n_kv_heads, n_q_heads, G, qtiles;
  int units;                 // U: 64-token units per line
  int max_ctx;               // ctx_len values are clamped to [0, max_ctx]
  int per_cta, extra;        // CTA c owns per_cta units, + 1 when c < extra
  int n_cta;
  FastDiv div_u, div_qtiles, div_kv;
  int nc;                    // consumer warps
  int ring_shift;            // S = 1 << ring_shift slots per consumer warp
  int fixed_off;             // byte offset of AttendFixed in shared memory
  float sl2;                 // softmax scale x log2(e)
  const uint2* frag;         // query fragments (preparation kernel)
  const uint2* qfrag;
  const float2* scal;
  KeyTables kt;              // key levels
  uint32_t tlo0, tlo1, thi0, thi1;   // value levels (fp16 bytes)
  float* partial;            // [n_cta][2][4][4E + 2]: acc[4E], m, l
  // finish
  const float* pi32;         // value codebook Pi [d_pad][d]
  float* out;                // [batch][n_q_heads][d]
  int d;
};

// 16-byte piece slot of coordinates 8 piece .. 8 piece + 7 in row `row` of a
// value tile.  XOR with the row (mod 8) spreads the 8 rows that one
// ldmatrix reads over the 8 16-byte bank groups; pieces 8..15 are also XORed
// with 4, because the two lanes that decode one token write pieces 8 apart
// at once (both halves of a row then land in different bank groups).
__device__ __forceinline__ int tile_swz(int row, int piece) { return piece ^ (row & 7) ^ ((piece >> 1) & 4); }

// N words (N even) from shared memory at a multiple of 8 bytes, in 8-byte
// loads, or 16-byte ones when N is a multiple of 4 and A16 says the address
// is a multiple of 16.  The two chunks that a lane decodes (8 VW bytes at
// token x 16 VW + half x 8 VW) load this way without bank conflicts at
// VW = 1, 2, 3 (chunk by chunk, two lanes shared each bank).
template <int N, bool A16>
__device__ __forceinline__ void lds_pairs(const uint8_t* src, uint32_t (&w)[N]) {
  static_assert(N % 2 == 0, "pairs of words");
  if constexpr (A16 && N % 4 == 0) {
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const uint4 v = reinterpret_cast<const uint4*>(src)[i];
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
      const uint2 v = reinterpret_cast<const uint2*>(src)[i];
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  }
}

// Shared memory: the consumer warps' rings (S slots each), then their tiles,
// then this fixed part.
template <int KC, int KQ>
struct AttendFixed {
  uint64_t full_bar[kAttMaxSlots];
  uint64_t empty_bar[kAttMaxSlots];
  int64_t kbase[kAttPages];                // byte offset of the key head block, -1 for a bad page
  int64_t vbase[kAttPages];                // value head block
  uint2 fr[2][KC * 32];                    // codebook fragments of the two lines
  uint2 fz[2][(KQ > 0 ? KQ : 1) * 32];     // sign-term fragments
  float2 scal[8];                          // {c0, c1} of query slot 4 line + q
  int flags;                               // bit 0: a wait gave up
  int slot_last[kAttMaxSlots];             // last unit (ordinal j) issued into each slot
};

// Byte sizes for key chunk words KW (norm slot KNB bytes), value chunk words
// VW and E coordinates per chunk.
template <int KW, int KNB, int VW, int E>
struct AttShape {
  static constexpr int kKeyRec = 16 * KW;
  static constexpr int kKeyNormOff = 64 * kKeyRec;
  static constexpr int kKeyBytes = (64 * (kKeyRec + KNB) + 15) / 16 * 16;
  static constexpr int kValRec = 16 * VW;
  static constexpr int kValNormOff = 64 * kValRec;
  static constexpr int kValBytes = (64 * (kValRec + 2) + 15) / 16 * 16;
  static constexpr int kSlot = kKeyBytes + kValBytes;
  static constexpr int kTile = 16 * 4 * E * 2;   // fp16 [16 tokens][4E coordinates]
  static constexpr int kWn = 8 * kBRow * 2;      // p ||v|| as fp16 hi + lo B rows [8][kBRow]
  static constexpr int kWarpTile = kTile + kWn;
};

template <int KB, int VB, int E, int F>
__global__ void __launch_bounds__((kAttMaxWarps + 1) * 32, 1) attend_kernel(AttendParams p) {
  using TS = TileShape<KB, E, F>;
  constexpr int KC = TS::KC, KQ = TS::KQ, KW = TS::W, KNB = TS::NB;
  constexpr int VW = ChunkWords<VB, E, 0>::W;
  using SH = AttShape<KW, KNB, VW, E>;
  constexpr int KREC = SH::kKeyRec, KNOFF = SH::kKeyNormOff;
  constexpr int VREC = SH::kValRec, VNOFF = SH::kValNormOff;
  constexpr int DP = 4 * E, MT = DP / 16, PW = DP / 8;   // coordinates, 16-coordinate tiles, 8-coordinate pieces
  extern __shared__ __align__(128) uint8_t smem[];
  auto& fx = *reinterpret_cast<AttendFixed<KC, KQ>*>(smem + p.fixed_off);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NT = blockDim.x;
  const int NC = p.nc;
  const bool producer = warp == NC;
  const int g = lane >> 2, t = lane & 3;
  const int c = blockIdx.x;
  const int i0 = c * p.per_cta + min(c, p.extra);
  const int n_units = p.per_cta + (c < p.extra ? 1 : 0);
  const int U = p.units;
  const int line0 = (int)fdiv((uint32_t)i0, p.div_u);
  const int n_lines = n_units > 0 ? (int)fdiv((uint32_t)(i0 + n_units - 1), p.div_u) - line0 + 1 : 0;
  const int ua0 = i0 - line0 * U;
  const int split = n_lines > 1 ? (line0 + 1) * U - i0 : n_units;   // units of line 0
  const int ps = p.page_shift, P = 1 << ps;
  const int S = 1 << p.ring_shift;
  // consumer warps [0, NC0) take line 0, [NC0, NC) line 1
  const int NC0 = n_lines > 1 ? min(NC - 1, max(1, (NC * split + n_units / 2) / n_units)) : NC;
  const int NC1 = NC - NC0;
  auto n_of = [&](int w) -> int {   // units of consumer warp w
    if (w < NC0) return w < split ? (split - w - 1) / NC0 + 1 : 0;
    const int w1 = w - NC0, n1 = n_units - split;
    return w1 < n1 ? (n1 - w1 - 1) / NC1 + 1 : 0;
  };
  auto unit_of = [&](int w, int j) -> int { return w < NC0 ? w + j * NC0 : split + (w - NC0) + j * NC1; };

  if (tid < NC * S) {
    mbar_init(&fx.full_bar[tid], 1);
    mbar_init(&fx.empty_bar[tid], 1);
    fx.slot_last[tid] = -1;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (tid == 0) fx.flags = 0;

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
    L.npg = s < n_lines && L.klo < L.khi ? ((L.khi - 1) >> ps) - L.first + 1 : 0;
    L.k1 = 0;
    L.ebase = 0;
    return L;
  };
  LineView L0 = make_line(0), L1 = make_line(1);
  L1.ebase = L0.npg;
  // every kernel before the preparation kernel has finished (it releases
  // this grid only after its own wait): the caches may be read already
  const int ctx0 = L0.npg > 0 ? p.ctx_len[L0.b] : 0;
  const int ctx1 = L1.npg > 0 ? p.ctx_len[L1.b] : 0;
  int64_t pk[4] = {0, 0, 0, 0}, pv[4] = {0, 0, 0, 0};   // kAttPages <= 4 * NT for NT >= 128
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int j = tid + k * NT;
    if (j < L0.npg + L1.npg) {
      const LineView& L = j < L0.npg ? L0 : L1;
      const int pidx = L.first + j - L.ebase;
      pk[k] = p.kcv.block_table[(int64_t)L.b * p.kcv.max_pages + pidx];
      pv[k] = p.vcv.block_table[(int64_t)L.b * p.vcv.max_pages + pidx];
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
      const bool used = L.k1 > L.klo && pidx <= ((L.k1 - 1) >> ps);   // pages past the context are not read
      const bool kval = pk[k] >= 0 && pk[k] < p.kcv.n_pages;
      const bool vval = pv[k] >= 0 && pv[k] < p.vcv.n_pages;
      fx.kbase[j] = kval ? pk[k] * p.kcv.page_bytes + (int64_t)L.h * p.kcv.head_block_bytes : -1;
      fx.vbase[j] = vval ? pv[k] * p.vcv.page_bytes + (int64_t)L.h * p.vcv.head_block_bytes : -1;
      if (used && !kval) report(p.kcv.err, TQ_DEV_ERR_PAGE);
      if (used && !vval) report(p.vcv.err, TQ_DEV_ERR_PAGE);
      bad = bad || (used && !(kval && vval));
    }
  }
  const bool fast = !__syncthreads_or(bad);   // also publishes the barriers' init

  if (producer) {
    // ---------------------------------------------------------- producer
    const uint64_t pol = evict_first_policy();   // both caches are streamed once per call
    // the copies of the j-th unit of consumer warp w into its slot (the slot
    // is free: j < S, or its previous unit was released)
    auto issue = [&](int w, int j) {
      const int slot = w * S + (j & (S - 1));
      fx.slot_last[slot] = j;
      uint64_t* bar = &fx.full_bar[slot];
      const uint32_t dst = smem_addr(smem) + slot * SH::kSlot;
      const int i = unit_of(w, j);
      const bool in1 = i >= split;
      const int pos = 64 * (in1 ? i - split : ua0 + i);
      const LineView& L = in1 ? L1 : L0;
      const int eb = L.ebase - L.first;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the consumer's reads of the slot first
      if (fast && P == 64 && pos < L.k1) {
        // one page head block per cache: records and norms in one copy each
        mbar_arrive_tx(bar, 64 * (KREC + KNB) + 64 * (VREC + 2));
        bulk_copy(dst, p.kcv.pages + fx.kbase[eb + (pos >> ps)], 64 * (KREC + KNB), bar, pol);
        bulk_copy(dst + SH::kKeyBytes, p.vcv.pages + fx.vbase[eb + (pos >> ps)], 64 * (VREC + 2), bar, pol);
        return;
      }
      // pieces of min(P, 64) tokens (16 on a cache with a bad page)
      const int piece = fast ? min(P, 64) : 16;
      uint32_t bytes = 0;
      for (int k = pos; k < pos + 64; k += piece) {
        if (k >= L.k1) break;
        if (fx.kbase[eb + (k >> ps)] >= 0) bytes += piece * (KREC + KNB);
        if (fx.vbase[eb + (k >> ps)] >= 0) bytes += piece * (VREC + 2);
      }
      mbar_arrive_tx(bar, bytes);          // 0 bytes: the phase completes on the arrival alone
      for (int k = pos; k < pos + 64; k += piece) {
        if (k >= L.k1) break;
        const int sl = k & (P - 1);
        const int64_t ko = fx.kbase[eb + (k >> ps)], vo = fx.vbase[eb + (k >> ps)];
        if (ko >= 0) {
          const uint8_t* hb = p.kcv.pages + ko;
          bulk_copy(dst + (k - pos) * KREC, hb + (int64_t)sl * KREC, piece * KREC, bar, pol);
          bulk_copy(dst + KNOFF + (k - pos) * KNB, hb + (int64_t)P * KREC + sl * KNB, piece * KNB, bar, pol);
        }
        if (vo >= 0) {
          const uint8_t* hb = p.vcv.pages + vo;
          const uint32_t vd = dst + SH::kKeyBytes;
          bulk_copy(vd + (k - pos) * VREC, hb + (int64_t)sl * VREC, piece * VREC, bar, pol);
          bulk_copy(vd + VNOFF + (k - pos) * 2, hb + (int64_t)P * VREC + sl * 2, piece * 2, bar, pol);
        }
      }
    };
    const int n_me = lane < NC ? n_of(lane) : 0;
    // one unit per consumer warp before the fragments are fetched
    if (n_me > 0) issue(lane, 0);
    asm volatile("barrier.sync 1, %0;" ::"r"(NT) : "memory");   // the consumers have the fragments
    // then lane w refills warp w's slots as they are released (non-blocking
    // tests: the lanes do not wait on one another's slots)
    int jn = 1;
    bool ok = true;
    const long long t0 = clock64();
    while (__any_sync(0xffffffffu, jn < n_me)) {
      bool did = false;
      if (jn < n_me) {
        const int slot = lane * S + (jn & (S - 1));
        if (jn < S || mbar_test(&fx.empty_bar[slot], (uint32_t)((jn >> p.ring_shift) - 1) & 1u)) {
          issue(lane, jn);
          ++jn;
          did = true;
        }
      }
      if (!__any_sync(0xffffffffu, did)) {
        const bool late = __shfl_sync(0xffffffffu, clock64() - t0 > kWaitCycles ? 1 : 0, 0) != 0;
        if (late) {
          ok = false;
          break;
        }
        __nanosleep(256);
      }
    }
    if (!ok && lane == 0) {
      atomicOr(&fx.flags, 1);
      report(p.kcv.err, TQ_DEV_ERR_TIMEOUT);
    }
  } else {
    // ---------------------------------------------------------- consumers
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");   // the finish kernel prefetches Pi meanwhile
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

  // consumer state (registers); the producer keeps m = -inf, l = 0, acc = 0
  float acc[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.0f;
  float m_run = -INFINITY, l_run = 0.0f;
  // query slot t's B values carry 2^vsc (set by the largest p ||v|| seen, kept
  // below 2^14) so that the fp16 hi + lo split keeps its precision whatever
  // the scale of the value norms; the accumulators are undone at the end
  int vsc = 0;
  bool vhas = false;
  if (!producer) {
    const int s = warp < NC0 ? 0 : 1;
    const LineView& L = s ? L1 : L0;
    const int k1 = L.k1, eb = L.ebase - L.first;
    QueryFrags<KC, KQ> qf;
#pragma unroll
    for (int kk = 0; kk < KC; ++kk) qf.bq[kk] = fx.fr[s][kk * 32 + lane];
#pragma unroll
    for (int kk = 0; kk < KQ; ++kk) qf.bz[kk] = fx.fz[s][kk * 32 + lane];
    qf.zsum = query_zsum<KQ>(qf.bz);
    const float2 sc = fx.scal[4 * s + t];
    qf.c0 = sc.x;
    qf.c1 = F > 0 ? sc.y : 0.0f;
    const int n_my = n_of(warp);
    uint64_t* fbars = fx.full_bar + warp * S;
    uint64_t* ebars = fx.empty_bar + warp * S;
    const uint8_t* ring = smem + warp * S * SH::kSlot;
    uint8_t* tile = smem + NC * S * SH::kSlot + warp * SH::kWarpTile;
    unsigned short* wh = reinterpret_cast<unsigned short*>(tile + SH::kTile);
    const uint32_t* whw = reinterpret_cast<const uint32_t*>(wh);
    uint4* tile4 = reinterpret_cast<uint4*>(tile);
    const int tk = lane >> 1, hh = lane & 1;   // decoding: token tk of a 16-token step, coordinates half hh
    for (int j = 0; j < n_my; ++j) {
      if (!mbar_wait_sleep(&fbars[j & (S - 1)], (uint32_t)(j >> p.ring_shift) & 1u)) {
        if (lane == 0) {
          atomicOr(&fx.flags, 1);
          report(p.kcv.err, TQ_DEV_ERR_TIMEOUT);
        }
        break;
      }
      const int i = unit_of(warp, j);
      const int pos0 = 64 * (s ? i - split : ua0 + i);
      const uint8_t* kst = ring + (j & (S - 1)) * SH::kSlot;
      const uint8_t* vst = kst + SH::kKeyBytes;
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {           // two 32-token halves of the unit
        const int pos = pos0 + 32 * hf;
        if (pos >= k1) break;                    // past the context (warp-uniform)
        // 1. logits of keys pos + g + 8 r (r = 0..3) for query slot t
        float lg[4];
        {
          const uint8_t* st = kst + hf * 32 * KREC;
          uint32_t wa0[KW], wb0[KW], wa1[KW], wb1[KW];
          lds_chunk<KW>(st + g * KREC + t * (4 * KW), wa0);
          lds_chunk<KW>(st + (g + 8) * KREC + t * (4 * KW), wb0);
          lds_chunk<KW>(st + (16 + g) * KREC + t * (4 * KW), wa1);
          lds_chunk<KW>(st + (24 + g) * KREC + t * (4 * KW), wb1);
          uint32_t na0, nb0, na1, nb1;
          unit_norms<KNB>(kst + KNOFF + hf * 32 * KNB, g, na0, nb0, na1, nb1);
          tile_logits<KB, E, F>(wa0, wb0, na0, nb0, qf, p.kt, lg[0], lg[1]);
          tile_logits<KB, E, F>(wa1, wb1, na1, nb1, qf, p.kt, lg[2], lg[3]);
        }
        // 2. online softmax (base 2) for query slot t over the 32 tokens
        bool ok[4];
        float sv[4], mx = -INFINITY;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int key = pos + g + 8 * r;
          ok[r] = key < k1;
          if (!fast && ok[r]) ok[r] = fx.kbase[eb + (key >> ps)] >= 0 && fx.vbase[eb + (key >> ps)] >= 0;
          sv[r] = ok[r] ? lg[r] * p.sl2 : -INFINITY;
          mx = fmaxf(mx, sv[r]);
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_run, mx);
        const float alpha = m_new == -INFINITY ? 1.0f : exp2f(m_run - m_new);
        float psum = 0.0f, pv[4];
        float pmax = 0.0f;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float pr = ok[r] ? exp2f(sv[r] - m_new) : 0.0f;
          psum += pr;
          // p ||v|| of token g + 8 r (the norm of a token that does not count is not read)
          const int tok = 32 * hf + g + 8 * r;
          const float vn = ok[r] ? __half2float(reinterpret_cast<const __half*>(vst + VNOFF)[tok]) : 0.0f;
          pv[r] = pr * vn;
          pmax = fmaxf(pmax, fabsf(pv[r]));
        }
        pmax = fmaxf(pmax, __shfl_xor_sync(0xffffffffu, pmax, 4));
        pmax = fmaxf(pmax, __shfl_xor_sync(0xffffffffu, pmax, 8));
        pmax = fmaxf(pmax, __shfl_xor_sync(0xffffffffu, pmax, 16));
        float beta = alpha;                         // accumulator factor: softmax and scale
        if (pmax > 0.0f) {
          const int e = (int)((__float_as_uint(pmax) >> 23) & 0xFFu) - 126;   // 2^(e-1) <= pmax < 2^e
          const int s_new = min(120, 14 - e);
          if (!vhas || s_new < vsc) {
            if (vhas) beta *= __int_as_float((max(-126, s_new - vsc) + 127) << 23);
            vsc = s_new;
            vhas = true;
          }
        }
        const float up = vhas ? __int_as_float((vsc + 127) << 23) : 0.0f;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          // token g + 8 r, query slot t: fp16 hi + lo, once per token and slot
          const float x = pv[r] * up;
          const __half hi = __float2half_rn(x);
          const __half lo = __float2half_rn(x - __half2float(hi));
          wh[(2 * t) * kBRow + g + 8 * r] = __half_as_ushort(hi);
          wh[(2 * t + 1) * kBRow + g + 8 * r] = __half_as_ushort(lo);
        }
        l_run = l_run * alpha + psum;
        m_run = m_new;
        if (__any_sync(0xffffffffu, beta != 1.0f)) {
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            acc[mt][0] *= beta; acc[mt][1] *= beta; acc[mt][2] *= beta; acc[mt][3] *= beta;
          }
        }
        // 3. values: two steps of 16 tokens
#pragma unroll 1
        for (int ks = 0; ks < 2; ++ks) {
          {
            const uint8_t* rec = vst + (32 * hf + 16 * ks + tk) * VREC;
            uint32_t cw2[2 * VW];                // chunks 2 hh and 2 hh + 1: contiguous
            lds_pairs<2 * VW, VW % 2 == 0>(rec + hh * (8 * VW), cw2);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              const int ch = 2 * hh + cc;
              const uint32_t* cw = cw2 + cc * VW;
#pragma unroll
              for (int kk = 0; kk < E / 8; ++kk) {
                const int piece = ch * (E / 8) + kk;
                tile4[tk * PW + tile_swz(tk, piece)] = decode8<VB, E>(cw, kk, p);
              }
            }
          }
          __syncwarp();                          // the tile and the weights
          uint32_t bw[2];
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int tt = 16 * ks + 2 * t + 8 * r;
            bw[r] = whw[(g * kBRow + tt) / 2];   // B column g: tokens tt, tt + 1
          }
          const int mi = lane >> 3, rr = lane & 7;
          const int row = 8 * (mi >> 1) + rr;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            const int piece = 2 * mt + (mi & 1);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_trans(smem_addr(tile + row * (DP * 2) + 16 * tile_swz(row, piece)), a0, a1, a2, a3);
            mma_f16(acc[mt], a0, a1, a2, a3, make_uint2(bw[0], bw[1]));
          }
          __syncwarp();                          // the tile is rewritten next
        }
      }
      __syncwarp();                              // every read of the slot precedes its release
      if (lane == 0) mbar_arrive(&ebars[j & (S - 1)]);
    }
  }

  // every thread of the CTA meets here; after a wait that gave up, the
  // copies already issued land (each wait bounded) before shared memory is
  // reused
  __syncthreads();
  if (fx.flags & 1) {
    for (int k = tid; k < NC * S; k += NT)
      if (fx.slot_last[k] >= 0) mbar_wait(&fx.full_bar[k], (uint32_t)(fx.slot_last[k] >> p.ring_shift) & 1u);
    __syncthreads();
  }
  // the warps' (m, l, acc) per query slot meet in shared memory (the rings
  // are free now): red[w][q][0, DP) acc, [DP] m, [DP + 1] l, rows of RSS
  // floats (padded so that the 4 query slots' lanes of a store fall in
  // different banks); the partials in global memory have rows of RS floats
  float* red = reinterpret_cast<float*>(smem);
  constexpr int RS = DP + 2, RSS = DP + 8;
  if (!producer) {
    float lt = l_run;
    lt += __shfl_xor_sync(0xffffffffu, lt, 4);
    lt += __shfl_xor_sync(0xffffffffu, lt, 8);
    lt += __shfl_xor_sync(0xffffffffu, lt, 16);
    float* rw = red + (warp * 4 + t) * RSS;
    const float unsc = vhas ? __int_as_float((127 - vsc) << 23) : 1.0f;   // 2^-vsc
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      rw[16 * mt + g] = (acc[mt][0] + acc[mt][1]) * unsc;       // hi + lo columns of query slot t
      rw[16 * mt + g + 8] = (acc[mt][2] + acc[mt][3]) * unsc;
    }
    if (g == 0) {
      rw[DP] = m_run;
      rw[DP + 1] = lt;
    }
  }
  __syncthreads();
  for (int s = 0; s < n_lines; ++s) {
    const int wa = s == 0 ? 0 : NC0, wb = s == 0 ? NC0 : NC;
    float* dst = p.partial + ((int64_t)c * 2 + s) * 4 * RS;
    for (int x = tid; x < 4 * RS; x += NT) {
      const int q = x / RS, k = x - q * RS;
      float M = -INFINITY;
      for (int w = wa; w < wb; ++w) M = fmaxf(M, red[(w * 4 + q) * RSS + DP]);
      float v = M;
      if (k != DP) {
        v = 0.0f;
        if (M != -INFINITY)
          for (int w = wa; w < wb; ++w) {
            const float mw = red[(w * 4 + q) * RSS + DP];
            if (mw != -INFINITY) v += red[(w * 4 + q) * RSS + k] * exp2f(mw - M);
          }
      }
      dst[x] = v;
    }
  }
}

// Merge of a line's partials and the rotation back: one CTA per (line, query
// slot < G); CL x DP threads (CL = 1024 / DP chunk lanes).  Thread (cl, k)
// loads its entries Pi[j][k] (j = cl, cl + CL, ...) before it waits for the
// attention kernel, then combines the partials of CTAs cl, cl + CL, ... of
// the line: o_k = sum_j Pi[j][k] a_j / l with a = sum_c 2^(m_c - M) acc_c,
// l = sum_c 2^(m_c - M) l_c, M = max_c m_c (o = 0 when no token counts).
template <int E>
__global__ void __launch_bounds__(1024) attend_finish_kernel(AttendParams p) {
  constexpr int DP = 4 * E, RS = DP + 2;
  constexpr int CL = 1024 / DP;
  constexpr int JN = (DP + CL - 1) / CL;
  __shared__ float red[CL][DP + 1];
  __shared__ float a[DP + 1];
  const int ln = blockIdx.x / 4, q = blockIdx.x % 4;
  const int gi = (int)fdiv((uint32_t)ln, p.div_qtiles), qt = ln - gi * p.qtiles;
  const int hql = qt * 4 + q;
  const int b = (int)fdiv((uint32_t)gi, p.div_kv), h = gi - b * p.n_kv_heads;
  const int k = threadIdx.x % DP, cl = threadIdx.x / DP;
  const int d = p.d;
  float pij[JN];
#pragma unroll
  for (int n = 0; n < JN; ++n) {
    const int j = cl + CL * n;
    pij[n] = (k < d && j < d) ? __ldg(p.pi32 + (size_t)j * d + k) : 0.0f;
  }
  __shared__ int crange[2];
  __shared__ float cmax[32];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (hql >= p.G) return;
  // the CTAs holding units of line ln: [c_a, c_b] (32-bit arithmetic: the
  // unit count is below 2^31)
  if (threadIdx.x == 0) {
    const int per = p.per_cta, big = p.extra * (per + 1);
    auto cta_of = [&](int x) { return x < big ? x / (per + 1) : p.extra + (x - big) / max(per, 1); };
    crange[0] = cta_of(ln * p.units);
    crange[1] = cta_of(ln * p.units + p.units - 1);
  }
  __syncthreads();
  const int c_a = crange[0], c_b = crange[1];
  // partial slot of CTA cc for line ln
  auto slot_of = [&](int cc) -> const float* {
    const int i0 = cc * p.per_cta + min(cc, p.extra);
    const int s = ln - (int)fdiv((uint32_t)i0, p.div_u);
    return p.partial + (((int64_t)cc * 2 + s) * 4 + q) * RS;
  };
  float M = -INFINITY;
  for (int cc = c_a + (int)threadIdx.x; cc <= c_b; cc += blockDim.x) M = fmaxf(M, slot_of(cc)[DP]);
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if ((threadIdx.x & 31) == 0) cmax[threadIdx.x >> 5] = M;
  __syncthreads();
  M = -INFINITY;
#pragma unroll
  for (int w = 0; w < 32; ++w) M = fmaxf(M, cmax[w]);
  float sa = 0.0f, sl = 0.0f;
  if (M != -INFINITY) {
    for (int cc = c_a + cl; cc <= c_b; cc += CL) {
      const float* src = slot_of(cc);
      const float mc = src[DP];
      if (mc == -INFINITY) continue;
      const float wgt = exp2f(mc - M);
      sa += wgt * src[k];
      if (k == 0) sl += wgt * src[DP + 1];
    }
  }
  red[cl][k] = sa;
  if (k == 0) red[cl][DP] = sl;
  __syncthreads();
  if (cl == 0) {
    float t2 = 0.0f;
#pragma unroll
    for (int x = 0; x < CL; ++x) t2 += red[x][k];
    a[k] = t2;
    if (k == 0) {
      float l2 = 0.0f;
#pragma unroll
      for (int x = 0; x < CL; ++x) l2 += red[x][DP];
      a[DP] = l2;
    }
  }
  __syncthreads();
  float o = 0.0f;
#pragma unroll
  for (int n = 0; n < JN; ++n) {
    const int j = cl + CL * n;
    if (j < DP) o = fmaf(pij[n], a[j], o);
  }
  __syncthreads();
  red[cl][k] = o;
  __syncthreads();
  if (cl == 0 && k < d) {
    float t2 = 0.0f;
#pragma unroll
    for (int x = 0; x < CL; ++x) t2 += red[x][k];
    const float l = a[DP];
    p.out[((int64_t)b * p.n_q_heads + (int64_t)h * p.G + hql) * d + k] = l > 0.0f ? t2 / l : 0.0f;
  }
}

}  // namespace tqd

namespace tq {

// Launch plan of the fused kernel: consumer warps, ring depth and shared memory.
struct AttendPlan {
  int nc, ring_shift, fixed_off, smem;
};

template <int KB, int VB, int E, int F>
bool attend_plan(AttendPlan* pl) {
  using TS = tqd::TileShape<KB, E, F>;
  using SH = tqd::AttShape<TS::W, TS::NB, tqd::ChunkWords<VB, E, 0>::W, E>;
  const int fixed = (int)sizeof(tqd::AttendFixed<TS::KC, TS::KQ>);
  const int smax = 227 * 1024;
  for (int rs = 1; rs >= 0; --rs) {
    const int per_warp = (1 << rs) * SH::kSlot + SH::kWarpTile;
    const int nc = std::min(tqd::kAttMaxWarps, (smax - fixed - 128) / per_warp);
    if (nc >= 3) {
      const int ring = nc * per_warp;
      // the end-of-kernel merge area (nc x 4 x (4E + 8) floats) reuses the rings
      if (nc * 4 * (4 * E + 8) * 4 > ring) continue;
      pl->nc = nc;
      pl->ring_shift = rs;
      pl->fixed_off = (ring + 127) / 128 * 128;
      pl->smem = pl->fixed_off + fixed;
      return true;
    }
  }
  return false;
}

template <int KB, int VB, int E, int F>
tq_status launch_attend_fused_t(tqd::AttendParams p, int lines, cudaStream_t st) {
  AttendPlan pl;
  if (!attend_plan<KB, VB, E, F>(&pl)) return fail(TQ_EUNSUPPORTED, "tq_attend: shared-memory plan");
  static PerDeviceOnce attr;
  if (const int dev_ = current_device(); attr.need(dev_)) {
    cudaError_t e = cudaFuncSetAttribute(tqd::attend_kernel<KB, VB, E, F>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
    if (e != cudaSuccess) return cuda_fail(e, "tq_attend: smem attribute");
    attr.mark(dev_);
  }
  p.nc = pl.nc;
  p.ring_shift = pl.ring_shift;
  p.fixed_off = pl.fixed_off;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.n_cta);
  cfg.blockDim = dim3((pl.nc + 1) * 32);
  cfg.dynamicSmemBytes = (size_t)pl.smem;
  cfg.stream = st;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, tqd::attend_kernel<KB, VB, E, F>, p);
  if (e != cudaSuccess) return cuda_fail(e, "tq_attend: attention launch");
  cudaLaunchConfig_t cf2 = {};
  cf2.gridDim = dim3((unsigned)(lines * 4));
  cf2.blockDim = dim3(1024);
  cf2.stream = st;
  cf2.attrs = attrs;
  cf2.numAttrs = 1;
  e = cudaLaunchKernelEx(&cf2, tqd::attend_finish_kernel<E>, p);
  if (e != cudaSuccess) return cuda_fail(e, "tq_attend: finish launch");
  return TQ_OK;
}

// Dispatch over (value bits, E, F) for one key width KB.
template <int KB>
tq_status launch_attend_fused_kb(const tqd::AttendParams& p, int vbits, int E, int F, int lines, cudaStream_t st) {
#define TQ_ATT_CASE(VB_, E_, F_) \
  if (vbits == VB_ && E == E_ && F == F_) return launch_attend_fused_t<KB, VB_, E_, F_>(p, lines, st);
#define TQ_ATT_VB(VB_) TQ_ATT_CASE(VB_, 32, 32) TQ_ATT_CASE(VB_, 32, 0) TQ_ATT_CASE(VB_, 16, 16) TQ_ATT_CASE(VB_, 16, 0)
  TQ_ATT_VB(1) TQ_ATT_VB(2) TQ_ATT_VB(3) TQ_ATT_VB(4)
#undef TQ_ATT_VB
#undef TQ_ATT_CASE
  return fail(TQ_EUNSUPPORTED, "tq_attend: no fused kernel for this (d, m, bits)");
}

}  // namespace tq
