// Key-side building blocks shared by the logits and the fused attention
// kernels: the MMA wrappers, the decoding of packed key chunks into MMA
// operands, and the logits of one 16-key tile ("TurboQuant explained",
// §Stage 2 and §How it works: the logit from the indices and sign bits).
#pragma once

#include "stream.cuh"

namespace tqd {

// Byte-permute tables of the reconstruction levels (kernel parameters).
struct KeyTables {
  uint32_t t0, t1;              // b <= 3: the int8 levels k_i (level i = k_i 2^-f), levels 0..7
  uint32_t lo0, lo1, hi0, hi1;  // b = 4: low / high bytes of the 8 fp16 magnitudes
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

// A read-only 16-byte load that the compiler keeps in program order with the
// other volatile instructions (the table loads must be issued before the
// dependent-launch wait, not sunk to their use).
__device__ __forceinline__ uint4 ldg_early(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
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
__device__ __forceinline__ void decode_nibble_pair(const uint32_t* w, int ks, const KeyTables& p,
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

// ---- one 16-key tile --------------------------------------------------------------

// Words of a record chunk and MMA k-steps for (b, E, F).
template <int BITS, int E, int F>
struct TileShape {
  static constexpr bool kInt8 = BITS <= 3;
  static constexpr int KC = kInt8 ? E / 8 : E / 4;   // codebook MMA k-steps
  static constexpr int KQ = F / 8;                   // sign-term MMA k-steps
  static constexpr int q0 = BITS == 1 ? (E + 31) / 32 : BITS == 2 ? E / 16
                          : BITS == 3 ? 3 * (E / 32) + 2 * ((E % 32) / 16) : E / 8;
  static constexpr int QW = (F + 31) / 32;           // QJL words per chunk
  static constexpr int W = q0 + QW;
  static constexpr int NB = F > 0 ? 4 : 2;           // bytes of a norm slot
};

// The query side of a tile: fragments and scales of one query tile (4
// query slots x high / low slices in the N = 8 columns).
template <int KC, int KQ>
struct QueryFrags {
  uint2 bq[KC];
  uint2 bz[KQ > 0 ? KQ : 1];
  float c0, c1, zsum;
};

// sum_i z_i of query t from its own sign-term fragments: weights 1 on the 2 z
// slots and 2 on the z slots give 2 sum z in columns (2t, 2t+1).
template <int KQ>
__device__ __forceinline__ float query_zsum(const uint2 (&bz)[KQ > 0 ? KQ : 1]) {
  if constexpr (KQ == 0) {
    return 0.0f;
  } else {
    int zs[4] = {0, 0, 0, 0};
#pragma unroll
    for (int kk = 0; kk < KQ; ++kk) mma_s8s8(zs, 0x01010101u, 0x01010101u, 0x02020202u, 0x02020202u, bz[kk]);
    return 0.5f * (float)(256 * zs[0] + zs[1]);
  }
}

// Logits of rows g (la) and g + 8 (lb) of one 16-key tile for this thread's
// query t.  wa / wb: the W words of chunk t of the two keys; na / nb: their
// norm slots (fp16 ||k||, then fp16 ||r|| when F > 0).
// Sign term: k-step kk of a QJL word uses bit planes 2 kk and 2 kk + 1
// against the query side's 2 z / z slots, every k-step and word brought to
// the common weight 128, in one of two forms that give the same sums:
//  * b != 2: the word shifted left by 6 - 2 kk puts the two planes at bits 6
//    and 7 of each byte (weight 128 at once), so the k-steps accumulate on one
//    MMA accumulator with nothing between them;
//  * b = 2: the planes are masked in place (weight 2^(2 kk + 1)) and a Horner
//    step (x 4) between k-steps brings a word to weight 2^(2 n - 1) (n
//    k-steps), then the word is scaled to 128.
// The first form measured faster at b = 1, 3 and 4, the second at b = 2.
template <int BITS, int E, int F>
__device__ __forceinline__ void tile_logits(const uint32_t* wa, const uint32_t* wb, uint32_t na, uint32_t nb,
                                            const QueryFrags<TileShape<BITS, E, F>::KC, TileShape<BITS, E, F>::KQ>& qf,
                                            const KeyTables& kt, float& la, float& lb) {
  using TS = TileShape<BITS, E, F>;
  constexpr int KC = TS::KC, q0 = TS::q0, QW = TS::QW;
  float cba, cbb;
  if constexpr (TS::kInt8) {
    // codebook term: the int8 levels k against the int8 slices of (Pi q)
    int ah[4] = {0, 0, 0, 0};
#pragma unroll
    for (int kk = 0; kk < KC; ++kk) {
      const uint32_t sa = code_selector<BITS, E>(wa, kk);
      const uint32_t sb = code_selector<BITS, E>(wb, kk);
      const uint32_t sa2 = sa >> 16, sb2 = sb >> 16;
      mma_s8s8(ah, prmt(kt.t0, kt.t1, sa), prmt(kt.t0, kt.t1, sb), prmt(kt.t0, kt.t1, sa2),
               prmt(kt.t0, kt.t1, sb2), qf.bq[kk]);
    }
    // columns 2t / 2t+1: high / low slice of query t; 256 hi + lo stays below
    // 2^31 (|k| <= 127, |z| <= 32639, d <= 256)
    cba = (float)(256 * ah[0] + ah[1]);
    cbb = (float)(256 * ah[2] + ah[3]);
  } else {
    float acc0[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < KC; ++ks) {
      uint32_t a0, a2, a1, a3;
      decode_nibble_pair(wa, ks, kt, a0, a2);
      decode_nibble_pair(wb, ks, kt, a1, a3);
      mma_f16(acc0, a0, a1, a2, a3, qf.bq[ks]);
    }
    // columns 2t (hi) and 2t+1 (lo) belong to query t of this tile
    cba = acc0[0] + acc0[1];
    cbb = acc0[2] + acc0[3];
  }
  if constexpr (F > 0) {
    // sign term: bit planes against the int8 slices of 2 z / z
    int qa[4] = {0, 0, 0, 0};                 // 128 sum beta z (hi, lo columns)
#pragma unroll
    for (int w = 0; w < QW; ++w) {
      const int nk = min(4, (F - 32 * w) / 8);   // k-steps of this word (4, or 2 for a half word)
      if constexpr (BITS != 2) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (k < nk) {
            const uint32_t xa = wa[q0 + w] << (6 - 2 * k), xb = wb[q0 + w] << (6 - 2 * k);
            mma_u8s8(qa, xa & 0x40404040u, xb & 0x40404040u, xa & 0x80808080u, xb & 0x80808080u,
                     qf.bz[4 * w + k]);
          }
        }
      } else {
        int a4[4] = {0, 0, 0, 0};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (k < nk) {
            if (k > 0) {
#pragma unroll
              for (int r = 0; r < 4; ++r) a4[r] *= 4;
            }
            const uint32_t m0 = 0x01010101u << (2 * k), m1 = m0 << 1;
            mma_u8s8(a4, wa[q0 + w] & m0, wb[q0 + w] & m0, wa[q0 + w] & m1, wb[q0 + w] & m1, qf.bz[4 * w + k]);
          }
        }
        const int sh = 6 - 2 * (nk - 1);         // weight 2^(2 nk - 1) -> 128
#pragma unroll
        for (int r = 0; r < 4; ++r) qa[r] += a4[r] << sh;
      }
    }
    // sum_i s_i z_i = sum z - 2 sum beta z
    const float ta = fmaf(-1.0f / 64.0f, (float)(256 * qa[0] + qa[1]), qf.zsum);
    const float tb = fmaf(-1.0f / 64.0f, (float)(256 * qa[2] + qa[3]), qf.zsum);
    const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&na));   // ||k||, ||r||
    const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&nb));
    la = fa.x * fmaf(qf.c1 * fa.y, ta, qf.c0 * cba);
    lb = fb.x * fmaf(qf.c1 * fb.y, tb, qf.c0 * cbb);
  } else {
    la = lo_half(na) * (qf.c0 * cba);
    lb = lo_half(nb) * (qf.c0 * cbb);
  }
}

// The two norm slots of the rows g, g + 8 of each 16-key tile of a staged unit.
template <int NB>
__device__ __forceinline__ void unit_norms(const uint8_t* nsl, int g, uint32_t& na0, uint32_t& nb0, uint32_t& na1,
                                           uint32_t& nb1) {
  if constexpr (NB == 4) {
    const uint32_t* n = reinterpret_cast<const uint32_t*>(nsl);
    na0 = n[g]; nb0 = n[g + 8]; na1 = n[16 + g]; nb1 = n[24 + g];
  } else {
    na0 = *reinterpret_cast<const unsigned short*>(nsl + 2 * g);
    nb0 = *reinterpret_cast<const unsigned short*>(nsl + 2 * (g + 8));
    na1 = *reinterpret_cast<const unsigned short*>(nsl + 32 + 2 * g);
    nb1 = *reinterpret_cast<const unsigned short*>(nsl + 32 + 2 * (g + 8));
  }
}

// A copy slot: one 64-key unit, 64 records (16W bytes each) then 64 norm slots.
template <int W, int NB>
struct SlotShape {
  static constexpr int kRecBytes = 16 * W;
  static constexpr int kNormOff = 64 * 16 * W;
  static constexpr int kBytes = (64 * (16 * W + NB) + 15) / 16 * 16;
};

// One line (sequence b, KV head h, query tile qt) of a CTA's share: keys
// [klo, khi) are the share's, keys [klo, k1) are read (k1 = min(khi,
// context)); its block-table entries are [first, first + npg), staged from
// entry ebase on.
struct LineView {
  int b, h, qt, klo, khi, k1, first, npg, ebase;
};

}  // namespace tqd
