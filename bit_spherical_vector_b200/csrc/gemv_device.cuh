#pragma once
// gemv_device.cuh -- device-side building blocks of the fused SVQ
// decode-and-multiply (shared by the grouped GEMV and the MoE kernels):
// cache-policy loads, lane-block loads and the per-block decode + dot product.
//
// Two decodes, one per arrangement of a block (layout.cuh):
//  * fragment decode (full 128-row tiles, the hot path): per round of 128
//    subvectors, ldmatrix gathers the fp16 codewords into tensor-core A
//    fragments, the sign bits are XORed onto their fp16 sign bits, four
//    mma.m16n8k16 form the eight-element dot products in fp32, and each is
//    scaled by its radius and accumulated in fp32;
//  * owner decode (a partial last tile): a lane owns 4 rows x 16 subvectors;
//    per subvector the codeword is gathered with one 16-byte shared-memory
//    load, signed by XOR, multiplied by x in fp16x2, the 8 products summed in
//    fp32 and scaled by the radius in fp32.
// The radius is r = offset + scale * code ("SAGE", arXiv 2610.14745, Figure 2
// caption: signs, direction index, quantized radius).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "layout.cuh"

namespace svq {
namespace {

// L2 cache policies: packed codes are read once per call (evict first), while a
// matrix's small reused tables -- codebook, permutation, radius parameters and
// the activations -- should stay resident across calls (evict last).  Without
// this a stream of layers evicts every table and each CTA's prologue pays HBM
// latency twice (permutation, then x).
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint4 ldg_stream(const void* p, uint64_t pol) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p), "l"(pol));
  return v;
}

__device__ __forceinline__ uint4 ldg_keep_v4(const uint4* p, uint64_t pol) {
  uint4 v;
  asm("ld.global.nc.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p), "l"(pol));
  return v;
}

__device__ __forceinline__ int ldg_keep_i32(const int32_t* p, uint64_t pol) {
  int v;
  asm("ld.global.nc.L2::cache_hint.b32 %0, [%1], %2;" : "=r"(v) : "l"(p), "l"(pol));
  return v;
}

__device__ __forceinline__ uint16_t ldg_keep_u16(const uint16_t* p, uint64_t pol) {
  uint16_t v;
  asm("ld.global.nc.L2::cache_hint.b16 %0, [%1], %2;" : "=h"(v) : "l"(p), "l"(pol));
  return v;
}

__device__ __forceinline__ uint4 lds128(const unsigned char* base, uint32_t byte_off) {
  return *reinterpret_cast<const uint4*>(base + byte_off);
}

template <int k>
__device__ __forceinline__ uint32_t shl(uint32_t x) {
  if constexpr (k >= 0) return x << k; else return x >> (-k);
}

__device__ __forceinline__ __half2 as_h2(uint32_t u) {
  return *reinterpret_cast<const __half2*>(&u);
}

__device__ __forceinline__ void load_block(uint4 (&d)[kChunks], const uint8_t* blk, int L, int lane,
                                           uint64_t pol) {
#pragma unroll
  for (int c = 0; c < kChunks; ++c) d[c] = ldg_stream(blk + ((size_t)c * L + lane) * 16, pol);
}

// Shared-memory codebook with R replicas (R = 8, 4 or 2): entry e of replica q
// sits in 16-byte slot e*R + q, lane l reads replica l % R.  With R = 8 the 8
// lanes of an LDS.128 phase always hit 8 different bank groups; cb_replicas
// lowers R for 512- and 1024-entry codebooks to keep the table at 32 KB (two
// lanes of a phase may then share a bank group); callers with more shared
// memory to spare pass their own R.  The payload's index field is moved to bit
// l0 = 4 + log2(R) (byte offset e * 16R) with one shift.
struct CbShift {
  uint32_t l0, r1, r2, mask;
};

__device__ __forceinline__ int cb_replicas(int b_d) { return b_d <= 8 ? 8 : (b_d == 9 ? 4 : 2); }

__device__ __forceinline__ CbShift cb_shift(int b_d, int R) {
  const uint32_t l0 = 4u + (R == 8 ? 3u : (R == 4 ? 2u : 1u));
  CbShift c;
  c.l0 = l0;
  c.r1 = 10u - l0;
  c.r2 = 20u - l0;
  c.mask = ((1u << b_d) - 1u) << l0;
  return c;
}

__device__ __forceinline__ CbShift cb_shift(int b_d) { return cb_shift(b_d, cb_replicas(b_d)); }

template <int MT>
__device__ __forceinline__ void process_block(const uint4 (&d)[kChunks], const unsigned char* xb,
                                              int xstride_bytes, const unsigned char* cbs, uint32_t q16,
                                              const CbShift& cs, uint32_t CODEM, const float2 (&scp)[2],
                                              const float2 (&ofp)[2], float2 (&acc)[2][MT]) {
  uint32_t w[kWords];
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    w[4 * c] = d[c].x; w[4 * c + 1] = d[c].y; w[4 * c + 2] = d[c].z; w[4 * c + 3] = d[c].w;
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    uint4 xv[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) xv[m] = lds128(xb, m * xstride_bytes + 16 * j);
    const uint32_t S = w[j];
    float vf[4];
    float dsum[4][MT];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int v = 4 * j + r;
      uint32_t ia, vb;
      if (v < 60) {
        const uint32_t pw = w[16 + v / 3];
        switch (v % 3) {
          case 0: ia = (pw << cs.l0) & cs.mask; vb = shl<13>(pw) & CODEM; break;
          case 1: ia = (pw >> cs.r1) & cs.mask; vb = shl<3>(pw) & CODEM; break;
          default: ia = (pw >> cs.r2) & cs.mask; vb = shl<-7>(pw) & CODEM; break;
        }
      } else {
        const int a = v - 60;
        const uint32_t pw = ((w[16 + 5 * a] >> 30) << 8) | ((w[17 + 5 * a] >> 30) << 6) |
                            ((w[18 + 5 * a] >> 30) << 4) | ((w[19 + 5 * a] >> 30) << 2) |
                            (w[20 + 5 * a] >> 30);
        ia = (pw << cs.l0) & cs.mask;
        vb = shl<13>(pw) & CODEM;
      }
      // replica offset q16 (below bit l0) and the scaled index do not overlap: OR, not add
      uint4 cw = lds128(cbs, ia | q16);
      vf[r] = __uint_as_float(vb | 0x3F800000u);     // 1 + code * 2^-BR
      cw.x ^= (S << (4 * r + 0)) & 0x80008000u;
      cw.y ^= (S << (4 * r + 1)) & 0x80008000u;
      cw.z ^= (S << (4 * r + 2)) & 0x80008000u;
      cw.w ^= (S << (4 * r + 3)) & 0x80008000u;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        // products in fp16 (|c| <= 1, so a product never exceeds |x|), summed in fp32
        const float2 p0 = __half22float2(__hmul2(as_h2(cw.x), as_h2(xv[m].x)));
        const float2 p1 = __half22float2(__hmul2(as_h2(cw.y), as_h2(xv[m].y)));
        const float2 p2 = __half22float2(__hmul2(as_h2(cw.z), as_h2(xv[m].z)));
        const float2 p3 = __half22float2(__hmul2(as_h2(cw.w), as_h2(xv[m].w)));
        const float2 q = __fadd2_rn(__fadd2_rn(p0, p1), __fadd2_rn(p2, p3));
        dsum[r][m] = q.x + q.y;
      }
    }
    // radius r = scp * v + ofp and accumulation, two rows per packed fp32x2 FMA
    const float2 r01 = __ffma2_rn(scp[0], make_float2(vf[0], vf[1]), ofp[0]);
    const float2 r23 = __ffma2_rn(scp[1], make_float2(vf[2], vf[3]), ofp[1]);
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      acc[0][m] = __ffma2_rn(r01, make_float2(dsum[0][m], dsum[1][m]), acc[0][m]);
      acc[1][m] = __ffma2_rn(r23, make_float2(dsum[2][m], dsum[3][m]), acc[1][m]);
    }
  }
}


// ------------------------------------------------------------------ fragment decode (full tiles)
// A full 128-row tile's block is decoded in 16 rounds (layout.cuh, fragment
// arrangement).  Round u = 2gp + rp covers groups 2gp, 2gp+1 and rows
// 4T+2rp, 4T+2rp+1 of every lane T: 128 subvectors.  Their eight-element dot
// products with x run on the tensor cores: four mma.m16n8k16 (fp16 inputs,
// fp32 accumulation), product i taking the 16 rows 16g + 4i + 2rp + e
// (g = 0..7, e = 0..1) as its A rows and the two groups as its two k-halves;
// the B operand holds x of group 2gp in column 2i (k-half 0) and of group
// 2gp+1 in column 2i+1 (k-half 1), zero elsewhere, so the four products
// accumulate into disjoint column pairs of one D fragment.  Lane T then holds
// exactly the four dot products of its own rows (4T+2rp+e, e = 0..1, groups
// 2gp+h, h = 0..1), scales them by their radii and accumulates in fp32.
//   * A operands come straight from the replicated codebook with one
//     ldmatrix.x4 per product (lane l gives the address of A row l%8 + 8((l/8)&1)
//     of k-half l/16; the eight lanes of each 8x8 matrix read eight different
//     replicas: conflict free);
//   * each A word then gets its two sign bits (sign word shifted so the pair
//     lands on the fp16 sign bits, then one XOR under mask);
//   * the four products run as two chains of two (they fill disjoint column
//     pairs, so the chains are added afterwards): half the dependent latency;
//   * each 10-bit slot is brought to bit 0 with one shift; the left shifts that
//     follow (sign pairs onto the fp16 sign bits, index to a byte offset, code
//     to the mantissa) are written as multiplications by values the compiler
//     cannot see (derived from a launch parameter equal to one), so they issue
//     as integer multiply-adds on the FMA pipe and leave the ALU pipe to the
//     masks and XORs.

// Per-launch constants of the fragment decode (uniform across a CTA's threads).
struct FragK {
  uint32_t imask;      // (1 << b_d) - 1: direction index of a slot brought to bit 0
  uint32_t ia_mul;     // 16 R: byte stride of a codebook entry (all replicas)
  uint32_t cv_mul;     // 2^13: radius code bits [b_d, 10) -> mantissa bits [23-BR, 23)
  uint32_t codem;      // ((1 << BR) - 1) << (23 - BR)
  uint32_t m2, m4, m8, m16, m256, m4096;   // 2^1..2^3, 2^4, 2^8, 2^12: sign word shifted left by w = 4i + j
};

__device__ __forceinline__ FragK frag_consts(uint32_t one, int b_d, int R) {
  FragK k;
  k.imask = (one << b_d) - one;
  k.ia_mul = (one << 4) * (uint32_t)R;
  k.cv_mul = one << 13;
  const uint32_t BR = 10u - (uint32_t)b_d;
  k.codem = BR ? (((one << BR) - one) << (23u - BR)) : 0u;
  k.m2 = one << 1; k.m4 = one << 2; k.m8 = one << 3; k.m16 = one << 4; k.m256 = one << 8; k.m4096 = one << 12;
  return k;
}

__device__ __forceinline__ uint32_t mul_lo(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.lo.u32 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t mad_lo(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t mad_hi(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&a)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t lds32(const unsigned char* base, uint32_t byte_off) {
  return *reinterpret_cast<const uint32_t*>(base + byte_off);
}

// d (+)= A B, m16n8k16, fp16 inputs, fp32 accumulators
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                         const float (&c)[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
        "f"(c[3]));
}

// Slot k of round b of a quarter: byte offset of its codebook row (this
// lane's address role) and the radius value v = 1 + code * 2^-BR of this
// lane's own subvector k (owner role), from the quarter's 160 payload bits
// (P[0..4], slot at bit 40b + 10k).
template <int BB, int KK>
__device__ __forceinline__ void frag_slot(const uint32_t (&P)[5], const FragK& fk, uint32_t base_q, uint32_t& addr,
                                          float& v) {
  constexpr int p = 40 * BB + 10 * KK;
  constexpr int wi = p >> 5, o = p & 31;
  uint32_t W;
  if constexpr (o == 0) W = P[wi];
  else if constexpr (o > 22) W = __funnelshift_r(P[wi], P[wi + 1], o);   // slot crosses two words
  else W = P[wi] >> o;
  addr = mad_lo(W & fk.imask, fk.ia_mul, base_q);
  v = __uint_as_float((mul_lo(W, fk.cv_mul) & fk.codem) | 0x3F800000u);
}

// Round b (0..3) of a quarter: 128 subvectors, four tensor-core products per
// token.  Sb: the round's sign word; B[m][i][h]: the B operands of the round's
// group pair for token m; a4[e][m]: per-row sums (.x, .y = the two groups).
template <int BB, int MT>
__device__ __forceinline__ void frag_round(uint32_t Sb, const uint32_t (&P)[5], const FragK& fk, uint32_t cb_base_q,
                                           const uint32_t (&B)[MT][4][2], float2 scp, float2 ofp,
                                           float2 (&a4)[4][MT]) {
  constexpr int rp = BB & 1;
  uint32_t addr[4];
  float v[4];
  frag_slot<BB, 0>(P, fk, cb_base_q, addr[0], v[0]);
  frag_slot<BB, 1>(P, fk, cb_base_q, addr[1], v[1]);
  frag_slot<BB, 2>(P, fk, cb_base_q, addr[2], v[2]);
  frag_slot<BB, 3>(P, fk, cb_base_q, addr[3], v[3]);
  uint32_t a[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) ldsm_x4(a[i], addr[i]);
  // Sb << (4i + j): Si = Sb << 4i (three independent multiplications), then << j
  const uint32_t Si[4] = {Sb, mul_lo(Sb, fk.m16), mul_lo(Sb, fk.m256), mul_lo(Sb, fk.m4096)};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[i][0] ^= Si[i] & 0x80008000u;
    a[i][1] ^= mul_lo(Si[i], fk.m2) & 0x80008000u;
    a[i][2] ^= mul_lo(Si[i], fk.m4) & 0x80008000u;
    a[i][3] ^= mul_lo(Si[i], fk.m8) & 0x80008000u;
  }
  // radii of this lane's four subvectors: rows 4T+2rp+e, groups 2gp+h (v[2e+h])
  const float r00 = __fmaf_rn(scp.x, v[0], ofp.x), r01 = __fmaf_rn(scp.x, v[1], ofp.x);
  const float r10 = __fmaf_rn(scp.y, v[2], ofp.y), r11 = __fmaf_rn(scp.y, v[3], ofp.y);
  const float zero4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    // two chains of two products (products 0,1 and 2,3 fill disjoint columns),
    // added afterwards: half the dependent tensor-core latency of one chain
    float c[4], e[4];
    mma16816(c, a[0], B[m][0][0], B[m][0][1], zero4);
    mma16816(e, a[2], B[m][2][0], B[m][2][1], zero4);
    mma16816(c, a[1], B[m][1][0], B[m][1][1], c);
    mma16816(e, a[3], B[m][3][0], B[m][3][1], e);
    const float2 d01 = __fadd2_rn(make_float2(c[0], c[1]), make_float2(e[0], e[1]));
    const float2 d23 = __fadd2_rn(make_float2(c[2], c[3]), make_float2(e[2], e[3]));
    a4[2 * rp][m] = __ffma2_rn(make_float2(r00, r01), d01, a4[2 * rp][m]);
    a4[2 * rp + 1][m] = __ffma2_rn(make_float2(r10, r11), d23, a4[2 * rp + 1][m]);
  }
}

// One quarter of a full-tile block (rounds 4A..4A+3, groups 4A..4A+3, all 128
// rows) for MT tokens.  sg: the quarter's sign chunk (chunk 2A of the lane);
// pw, p5: its payload words (chunk 2A+1 and word A of chunk 8); xq: the
// quarter's 32 columns of x in stored order ([MT] rows, stride xstride bytes);
// cb_base_q: shared-window address of the codebook table plus this lane's
// replica offset; bm[i][h]: ~0 when this lane supplies the B operand of
// product i in k-half h, else 0; xw_off: this lane's x word in a group pair;
// acc[rp][m]: (row 4T+2rp, row 4T+2rp+1) sums.
template <int MT>
__device__ __forceinline__ void frag_quarter(uint4 sg, uint4 pw, uint32_t p5, const unsigned char* xq,
                                             int xstride_bytes, uint32_t cb_base_q, const FragK& fk,
                                             const uint32_t (&bm)[4][2], uint32_t xw_off, const float2 (&scp)[2],
                                             const float2 (&ofp)[2], float2 (&acc)[2][MT]) {
  float2 a4[4][MT];
#pragma unroll
  for (int e = 0; e < 4; ++e)
#pragma unroll
    for (int m = 0; m < MT; ++m) a4[e][m] = make_float2(0.f, 0.f);
  const uint32_t P[5] = {pw.x, pw.y, pw.z, pw.w, p5};
  uint32_t B[MT][4][2];
#pragma unroll
  for (int gp = 0; gp < 2; ++gp) {
    // B operands of group pair gp (shared by its two rounds): this lane's x word,
    // kept only in the product and k-half it supplies
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const uint32_t xw = lds32(xq, m * xstride_bytes + 32 * gp + xw_off);
#pragma unroll
      for (int i = 0; i < 4; ++i) { B[m][i][0] = xw & bm[i][0]; B[m][i][1] = xw & bm[i][1]; }
    }
    if (gp == 0) {
      frag_round<0, MT>(sg.x, P, fk, cb_base_q, B, scp[0], ofp[0], a4);
      frag_round<1, MT>(sg.y, P, fk, cb_base_q, B, scp[1], ofp[1], a4);
    } else {
      frag_round<2, MT>(sg.z, P, fk, cb_base_q, B, scp[0], ofp[0], a4);
      frag_round<3, MT>(sg.w, P, fk, cb_base_q, B, scp[1], ofp[1], a4);
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    acc[0][m].x += a4[0][m].x + a4[0][m].y;
    acc[0][m].y += a4[1][m].x + a4[1][m].y;
    acc[1][m].x += a4[2][m].x + a4[2][m].y;
    acc[1][m].y += a4[3][m].x + a4[3][m].y;
  }
}

// A whole full-tile block (four quarters) for MT tokens: d, the lane's 36
// words; xb, the block's 128 columns of x in stored order.
template <int MT>
__device__ __forceinline__ void process_block_frag(const uint4 (&d)[kChunks], const unsigned char* xb,
                                                   int xstride_bytes, uint32_t cb_base_q, const FragK& fk,
                                                   const uint32_t (&bm)[4][2], uint32_t xw_off,
                                                   const float2 (&scp)[2], const float2 (&ofp)[2],
                                                   float2 (&acc)[2][MT]) {
  frag_quarter<MT>(d[0], d[1], d[8].x, xb, xstride_bytes, cb_base_q, fk, bm, xw_off, scp, ofp, acc);
  frag_quarter<MT>(d[2], d[3], d[8].y, xb + 64, xstride_bytes, cb_base_q, fk, bm, xw_off, scp, ofp, acc);
  frag_quarter<MT>(d[4], d[5], d[8].z, xb + 128, xstride_bytes, cb_base_q, fk, bm, xw_off, scp, ofp, acc);
  frag_quarter<MT>(d[6], d[7], d[8].w, xb + 192, xstride_bytes, cb_base_q, fk, bm, xw_off, scp, ofp, acc);
}

}  // namespace
}  // namespace svq
