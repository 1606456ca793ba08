#pragma once
// gemv_device.cuh -- device-side building blocks of the fused SVQ
// decode-and-multiply (shared by the grouped GEMV and the MoE kernels):
// cache-policy loads, lane-block loads and the per-block decode + dot product.
//
// A lane owns 4 rows x 16 subvectors of a block (layout.cuh).  For each
// subvector: idx and radius code come out of the payload word with one shift
// and one mask each; the fp16 codeword is gathered from the lane's replica of
// the shared-memory codebook (conflict free); the subvector's sign bits are
// XORed onto the fp16 sign bits (the shifted sign word puts each pair's two
// signs on bits 15 and 31); the 8 products of fp16 codeword entries and fp16
// activations are accumulated in fp32 with mixed-precision FMAs (each product
// exact in fp32, one rounding per addition) and the radius r = offset + scale *
// code ("SAGE", arXiv 2610.14745, Figure 2 caption: signs, direction index,
// quantized radius) scales the sum in fp32.
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

// acc += a.lo * b.lo + a.hi * b.hi for fp16 pairs a, b: two fp32 FMAs on fp16
// inputs (fma.rn.f32.f16: the product is exact in fp32, one rounding each).
__device__ __forceinline__ void fma_f32_h2(float& acc, uint32_t a, uint32_t b) {
  asm("{\n\t.reg .f16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\t"
      "mov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.f16 %0, al, bl, %0;\n\t"
      "fma.rn.f32.f16 %0, ah, bh, %0;\n\t}"
      : "+f"(acc)
      : "r"(a), "r"(b));
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

// kLut: the radius of row r (of the lane's 4) and code c is the table level
// lut_lane[(c * 4 + r) * 32] (lut_lane = the tile's shared-memory table
// [code][row of lane][lane] plus this lane; conflict free), instead of
// scp * v + ofp.
template <int MT, bool kLut = false>
__device__ __forceinline__ void process_block(const uint4 (&d)[kChunks], const unsigned char* xb,
                                              int xstride_bytes, const unsigned char* cbs, uint32_t q16,
                                              const CbShift& cs, uint32_t CODEM, const float2 (&scp)[2],
                                              const float2 (&ofp)[2], float2 (&acc)[2][MT],
                                              const float* lut_lane = nullptr, int bd = 0) {
  const uint32_t cmask_l = kLut ? (1u << (10 - bd)) - 1u : 0u;
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
    uint32_t cdl[4];                                 // (kLut) radius code of each row
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
        if constexpr (kLut) cdl[r] = (pw >> (bd + 10 * (v % 3))) & cmask_l;
      } else {
        const int a = v - 60;
        const uint32_t pw = ((w[16 + 5 * a] >> 30) << 8) | ((w[17 + 5 * a] >> 30) << 6) |
                            ((w[18 + 5 * a] >> 30) << 4) | ((w[19 + 5 * a] >> 30) << 2) |
                            (w[20 + 5 * a] >> 30);
        ia = (pw << cs.l0) & cs.mask;
        vb = shl<13>(pw) & CODEM;
        if constexpr (kLut) cdl[r] = (pw >> bd) & cmask_l;
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
        float s8 = 0.f;
        fma_f32_h2(s8, cw.x, xv[m].x);
        fma_f32_h2(s8, cw.y, xv[m].y);
        fma_f32_h2(s8, cw.z, xv[m].z);
        fma_f32_h2(s8, cw.w, xv[m].w);
        dsum[r][m] = s8;
      }
    }
    // radius r = scp * v + ofp (or the table level) and accumulation, two rows per packed fp32x2 FMA
    float2 r01, r23;
    if constexpr (kLut) {
      r01 = make_float2(lut_lane[(cdl[0] * 4 + 0) * 32], lut_lane[(cdl[1] * 4 + 1) * 32]);
      r23 = make_float2(lut_lane[(cdl[2] * 4 + 2) * 32], lut_lane[(cdl[3] * 4 + 3) * 32]);
    } else {
      r01 = __ffma2_rn(scp[0], make_float2(vf[0], vf[1]), ofp[0]);
      r23 = __ffma2_rn(scp[1], make_float2(vf[2], vf[3]), ofp[1]);
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      acc[0][m] = __ffma2_rn(r01, make_float2(dsum[0][m], dsum[1][m]), acc[0][m]);
      acc[1][m] = __ffma2_rn(r23, make_float2(dsum[2][m], dsum[3][m]), acc[1][m]);
    }
  }
}

}  // namespace
}  // namespace svq
