#pragma once
// gemv_impl.cuh -- fused SVQ decode-and-multiply kernel for small batches (1..8 tokens per
// pass), y = W x[perm], over a group of up to eight independent matrices in one
// launch.
//
// Method ("SAGE", arXiv 2610.14745): a subvector of eight weights is
// r * sign (.) c_idx (Figure 2 caption: signs, direction index, quantized
// radius); it multiplies eight reordered activations x[perm[8g..8g+7]]
// (Figure 6 caption); weights are reconstructed on demand, never stored dense
// (Figures 1 and 5).
//
// B200 mapping:
//   * a CTA of 8 warps works on one matrix, one k-slice and up to 8 row tiles;
//     each warp owns a 128-row tile and each lane owns 4 complete rows, so a
//     row's partial sum never leaves its thread (no shuffles in the hot loop);
//   * packed codes stream from HBM with 16-byte coalesced loads
//     (ld.global.nc.L1::no_allocate), one block (9 loads per lane) ahead;
//   * the fp16 codebook sits in shared memory as 8 replicas, entry e of
//     replica q at 16-byte slot 8e + q, and lane l reads replica l % 8: the 8
//     lanes of each quarter-warp phase of an LDS.128 hit 8 different bank
//     groups whatever the indices, so the random gather is conflict free;
//   * x[perm] for the CTA's k-slice is gathered into shared memory once and
//     read with broadcast loads;
//   * signs are applied by XOR on fp16 sign bits; the eight products of a
//     subvector are summed in fp16x2, then scaled by the radius and
//     accumulated across subvectors in fp32;
//   * split-K partials go to the workspace; the last CTA of a row chunk (found
//     with a counter) sums them in a fixed order, so results are reproducible.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "layout.cuh"
#include "svq_internal.h"
#include "gemv_params.h"

namespace svq {
namespace {

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
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

__device__ __forceinline__ void load_block(uint4 (&d)[kChunks], const uint8_t* blk, int L, int lane) {
#pragma unroll
  for (int c = 0; c < kChunks; ++c) d[c] = ldg_stream(blk + ((size_t)c * L + lane) * 16);
}

template <int BD, int MT>
__device__ __forceinline__ void process_block(const uint4 (&d)[kChunks], const unsigned char* xb,
                                              int xstride_bytes, const unsigned char* cbq, const float (&scp)[4], const float (&ofp)[4],
                                              float (&acc)[4][MT]) {
  constexpr int BR = 10 - BD;
  constexpr uint32_t IDX7 = ((1u << BD) - 1u) << 7;
  constexpr uint32_t CODEM = BR ? (((1u << BR) - 1u) << (23 - BR)) : 0u;
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
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int v = 4 * j + r;
      uint32_t ia, vb;
      if (v < 60) {
        const uint32_t pw = w[16 + v / 3];
        switch (v % 3) {
          case 0: ia = shl<7>(pw) & IDX7; vb = shl<13>(pw) & CODEM; break;
          case 1: ia = shl<-3>(pw) & IDX7; vb = shl<3>(pw) & CODEM; break;
          default: ia = shl<-13>(pw) & IDX7; vb = shl<-7>(pw) & CODEM; break;
        }
      } else {
        const int a = v - 60;
        const uint32_t pw = ((w[16 + 5 * a] >> 30) << 8) | ((w[17 + 5 * a] >> 30) << 6) |
                            ((w[18 + 5 * a] >> 30) << 4) | ((w[19 + 5 * a] >> 30) << 2) |
                            (w[20 + 5 * a] >> 30);
        ia = shl<7>(pw) & IDX7;
        vb = shl<13>(pw) & CODEM;
      }
      uint4 cw = lds128(cbq, ia);
      const float vf = __uint_as_float(vb | 0x3F800000u);     // 1 + code * 2^-BR
      cw.x ^= (S << (4 * r + 0)) & 0x80008000u;
      cw.y ^= (S << (4 * r + 1)) & 0x80008000u;
      cw.z ^= (S << (4 * r + 2)) & 0x80008000u;
      cw.w ^= (S << (4 * r + 3)) & 0x80008000u;
      const float rr = fmaf(scp[r], vf, ofp[r]);
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        __half2 p = __hmul2(as_h2(cw.x), as_h2(xv[m].x));
        p = __hfma2(as_h2(cw.y), as_h2(xv[m].y), p);
        p = __hfma2(as_h2(cw.z), as_h2(xv[m].z), p);
        p = __hfma2(as_h2(cw.w), as_h2(xv[m].w), p);
        const float dsum = __low2float(p) + __high2float(p);
        acc[r][m] = fmaf(rr, dsum, acc[r][m]);
      }
    }
  }
}

template <int BD, int MT>
__device__ __forceinline__ void gemv_cta(const GemvKMat& g, int c, unsigned char* smem, int y_f32) {
  constexpr int BR = 10 - BD;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = g.N, K = g.K, B = K / kBlockCols;
  const int s = c % g.S, rc = c / g.S;
  const int b0 = (int)(((long long)B * s) / g.S), b1 = (int)(((long long)B * (s + 1)) / g.S);
  const int nb = b1 - b0, ncols = nb * kBlockCols;
  const int t = rc * kGemvWarps + warp;
  const int L = (t < num_tiles(N)) ? tile_lanes(N, t) : 0;
  const bool on = lane < L;
  const int row0 = t * kTileRows + 4 * lane;

  uint4* cbs = reinterpret_cast<uint4*>(smem);
  unsigned char* xs = smem + ((size_t)16 << BD) * 8;

  const uint8_t* tile_base = g.packed + (on ? tile_offset(K, t) : 0);
  const size_t blk_bytes = (size_t)L * kLaneBlockBytes;

  uint4 d0[kChunks], d1[kChunks];
  if (on && nb > 0) load_block(d0, tile_base + (size_t)b0 * blk_bytes, L, lane);

  // Codebook replicas: entry e, replica q -> 16-byte slot 8e + q.
  for (int i = threadIdx.x; i < (8 << BD); i += blockDim.x) cbs[i] = __ldg(g.codebook + (i >> 3));
  // x[perm] for this k-slice, token-major, zero for tokens >= M.
  const __half* xh = reinterpret_cast<const __half*>(g.x);
  __half* xsh = reinterpret_cast<__half*>(xs);
  for (int i = threadIdx.x; i < MT * ncols; i += blockDim.x) {
    const int m = i / ncols, j = i - m * ncols;
    __half v = __ushort_as_half(0);
    if (m < g.M) v = xh[(size_t)m * K + __ldg(g.perm + (size_t)b0 * kBlockCols + j)];
    xsh[i] = v;
  }
  // Radius r = offset + scale * code, written as r = scp * v + ofp with v = 1 + code * 2^-BR.
  float scp[4], ofp[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    float sc = 0.f, of = 0.f;
    if (on) {
      sc = __half2float(__ushort_as_half(g.scale[row0 + r]));
      of = __half2float(__ushort_as_half(g.offset[row0 + r]));
    }
    if (BR > 0) { scp[r] = sc * (float)(1 << BR); ofp[r] = of - scp[r]; }
    else { scp[r] = 0.f; ofp[r] = of; }
  }
  __syncthreads();

  float acc[4][MT];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[r][m] = 0.f;

  const unsigned char* cbq = reinterpret_cast<const unsigned char*>(cbs) + (lane & 7) * 16;
  const unsigned char* xbase = xs;
  const int xstride = ncols * 2;
  if (on) {
    int b = 0;
    for (; b + 1 < nb; b += 2) {
      load_block(d1, tile_base + (size_t)(b0 + b + 1) * blk_bytes, L, lane);
      process_block<BD, MT>(d0, xbase + b * kBlockCols * 2, xstride, cbq, scp, ofp, acc);
      if (b + 2 < nb) load_block(d0, tile_base + (size_t)(b0 + b + 2) * blk_bytes, L, lane);
      process_block<BD, MT>(d1, xbase + (b + 1) * kBlockCols * 2, xstride, cbq, scp, ofp, acc);
    }
    if (b < nb) process_block<BD, MT>(d0, xbase + b * kBlockCols * 2, xstride, cbq, scp, ofp, acc);
  }

  const int M = g.M;
  if (g.S == 1) {
    if (on) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m >= M) break;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const size_t o = (size_t)m * N + row0 + r;
          if (y_f32) reinterpret_cast<float*>(g.y)[o] = acc[r][m];
          else reinterpret_cast<__half*>(g.y)[o] = __float2half_rn(acc[r][m]);
        }
      }
    }
    return;
  }

  // Split-K: write partials, then the last CTA of this row chunk reduces them.
  if (on) {
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m >= M) break;
#pragma unroll
      for (int r = 0; r < 4; ++r) g.partial[((size_t)s * M + m) * N + row0 + r] = acc[r][m];
    }
  }
  __threadfence();
  __syncthreads();
  __shared__ int s_last;
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(&g.counters[rc], 1u);
    s_last = (prev == (unsigned)(g.S - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int rbeg = rc * kGemvWarps * kTileRows;
  const int rows = min(N - rbeg, kGemvWarps * kTileRows);
  for (int i = threadIdx.x; i < rows * M; i += blockDim.x) {
    const int m = i / rows, n = rbeg + (i - m * rows);
    float sum = 0.f;
    for (int k = 0; k < g.S; ++k) sum += __ldcg(g.partial + ((size_t)k * M + m) * N + n);
    const size_t o = (size_t)m * N + n;
    if (y_f32) reinterpret_cast<float*>(g.y)[o] = sum;
    else reinterpret_cast<__half*>(g.y)[o] = __float2half_rn(sum);
  }
  if (threadIdx.x == 0) g.counters[rc] = 0u;
}

template <int MT>
__global__ void __launch_bounds__(kGemvWarps * 32, MT <= 2 ? 2 : 1)
gemv_kernel(const __grid_constant__ GemvKParams P) {
  extern __shared__ __align__(1024) unsigned char smem[];
  int mi = 0;
  while (mi + 1 < P.n_mats && (int)blockIdx.x >= P.mats[mi + 1].cta_begin) ++mi;
  const GemvKMat& g = P.mats[mi];
  const int c = (int)blockIdx.x - g.cta_begin;
  switch (g.b_d) {
    case 1: gemv_cta<1, MT>(g, c, smem, P.y_f32); break;
    case 2: gemv_cta<2, MT>(g, c, smem, P.y_f32); break;
    case 3: gemv_cta<3, MT>(g, c, smem, P.y_f32); break;
    case 4: gemv_cta<4, MT>(g, c, smem, P.y_f32); break;
    case 5: gemv_cta<5, MT>(g, c, smem, P.y_f32); break;
    case 6: gemv_cta<6, MT>(g, c, smem, P.y_f32); break;
    case 7: gemv_cta<7, MT>(g, c, smem, P.y_f32); break;
    case 8: gemv_cta<8, MT>(g, c, smem, P.y_f32); break;
    case 9: gemv_cta<9, MT>(g, c, smem, P.y_f32); break;
    default: gemv_cta<10, MT>(g, c, smem, P.y_f32); break;
  }
}

}  // namespace

template <int MT>
cudaError_t launch_gemv_mt(const GemvKParams& p, int grid, size_t smem, cudaStream_t st) {
  static unsigned long long attr_set = 0;       // one bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !((attr_set >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(gemv_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kGemvSmemMax);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set |= 1ull << dev;
  }
  gemv_kernel<MT><<<grid, kGemvWarps * 32, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace svq
