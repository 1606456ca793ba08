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
//   * a CTA of 4 warps works on one 128-row tile of one matrix and one k-slice;
//     the warps split the slice's blocks, each lane owns 4 complete rows, so a
//     row's partial sum never leaves its thread in the hot loop; the warps'
//     sums are combined once in shared memory;
//   * packed codes stream from HBM with 16-byte coalesced loads
//     (ld.global.nc.L1::no_allocate), one block (9 loads per lane) ahead;
//   * the fp16 codebook sits in shared memory as 8 replicas, entry e of
//     replica q at 16-byte slot 8e + q, and lane l reads replica l % 8: the 8
//     lanes of each quarter-warp phase of an LDS.128 hit 8 different bank
//     groups whatever the indices, so the random gather is conflict free;
//   * each warp gathers x[perm] for its blocks itself, software-pipelined: the
//     permutation of block b+2 and the activations of block b+1 are loaded
//     while block b is decoded, into the other of two small shared-memory
//     slots that the lanes read with broadcast loads;
//   * signs are applied by XOR on fp16 sign bits; the eight products of a
//     subvector are summed in fp16x2, then scaled by the radius and
//     accumulated across subvectors in fp32;
//   * split-K partials go to the workspace; the last CTA of a tile (found with a
//     counter) sums them in slice order, so results are reproducible.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "layout.cuh"
#include "svq_internal.h"
#include "gemv_params.h"
#include "gemv_device.cuh"

namespace svq {
namespace {

// One CTA = one 128-row tile of one matrix and one k-slice; its warps split the
// k-slice's blocks and their partial sums are combined in shared memory.
template <int MT>
__device__ __forceinline__ void gemv_cta(const GemvKMat& g, int c, unsigned char* smem, int y_f32) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BD = g.b_d, BR = 10 - BD;
  const int R = cb_replicas(BD);
  const CbShift cs = cb_shift(BD);
  const uint32_t CODEM = BR ? (((1u << BR) - 1u) << (23 - BR)) : 0u;
  const int N = g.N, K = g.K, B = K / kBlockCols, S = g.S, M = g.M;
  const int t = c / S, s = c - t * S;
  const int kb0 = (int)(((long long)B * s) / S), kb1 = (int)(((long long)B * (s + 1)) / S);
  const int nbk = kb1 - kb0;
  const int wb0 = kb0 + (nbk * warp) / kGemvWarps, wb1 = kb0 + (nbk * (warp + 1)) / kGemvWarps;
  const int nb = wb1 - wb0;
  const int L = tile_lanes(N, t);
  const bool on = lane < L;
  const int row0 = t * kTileRows + 4 * lane;

  uint4* cbs = reinterpret_cast<uint4*>(smem);
  // Per warp: two x slots (double buffer) of MT rows x 128 columns fp16.
  unsigned char* xs = smem + ((size_t)16 * R << BD) + (size_t)warp * 2 * MT * kBlockCols * 2;
  constexpr int kXSlot = MT * kBlockCols * 2;          // bytes per slot
  float* red = reinterpret_cast<float*>(smem + ((size_t)16 * R << BD) +
                                        (size_t)kGemvWarps * 2 * kXSlot);   // [warps][MT][128]

  const uint8_t* tile_base = g.packed + tile_offset(K, t);
  const size_t blk_bytes = (size_t)L * kLaneBlockBytes;
  const uint64_t pol_stream = policy_evict_first(), pol_keep = policy_evict_last();
  uint4 d0[kChunks], d1[kChunks];
  if (on && nb > 0) load_block(d0, tile_base + (size_t)wb0 * blk_bytes, L, lane, pol_stream);

  // Codebook replicas: thread i fills slot i (entry i / R, replica i % R) with an
  // asynchronous global->shared copy; a warp covers consecutive slots.
  const uint32_t cb_s = (uint32_t)__cvta_generic_to_shared(cbs);
  for (int i = threadIdx.x; i < (R << BD); i += blockDim.x)
    asm volatile("cp.async.ca.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(cb_s + 16u * i),
                 "l"(g.codebook + i / R), "l"(pol_keep)
                 : "memory");
  asm volatile("cp.async.commit_group;" ::: "memory");
  // Radius parameters of this lane's rows and the permutation of the warp's
  // first two blocks (all weights: independent of earlier kernels).
  float sc[4] = {0.f, 0.f, 0.f, 0.f}, of[4] = {0.f, 0.f, 0.f, 0.f};
  if (on) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      sc[r] = __half2float(__ushort_as_half(ldg_keep_u16(g.scale + row0 + r, pol_keep)));
      of[r] = __half2float(__ushort_as_half(ldg_keep_u16(g.offset + row0 + r, pol_keep)));
    }
  }
  // x[perm] pipeline: lane l owns columns l, l+32, l+64, l+96 of a block.  The
  // permutation of block b+2 and the activations of block b+1 are loaded while
  // block b is decoded; the activations land in the other x slot.
  const int32_t* pw = g.perm + (size_t)wb0 * kBlockCols + lane;
  const uint16_t* xg = g.x;
  int pj_a[4], pj_b[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    pj_a[u] = nb > 0 ? ldg_keep_i32(pw + 32 * u, pol_keep) : 0;
    pj_b[u] = nb > 1 ? ldg_keep_i32(pw + kBlockCols + 32 * u, pol_keep) : 0;
  }
  // The activations may be written by the previous kernel in the stream
  // (programmatic dependent launch): wait for it before reading x.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  uint16_t hx[MT][4];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int u = 0; u < 4; ++u) hx[m][u] = (m < M && nb > 0) ? ldg_keep_u16(xg + (size_t)m * K + pj_a[u], pol_keep) : 0;
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int u = 0; u < 4; ++u)
      reinterpret_cast<uint16_t*>(xs + m * kBlockCols * 2)[lane + 32 * u] = hx[m][u];
  // Let the next kernel in the stream start its own weight-only prologue as this
  // grid's CTAs retire.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // Radius r = offset + scale * code, written as r = scp * v + ofp with v = 1 + code * 2^-BR.
  float2 scp[2], ofp[2];
  {
    float sp[4], op[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      if (BR > 0) { sp[r] = sc[r] * (float)(1 << BR); op[r] = of[r] - sp[r]; }
      else { sp[r] = 0.f; op[r] = of[r]; }
    }
    scp[0] = make_float2(sp[0], sp[1]); scp[1] = make_float2(sp[2], sp[3]);
    ofp[0] = make_float2(op[0], op[1]); ofp[1] = make_float2(op[2], op[3]);
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();

  float2 acc[2][MT];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[h][m] = make_float2(0.f, 0.f);

  const unsigned char* cbb = reinterpret_cast<const unsigned char*>(cbs);
  const uint32_t q16 = (uint32_t)(lane % R) * 16;
  for (int b = 0; b < nb; ++b) {
    // activations of block b+1 (permutation already loaded), permutation of block b+2
    if (b + 1 < nb) {
#pragma unroll
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int u = 0; u < 4; ++u) hx[m][u] = m < M ? ldg_keep_u16(xg + (size_t)m * K + pj_b[u], pol_keep) : 0;
      if (b + 2 < nb) {
#pragma unroll
        for (int u = 0; u < 4; ++u) pj_b[u] = ldg_keep_i32(pw + (size_t)(b + 2) * kBlockCols + 32 * u, pol_keep);
      }
    }
    if (on) {
      if (b + 1 < nb) load_block(d1, tile_base + (size_t)(wb0 + b + 1) * blk_bytes, L, lane, pol_stream);
      process_block<MT>(d0, xs + (b & 1) * kXSlot, kBlockCols * 2, cbb, q16, cs, CODEM, scp, ofp, acc);
#pragma unroll
      for (int k = 0; k < kChunks; ++k) d0[k] = d1[k];
    }
    if (b + 1 < nb) {
      __syncwarp();                                   // all lanes done reading the slot about to be reused
      unsigned char* nx = xs + ((b + 1) & 1) * kXSlot;
#pragma unroll
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int u = 0; u < 4; ++u) reinterpret_cast<uint16_t*>(nx + m * kBlockCols * 2)[lane + 32 * u] = hx[m][u];
      __syncwarp();
    }
  }

  // Combine the warps' partial sums of the tile's 128 rows (fixed order).
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    float* rr = red + ((size_t)warp * MT + m) * kTileRows + 4 * lane;
    *reinterpret_cast<float4*>(rr) = make_float4(acc[0][m].x, acc[0][m].y, acc[1][m].x, acc[1][m].y);
  }
  __syncthreads();
  const int rows = L * 4;
  const int nout = rows * M;
  if (S == 1) {
    for (int i = threadIdx.x; i < nout; i += blockDim.x) {
      const int om = i / rows, on_i = i - om * rows;
      float outv = 0.f;
#pragma unroll
      for (int w8 = 0; w8 < kGemvWarps; ++w8) outv += red[((size_t)w8 * MT + om) * kTileRows + on_i];
      const size_t o = (size_t)om * N + t * kTileRows + on_i;
      if (y_f32) reinterpret_cast<float*>(g.y)[o] = outv;
      else reinterpret_cast<__half*>(g.y)[o] = __float2half_rn(outv);
    }
    return;
  }

  // Split-K: write this k-slice's partial, then the last CTA of the tile sums the
  // S partials in slice order.
  for (int i = threadIdx.x; i < nout; i += blockDim.x) {
    const int om = i / rows, on_i = i - om * rows;
    float outv = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < kGemvWarps; ++w8) outv += red[((size_t)w8 * MT + om) * kTileRows + on_i];
    g.partial[((size_t)s * M + om) * N + t * kTileRows + on_i] = outv;
  }
  __threadfence();
  __syncthreads();
  __shared__ int s_last;
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(&g.counters[t], 1u);
    s_last = (prev == (unsigned)(S - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int i = threadIdx.x; i < nout; i += blockDim.x) {
    const int om = i / rows, n = t * kTileRows + (i - om * rows);
    float sum = 0.f;
    int k = 0;
    for (; k + 8 <= S; k += 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldcg(g.partial + ((size_t)(k + u) * M + om) * N + n);
#pragma unroll
      for (int u = 0; u < 8; ++u) sum += v[u];
    }
    for (; k < S; ++k) sum += __ldcg(g.partial + ((size_t)k * M + om) * N + n);
    const size_t o = (size_t)om * N + n;
    if (y_f32) reinterpret_cast<float*>(g.y)[o] = sum;
    else reinterpret_cast<__half*>(g.y)[o] = __float2half_rn(sum);
  }
  if (threadIdx.x == 0) g.counters[t] = 0u;
}

template <int MT>
__global__ void __launch_bounds__(kGemvWarps * 32, MT <= 2 ? 4 : 2)
gemv_kernel(const __grid_constant__ GemvKParams P) {
  extern __shared__ __align__(1024) unsigned char smem[];
  int mi = 0;
  while (mi + 1 < P.n_mats && (int)blockIdx.x >= P.mats[mi + 1].cta_begin) ++mi;
  const GemvKMat& g = P.mats[mi];
  const int c = (int)blockIdx.x - g.cta_begin;
  gemv_cta<MT>(g, c, smem, P.y_f32);
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
  // Programmatic dependent launch: the kernel's weight-only prologue may overlap
  // the tail of the previous kernel in the stream (it waits for that kernel
  // before reading x).
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kGemvWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gemv_kernel<MT>, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace svq
