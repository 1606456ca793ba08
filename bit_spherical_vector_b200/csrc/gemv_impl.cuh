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
//   * one CTA per SM; each matrix of the group gets SMs in proportion to its
//     blocks, and each CTA a contiguous range of the matrix's blocks (128-row
//     tile x 128 columns, in storage order, crossing tile boundaries), so all
//     SMs stream about the same number of bytes;
//   * the warps of a CTA split its range contiguously again; each lane owns 4
//     complete rows of the current tile, so a row's partial sum never leaves
//     its thread in the hot loop;
//   * packed codes stream from HBM with 16-byte coalesced loads
//     (ld.global.nc.L1::no_allocate, L2 evict-first), one block (9 loads per
//     lane) ahead of the decode;
//   * the fp16 codebook sits in shared memory as 8 replicas (4 for 1024
//     entries), entry e of replica q at 16-byte slot 8e + q, and lane l reads
//     replica l % 8: the 8 lanes of each quarter-warp phase of an LDS.128 hit 8
//     different bank groups whatever the indices, so the random gather is
//     conflict free;
//   * each warp gathers x[perm] for its blocks itself, software-pipelined: the
//     permutation of block b+2 and the activations of block b+1 are loaded
//     while block b is decoded, into the other of two small shared-memory
//     slots that the lanes read with broadcast loads;
//   * signs are applied by XOR on fp16 sign bits; the eight products of a
//     subvector (fp16 codeword entries times fp16 activations, each exact in
//     fp32) are accumulated in fp32 by mixed-precision FMAs, then scaled by
//     the radius and accumulated across subvectors in fp32;
//   * when a warp's range leaves a tile it parks that tile's sums in shared
//     memory; the last warp of the CTA to leave the tile (a shared-memory
//     counter) adds the parked sums in range order, so tiles complete while
//     other warps still decode; a tile shared by several CTAs goes through the
//     workspace, where the last CTA to finish it (a global counter) adds the
//     slots in CTA order, so results are reproducible.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>

#include "layout.cuh"
#include "svq_internal.h"
#include "gemv_params.h"
#include "gemv_device.cuh"

namespace svq {
namespace {

__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Called by a whole warp after it parked its sums of tile t.  The last warp of
// the CTA to do so adds the parked sums of every warp range touching t in range
// order (rb: the CTA's W + 1 range boundaries, then each range's first tile); a
// tile that lies wholly in the CTA's range goes to y, a tile shared by CTAs
// c0..c1 to its workspace slot (k = c - c0), and the last CTA to deposit a slot
// adds all slots in CTA order.  Kept out of line: it
// runs once or twice per warp, and inlining it would cost the hot loop registers.
template <int MT>
__device__ __noinline__ void tile_piece_done(const GemvKMat& g, int c, int t, const float* red, int* tcnt,
                                             const int* rb, int ta, bool whole, long long G, long long T,
                                             int npw, int y_f32, int lane) {
  constexpr int W = gemv_warps(MT);
  const int N = g.N, B = pad_cols(g.K) / kBlockCols, M = g.M;   // blocks of the padded layout
  const int tq0 = t * B, tq1 = tq0 + B;               // blocks of tile t
  __threadfence_block();
  __syncwarp();
  // ranges r_lo..r_hi (consecutive) touch tile t; empty ranges (only when the
  // CTA has fewer blocks than warps) touch nothing
  int r_lo = W, r_hi = -1, touching = 0;
#pragma unroll
  for (int r = 0; r < W; ++r) {
    const bool tr = rb[r] < rb[r + 1] && rb[r] < tq1 && rb[r + 1] > tq0;
    touching += tr ? 1 : 0;
    if (tr) { r_lo = min(r_lo, r); r_hi = r; }
  }
  int last = 0;
  if (lane == 0) last = atomicAdd(&tcnt[t - ta], 1) == touching - 1;
  if (!__shfl_sync(0xFFFFFFFFu, last, 0)) return;
  __threadfence_block();
  float4 v[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) v[m] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int r = r_lo; r <= r_hi; ++r) {
    if (rb[r] == rb[r + 1]) continue;
    const float* src = red + ((size_t)r * npw + (t - rb[W + 1 + r])) * MT * kTileRows + 4 * lane;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float4 u = *reinterpret_cast<const float4*>(src + m * kTileRows);
      v[m].x += u.x; v[m].y += u.y; v[m].z += u.z; v[m].w += u.w;
    }
  }
  auto write_y = [&]() {
    const int n0 = t * kTileRows + 4 * lane;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m >= M) break;
      const float vv[4] = {v[m].x, v[m].y, v[m].z, v[m].w};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (n0 + r >= N) break;                        // padding rows of a ragged N
        const size_t o = (size_t)m * N + n0 + r;
        if (y_f32) reinterpret_cast<float*>(g.y)[o] = vv[r];
        else reinterpret_cast<__half*>(g.y)[o] = __float2half_rn(vv[r]);
      }
    }
  };
  const bool in_tile = lane < tile_lanes(pad_rows(N), t);
  if (whole) {                                         // the tile lies wholly in this CTA's range
    if (in_tile) write_y();
    return;
  }
  // CTAs c0..c1 share tile t (CTA of block q: ((q + 1) G - 1) / T)
  const int c0 = (int)((((long long)t * B + 1) * G - 1) / T);
  const int c1 = (int)((((long long)(t + 1) * B) * G - 1) / T);
  float* slots = g.partial + (size_t)t * g.kmax * MT * kTileRows + 4 * lane;
  if (in_tile) {
#pragma unroll
    for (int m = 0; m < MT; ++m)
      *reinterpret_cast<float4*>(slots + ((size_t)(c - c0) * MT + m) * kTileRows) = v[m];
  }
  // Hand-off: the counter increment has acquire-release semantics at GPU scope,
  // so this warp's slot stores (ordered before it by __syncwarp) are visible to
  // the CTA that sees the final count, and that CTA sees every earlier slot.
  __syncwarp();
  int glast = 0;
  if (lane == 0) glast = atom_add_acq_rel_gpu(&g.counters[t], 1u) == (unsigned)(c1 - c0);
  if (!__shfl_sync(0xFFFFFFFFu, glast, 0)) return;
  __syncwarp();                                        // the other lanes read after lane 0's acquire
#pragma unroll
  for (int m = 0; m < MT; ++m) v[m] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (in_tile) {
    for (int k = 0; k <= c1 - c0; ++k) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const float4 u = __ldcg(reinterpret_cast<const float4*>(slots + ((size_t)k * MT + m) * kTileRows));
        v[m].x += u.x; v[m].y += u.y; v[m].z += u.z; v[m].w += u.w;
      }
    }
    write_y();
  }
  if (lane == 0) g.counters[t] = 0u;
}

// One CTA = one contiguous range of one matrix's blocks.  kPerm: the matrix has
// a permutation (x is gathered through it); without one, x is already in stored
// column order and lane l reads columns l, l+32, l+64, l+96 of each block.
// kLut: the matrix carries a per-row radius table (g.lut): the levels of the
// CTA's row tiles are staged in shared memory by the prologue.
template <int MT, bool kPerm, bool kLut>
__device__ __forceinline__ void gemv_cta(const GemvKMat& g, int c, unsigned char* smem, int y_f32) {
  constexpr int W = gemv_warps(MT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BD = g.b_d, BR = 10 - BD;
  const int R = gemv_cb_replicas(BD);
  const CbShift cs = cb_shift(BD, R);
  const uint32_t CODEM = BR ? (((1u << BR) - 1u) << (23 - BR)) : 0u;
  // N, K: the matrix; Np, Kp: its (padded) layout -- columns >= K read x as 0,
  // rows >= N are computed but never written
  const int N = g.N, K = g.K, Np = pad_rows(N), Kp = pad_cols(K), B = Kp / kBlockCols, M = g.M, npw = g.npw;
  const long long T = (long long)num_tiles(Np) * B, G = g.ctas;
  // this CTA's blocks [qa, qb) and this warp's blocks [wq0, wq0 + nb)
  const int qa = (int)(c * T / G), qb = (int)((c + 1) * T / G);
  const int n = qb - qa;
  // Warp ranges: range r covers [qa + n*r/W, qa + n*(r+1)/W).  Warp w takes range
  // wr = (w % 4) * (W / 4) + w / 4, so the warps of one SM sub-partition (w, w+4,
  // ...) hold consecutive ranges and each sub-partition issues a quarter of the
  // CTA's blocks (ranges of 2 and 3 blocks would otherwise pile up on one).
  auto range_begin = [&](int r) -> int { return qa + (int)((long long)n * r / W); };
  const int wr = (warp & 3) * (W / 4) + (warp >> 2);
  const int wq0 = range_begin(wr);
  const int nb = range_begin(wr + 1) - wq0;
  const int ta = qa / B, tb = (qb - 1) / B;

  // The CTA's last tile is shared with the next CTA when the range ends inside
  // it; warps whose range reaches into it walk their range backwards, so that
  // tile's sums are complete early and its cross-CTA hand-off overlaps the rest
  // of the decode instead of trailing it.
  const bool first_shared = (long long)ta * B < qa, last_shared = (long long)(tb + 1) * B > qb;
  const bool rev = nb > 0 && last_shared && (wq0 + nb - 1) / B == tb && !(first_shared && wq0 / B == ta);
  auto q_of = [&](int b) -> int { return rev ? wq0 + nb - 1 - b : wq0 + b; };
  const int t_first = nb > 0 ? wq0 / B : 0;           // piece p of the range holds tile t_first + p

  uint4* cbs = reinterpret_cast<uint4*>(smem);
  // Per warp: two x slots (double buffer) of MT rows x 128 columns fp16.
  constexpr int kXSlot = MT * kBlockCols * 2;          // bytes per x slot
  unsigned char* xs = smem + ((size_t)16 * R << BD) + (size_t)warp * 2 * kXSlot;
  // [W][npw][MT][128]: each warp range's sums for each tile it touches, then the
  // W + 1 range boundaries and the W ranges' first tiles (36 ints), then one
  // completion counter per tile of the range
  float* red = reinterpret_cast<float*>(smem + ((size_t)16 * R << BD) + (size_t)W * 2 * kXSlot);
  int* rbt = reinterpret_cast<int*>(red + (size_t)W * npw * MT * kTileRows);
  int* tcnt = rbt + 36;
  // (kLut) radius levels of tiles ta..tb as fp32, [tile][code][row of lane][lane]
  float* lutsm = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(tcnt) +
                                          ((size_t)(tb - ta + 1) * 4 + 15) / 16 * 16);
  for (int i = threadIdx.x; i <= tb - ta; i += blockDim.x) tcnt[i] = 0;
  if (threadIdx.x <= W) rbt[threadIdx.x] = range_begin(threadIdx.x);
  if (threadIdx.x < W) rbt[W + 1 + threadIdx.x] = range_begin(threadIdx.x) / B;   // first tile of range

  const uint64_t pol_stream = policy_evict_first(), pol_keep = policy_evict_last();
  auto block_ptr = [&](int q, int L) -> const uint8_t* {
    const int t = q / B, kb = q - t * B;
    return g.packed + tile_offset(Kp, t) + (size_t)kb * L * kLaneBlockBytes;
  };
  // x index of this lane's columns of block q (lane + 32u): perm[col], or col;
  // -1 for padding columns (col >= K), whose activations read as zero
  auto load_pj = [&](int q, int (&pj)[4]) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int col = (q % B) * kBlockCols + lane + 32 * u;
      if constexpr (kPerm) pj[u] = col < K ? ldg_keep_i32(g.perm + col, pol_keep) : -1;
      else pj[u] = col < K ? col : -1;
    }
  };
  auto x_at = [&](int m, int pj) -> uint16_t {
    return (m < M && pj >= 0) ? ldg_keep_u16(g.x + (size_t)m * K + pj, pol_keep) : (uint16_t)0;
  };

  int t_cur = nb > 0 ? q_of(0) / B : 0;
  int L_cur = tile_lanes(Np, t_cur);
  uint4 d0[kChunks], d1[kChunks];
  if (nb > 0 && lane < L_cur) load_block(d0, block_ptr(q_of(0), L_cur), L_cur, lane, pol_stream);

  // Codebook: each entry is read from global memory once (up to 4 entries per
  // thread, loads kept in flight through the prologue) and written to its R
  // replica slots e*R + q after the dependency wait.
  constexpr int kCbPer = 4;                            // 1024 entries / 256+ threads
  uint4 cbv[kCbPer];
#pragma unroll
  for (int k = 0; k < kCbPer; ++k) {
    const int e = threadIdx.x + k * blockDim.x;
    if (e < (1 << BD)) cbv[k] = ldg_keep_v4(g.codebook + e, pol_keep);
  }
  // Radius parameters of this lane's rows of the first tile and the permutation
  // of the warp's first two blocks (all weights: independent of earlier kernels).
  // (kept as raw fp16 bits until they are needed, so the loads stay in flight
  // through the rest of the prologue)
  uint16_t sc[4] = {0, 0, 0, 0}, of[4] = {0, 0, 0, 0};
  if constexpr (kLut) {
    // the per-row radius tables of the CTA's tiles: eight loads in flight per
    // thread before their stores (weights: read before the dependency wait)
    const int nrl = 1 << BR, per_tile = kTileRows << BR, total = (tb - ta + 1) * per_tile;
    for (int i0 = threadIdx.x; i0 < total; i0 += 8 * blockDim.x) {
      uint16_t hv[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int i = i0 + k * blockDim.x;
        const int tt = i / per_tile, rem = i - tt * per_tile;
        const int n = (ta + tt) * kTileRows + (rem >> BR);
        hv[k] = (i < total && n < N) ? ldg_keep_u16(g.lut + (size_t)n * nrl + (rem & (nrl - 1)), pol_keep)
                                     : (uint16_t)0;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int i = i0 + k * blockDim.x;
        if (i >= total) break;
        const int tt = i / per_tile, rem = i - tt * per_tile;
        const int row = rem >> BR, code = rem & (nrl - 1);
        lutsm[((tt * nrl + code) * 4 + (row & 3)) * 32 + (row >> 2)] = __half2float(__ushort_as_half(hv[k]));
      }
    }
  }
  if (!kLut && nb > 0 && lane < L_cur) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int n = t_cur * kTileRows + 4 * lane + r;
      sc[r] = n < N ? ldg_keep_u16(g.scale + n, pol_keep) : (uint16_t)0;
      of[r] = n < N ? ldg_keep_u16(g.offset + n, pol_keep) : (uint16_t)0;
    }
  }
  // x[perm] pipeline: lane l owns columns l, l+32, l+64, l+96 of a block.  The
  // permutation of block b+2 and the activations of block b+1 are loaded while
  // block b is decoded; the activations land in the other x slot.
  int pj_a[4] = {-1, -1, -1, -1}, pj_b[4] = {-1, -1, -1, -1};
  if (nb > 0) load_pj(q_of(0), pj_a);
  if (nb > 1) load_pj(q_of(1), pj_b);
  // The activations may be written by the previous kernel in the stream
  // (programmatic dependent launch): wait for it before reading x.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  uint16_t hx[MT][4];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int u = 0; u < 4; ++u) hx[m][u] = x_at(m, pj_a[u]);
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
  auto radius_pairs = [&](const uint16_t (&s4)[4], const uint16_t (&o4)[4]) {
    float sp[4], op[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float sf = __half2float(__ushort_as_half(s4[r])), of_ = __half2float(__ushort_as_half(o4[r]));
      if (BR > 0) { sp[r] = sf * (float)(1 << BR); op[r] = of_ - sp[r]; }
      else { sp[r] = 0.f; op[r] = of_; }
    }
    scp[0] = make_float2(sp[0], sp[1]); scp[1] = make_float2(sp[2], sp[3]);
    ofp[0] = make_float2(op[0], op[1]); ofp[1] = make_float2(op[2], op[3]);
  };
  radius_pairs(sc, of);
#pragma unroll
  for (int k = 0; k < kCbPer; ++k) {
    const int e = threadIdx.x + k * blockDim.x;
    // thread e writes its replicas in the order (q + e) % R, so the eight
    // threads of a store phase hit eight different bank groups
    if (e < (1 << BD))
      for (int q = 0; q < R; ++q) cbs[e * R + ((q + e) & (R - 1))] = cbv[k];
  }
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
        for (int u = 0; u < 4; ++u) hx[m][u] = x_at(m, pj_b[u]);
      if (b + 2 < nb) load_pj(q_of(b + 2), pj_b);
    }
    // packed codes of block b+1, and the radius parameters of its tile if it is a new one
    int t_next = t_cur, L_next = L_cur;
    if (b + 1 < nb) {
      const int qn = q_of(b + 1);
      t_next = qn / B;
      L_next = tile_lanes(Np, t_next);
      if (lane < L_next) {
        load_block(d1, block_ptr(qn, L_next), L_next, lane, pol_stream);
        if (!kLut && t_next != t_cur) {
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int n = t_next * kTileRows + 4 * lane + r;
            sc[r] = n < N ? ldg_keep_u16(g.scale + n, pol_keep) : (uint16_t)0;
            of[r] = n < N ? ldg_keep_u16(g.offset + n, pol_keep) : (uint16_t)0;
          }
        }
      }
    }
    if (lane < L_cur)
      process_block<MT, kLut>(d0, xs + (b & 1) * kXSlot, kBlockCols * 2, cbb, q16, cs, CODEM, scp, ofp, acc,
                              lutsm + ((size_t)(t_cur - ta) << BR) * kTileRows + lane, BD);
#pragma unroll
    for (int k = 0; k < kChunks; ++k) d0[k] = d1[k];
    if (b + 1 == nb || t_next != t_cur) {
      // the warp leaves tile t_cur: park its sums (lanes beyond the tile park zeros)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        float* rr = red + (((size_t)wr * npw + (t_cur - t_first)) * MT + m) * kTileRows + 4 * lane;
        *reinterpret_cast<float4*>(rr) = make_float4(acc[0][m].x, acc[0][m].y, acc[1][m].x, acc[1][m].y);
        acc[0][m] = make_float2(0.f, 0.f);
        acc[1][m] = make_float2(0.f, 0.f);
      }
      const bool whole = t_cur * B >= qa && (t_cur + 1) * B <= qb;
      tile_piece_done<MT>(g, c, t_cur, red, tcnt, rbt, ta, whole, G, T, npw, y_f32, lane);
      if (b + 1 < nb) {
        t_cur = t_next;
        L_cur = L_next;
        radius_pairs(sc, of);
      }
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
}

// PM: 1 = every matrix of the launch has a permutation, 0 = none has, 2 = mixed
// (each CTA follows its own matrix).  The uniform cases get kernels of their own
// so each is compiled (registers, schedule) for one path only.
// LM: every matrix of the launch carries a per-row radius table (or none does).
template <int MT, int PM, bool LM>
__global__ void __launch_bounds__(gemv_warps(MT) * 32, 1)
gemv_kernel(const __grid_constant__ GemvKParams P) {
  extern __shared__ __align__(1024) unsigned char smem[];
  int mi = 0;
  while (mi + 1 < P.n_mats && (int)blockIdx.x >= P.mats[mi + 1].cta_begin) ++mi;
  const GemvKMat& g = P.mats[mi];
  const int c = (int)blockIdx.x - g.cta_begin;
  if constexpr (PM == 1) {
    gemv_cta<MT, true, LM>(g, c, smem, P.y_f32);
  } else if constexpr (PM == 0) {
    gemv_cta<MT, false, LM>(g, c, smem, P.y_f32);
  } else {
    if (g.perm) gemv_cta<MT, true, LM>(g, c, smem, P.y_f32);
    else gemv_cta<MT, false, LM>(g, c, smem, P.y_f32);
  }
}

template <int MT, int PM, bool LM>
cudaError_t launch_gemv_pm(const GemvKParams& p, int grid, size_t smem, cudaStream_t st) {
  static std::atomic<unsigned long long> attr_set{0};   // one bit per device (setting it twice is harmless)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !((attr_set.load(std::memory_order_acquire) >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(gemv_kernel<MT, PM, LM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kGemvSmemMax);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set.fetch_or(1ull << dev, std::memory_order_release);
  }
  // Programmatic dependent launch: the kernel's weight-only prologue may overlap
  // the tail of the previous kernel in the stream (it waits for that kernel
  // before reading x).
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(gemv_warps(MT) * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gemv_kernel<MT, PM, LM>, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

template <int MT, bool LM>
cudaError_t launch_gemv_lm(const GemvKParams& p, int grid, size_t smem, cudaStream_t st) {
  int with = 0;
  for (int i = 0; i < p.n_mats; ++i) with += p.mats[i].perm != nullptr;
  if (with == p.n_mats) return launch_gemv_pm<MT, 1, LM>(p, grid, smem, st);
  if (with == 0) return launch_gemv_pm<MT, 0, LM>(p, grid, smem, st);
  return launch_gemv_pm<MT, 2, LM>(p, grid, smem, st);
}

template <int MT>
cudaError_t launch_gemv_mt(const GemvKParams& p, int grid, size_t smem, cudaStream_t st) {
  int with = 0;
  for (int i = 0; i < p.n_mats; ++i) with += p.mats[i].lut != nullptr;
  if (with == p.n_mats) return launch_gemv_lm<MT, true>(p, grid, smem, st);
  if (with == 0) return launch_gemv_lm<MT, false>(p, grid, smem, st);
  return cudaErrorInvalidValue;                        // mixed: refused by the planner already
}

}  // namespace svq
