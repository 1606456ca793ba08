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
//     work, and each CTA a contiguous range of the matrix's units (a quarter
//     block -- 128 rows x 4 subvector groups -- in full tiles, a whole block in
//     a partial last tile), in storage order and crossing tile boundaries, so
//     all SMs stream about the same number of bytes;
//   * the warps of a CTA split its range contiguously again; in a full tile
//     lane T accumulates rows 4T..4T+3, so a row's partial sum never leaves its
//     thread in the hot loop;
//   * packed codes stream from HBM with 16-byte coalesced loads
//     (ld.global.nc.L1::no_allocate, L2 evict-first), one unit ahead of the
//     decode, plus an L2 prefetch of the next block;
//   * the fp16 codebook sits in shared memory as 8 replicas (4 for 1024
//     entries), entry e of replica q at 16-byte slot 8e + q; ldmatrix gathers
//     the codewords straight into tensor-core A fragments, the eight lanes of
//     each 8x8 matrix reading eight different replicas (conflict free);
//   * signs are applied by XOR on the fp16 sign bits of the A fragments, the
//     eight-element dot products run as mma.m16n8k16 with fp32 accumulation,
//     and each product is scaled by its radius and accumulated in fp32
//     (gemv_device.cuh, fragment decode);
//   * x: staged in shared memory by the prologue, either in stored order as
//     well (the decode reads its B operands from there) or in natural order
//     only, each warp then gathering x[perm] for its next unit into a small
//     double-buffered slot while it decodes the current one;
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
#include <type_traits>

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

// Work units of a matrix: a quarter block (rounds 4A..4A+3: 128 rows x 4
// groups) in the full 128-row tiles, a whole block in a partial last tile.
// Units are numbered tile by tile, block by block, quarter by quarter; the CTAs
// of a matrix take contiguous unit ranges, the warps of a CTA contiguous
// sub-ranges.
struct Units {
  int B, full_tiles, ufull, U;
  __device__ __forceinline__ int tile_u0(int t) const { return t < full_tiles ? 4 * B * t : ufull; }
  __device__ __forceinline__ int tile_u1(int t) const { return t < full_tiles ? 4 * B * (t + 1) : U; }
  __device__ __forceinline__ int tile_of(int u) const { return u < ufull ? u / (4 * B) : full_tiles; }
};

__device__ __forceinline__ Units make_units(int N, int K) {
  Units un;
  un.B = K / kBlockCols;
  un.full_tiles = N / kTileRows;
  un.ufull = 4 * un.B * un.full_tiles;
  un.U = un.ufull + (N % kTileRows ? un.B : 0);
  return un;
}

// Called by a whole warp after it parked its sums of tile t.  The last warp of
// the CTA to do so adds the parked sums of every warp range touching t in range
// order (rb: the CTA's W + 1 range boundaries in units, then each range's first
// tile); a tile that lies wholly in the CTA's range goes to y, a tile shared by
// CTAs c0..c1 to its workspace slot (k = c - c0), and the last CTA to deposit a
// slot adds all slots in CTA order.  Kept out of line: it runs once or twice
// per warp, and inlining it would cost the hot loop registers.
template <int MT>
__device__ __noinline__ void tile_piece_done(const GemvKMat& g, const Units& un, int c, int t, const float* red,
                                             int* tcnt, const int* rb, int ta, bool whole, long long G, int npw,
                                             int y_f32, int lane) {
  constexpr int W = gemv_warps(MT);
  const int N = g.N, M = g.M;
  const int tq0 = un.tile_u0(t), tq1 = un.tile_u1(t);   // units of tile t
  __threadfence_block();
  __syncwarp();
  // ranges r_lo..r_hi (consecutive) touch tile t; empty ranges (only when the
  // CTA has fewer units than warps) touch nothing
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
      // y rows are N * 4 (or 2) bytes apart and N % 4 == 0, so the 4 outputs of a
      // lane share the alignment of y itself: vector stores when y allows them
      const float vv[4] = {v[m].x, v[m].y, v[m].z, v[m].w};
      if (y_f32) {
        float* yp = reinterpret_cast<float*>(g.y) + (size_t)m * N + n0;
        if ((reinterpret_cast<uintptr_t>(g.y) & 15) == 0) *reinterpret_cast<float4*>(yp) = v[m];
        else for (int r = 0; r < 4; ++r) yp[r] = vv[r];
      } else {
        __half* yp = reinterpret_cast<__half*>(g.y) + (size_t)m * N + n0;
        if ((reinterpret_cast<uintptr_t>(g.y) & 7) == 0) {
          const __half2 h01 = __floats2half2_rn(vv[0], vv[1]), h23 = __floats2half2_rn(vv[2], vv[3]);
          uint2 hv;
          hv.x = *reinterpret_cast<const uint32_t*>(&h01);
          hv.y = *reinterpret_cast<const uint32_t*>(&h23);
          *reinterpret_cast<uint2*>(yp) = hv;
        } else {
          for (int r = 0; r < 4; ++r) yp[r] = __float2half_rn(vv[r]);
        }
      }
    }
  };
  const bool in_tile = lane < tile_lanes(N, t);
  if (whole) {                                         // the tile lies wholly in this CTA's range
    if (in_tile) write_y();
    return;
  }
  // CTAs c0..c1 share tile t (CTA of unit u: ((u + 1) G - 1) / U)
  const long long U = un.U;
  const int c0 = (int)((((long long)tq0 + 1) * G - 1) / U);
  const int c1 = (int)((((long long)tq1) * G - 1) / U);
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

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(p));
}

// Packed-code registers of one full-tile unit: its sign chunk and its payload chunk.
struct QRegs {
  uint4 s, p;
};

// One CTA = one contiguous range of one matrix's units.  kPerm: the matrix has
// a permutation (x is gathered through it); without one, x is already in stored
// column order.  kXM: where the decode reads x from --
//   2: shared memory, all K columns in stored order, written once by the CTA's
//      prologue (natural-order copy, then one permuting pass); the hot loop
//      reads its operands straight from there;
//   1: a natural-order copy in shared memory, gathered unit by unit into small
//      per-warp slots (when a stored-order copy as well does not fit);
//   0: global memory, gathered unit by unit into the slots.
template <int MT, bool kPerm, int kXM>
__device__ __forceinline__ void gemv_cta(const GemvKMat& g, int c, unsigned char* smem, int y_f32, uint32_t one) {
  constexpr bool kXS = kXM >= 1;                       // x staged in shared memory (natural order)
  constexpr bool kXP = kXM == 2;                       // ... and read by the decode in stored order
  constexpr bool kXPerm = kXP && kPerm;                // a separate stored-order copy is built
  constexpr int W = gemv_warps(MT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BD = g.b_d, BR = 10 - BD;
  const int R = gemv_cb_replicas(BD);
  const int N = g.N, K = g.K, M = g.M, npw = g.npw;
  const Units un = make_units(N, K);
  const int B = un.B;
  const long long G = g.ctas;
  // this CTA's units [ua, ub) and this warp's units [u0, u1)
  const int ua = (int)(c * (long long)un.U / G), ub = (int)((c + 1) * (long long)un.U / G);
  const int n = ub - ua;
  // Warp ranges: range r covers [ua + n*r/W, ua + n*(r+1)/W).  Warp w takes range
  // wr = (w % 4) * (W / 4) + w / 4, so the warps of one SM sub-partition (w, w+4,
  // ...) hold consecutive ranges and each sub-partition issues a quarter of the
  // CTA's units.
  auto range_begin = [&](int r) -> int { return ua + (int)((long long)n * r / W); };
  const int wr = (warp & 3) * (W / 4) + (warp >> 2);
  const int u0 = range_begin(wr), u1 = range_begin(wr + 1);
  const int ta = un.tile_of(ua), tb = un.tile_of(ub - 1);
  const int t_first = u0 < u1 ? un.tile_of(u0) : 0;   // piece p of the range holds tile t_first + p
  const int uf = min(u1, un.ufull);                      // full-tile units [u0, uf), partial-tile blocks [max(u0, ufull), u1)
  const int nfull = max(0, uf - u0);

  // Shared memory: codebook replicas, then (kXS) x in natural order [MT][K],
  // then (kXPerm) x in stored order [MT][K], then (kXM < 2) per warp two x slots
  // (double buffer) of MT rows x 128 columns fp16 (a full-tile unit uses its
  // first 32 columns), then [W][npw][MT][128] parked sums, the W + 1 range
  // boundaries and the W ranges' first tiles (36 ints), and one completion
  // counter per tile of the CTA's range.
  uint4* cbs = reinterpret_cast<uint4*>(smem);
  constexpr int kXSlot = MT * kBlockCols * 2;          // bytes per x slot
  const size_t xbytes = (size_t)MT * K * 2;            // one staged copy of x
  unsigned char* xn = smem + ((size_t)16 * R << BD);   // x in natural column order (kXS)
  unsigned char* xp = kXPerm ? xn + xbytes : xn;       // x in stored column order (kXP)
  unsigned char* xs_all = xn + (kXS ? xbytes : 0) + (kXPerm ? xbytes : 0);
  unsigned char* xs = xs_all + (kXP ? 0 : (size_t)warp * 2 * kXSlot);
  // token stride of the x operand the decode reads: a slot row, or a staged row of K columns
  const int xstride = kXP ? 2 * K : kBlockCols * 2;
  float* red = reinterpret_cast<float*>(xs_all + (kXP ? 0 : (size_t)W * 2 * kXSlot));
  int* rbt = reinterpret_cast<int*>(red + (size_t)W * npw * MT * kTileRows);
  int* tcnt = rbt + 36;
  for (int i = threadIdx.x; i <= tb - ta; i += blockDim.x) tcnt[i] = 0;
  if (threadIdx.x <= W) rbt[threadIdx.x] = range_begin(threadIdx.x);
  if (threadIdx.x < W) rbt[W + 1 + threadIdx.x] = un.tile_of(range_begin(threadIdx.x));   // first tile of range

  const uint64_t pol_stream = policy_evict_first(), pol_keep = policy_evict_last();

  // Full-tile blocks are contiguous in the device layout (block q of the
  // matrix at q * 4608 bytes): unit u's sign chunk is chunk 2A of block u/4
  // (A = u % 4), its payload chunk chunk 2A+1, and the block's chunk 8 holds the
  // fifth payload word of each quarter.
  const uint8_t* pk_lane = g.packed + (size_t)lane * 16;
  auto unit_off = [&](int u) -> size_t { return (size_t)(u >> 2) * 4608 + (size_t)(u & 3) * 1024; };
  auto load_unit = [&](QRegs& r, int u) {
    const uint8_t* p = pk_lane + unit_off(u);
    r.s = ldg_stream(p, pol_stream);
    r.p = ldg_stream(p + 512, pol_stream);
  };
  auto load_c8 = [&](int u) -> uint4 { return ldg_stream(pk_lane + (size_t)(u >> 2) * 4608 + 4096, pol_stream); };

  QRegs qa{}, qb{};
  uint4 c8 = make_uint4(0, 0, 0, 0), c8n = c8;
  if (nfull > 0) { load_unit(qa, u0); c8 = load_c8(u0); }

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
  // Radius parameters of this lane's rows of the first tile (raw fp16 bits
  // until they are needed, so the loads stay in flight through the prologue).
  int t = u0 < u1 ? un.tile_of(u0) : 0;
  uint16_t sc[4] = {0, 0, 0, 0}, of[4] = {0, 0, 0, 0};
  auto load_radius = [&](int tt) {
    if (lane < tile_lanes(N, tt)) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        sc[r] = ldg_keep_u16(g.scale + tt * kTileRows + 4 * lane + r, pol_keep);
        of[r] = ldg_keep_u16(g.offset + tt * kTileRows + 4 * lane + r, pol_keep);
      }
    }
  };
  if (u0 < u1) load_radius(t);
  // x columns: unit u covers columns 32 (u - 4 B t) .. +31 of its tile's row of
  // blocks; lane l takes column 32 (u - 4 B t) + l.  The permutation entry of
  // unit i+2 is loaded while unit i is decoded, the activations of unit i+1 are
  // gathered after it (from shared memory when x is staged there).
  int col1 = 0, col2 = 0;                              // column of units u0+1 and u0+2 for this lane
  {
    const int tu0 = 4 * B * t;
    col1 = 32 * (u0 + 1 - tu0) + lane;
    if (col1 >= K) col1 -= K;
    col2 = col1 + 32;
    if (col2 >= K) col2 -= K;
  }
  const int col0 = nfull > 0 ? 32 * (u0 - 4 * B * t) + lane : 0;
  int pj0 = 0, pj1 = 0;                                // x index of units u0 and u0+1
  if constexpr (!kXP) {
    if constexpr (kPerm) {
      if (nfull > 0) pj0 = ldg_keep_i32(g.perm + col0, pol_keep);
      if (nfull > 1) pj1 = ldg_keep_i32(g.perm + col1, pol_keep);
    } else {
      pj0 = col0;
      pj1 = col1;
    }
  }
  // Stored-order staging (kXPerm): the permutation is weight data, so its first
  // kPP groups of four entries per thread are loaded before the dependency wait.
  constexpr int kPP = 8;
  const int nq = K >> 2;                               // groups of four columns
  const bool pvec = (reinterpret_cast<uintptr_t>(g.perm) & 15) == 0;
  auto load_perm4 = [&](int i) -> int4 {
    if (pvec) {
      const uint4 v = ldg_keep_v4(reinterpret_cast<const uint4*>(g.perm) + i, pol_keep);
      return make_int4((int)v.x, (int)v.y, (int)v.z, (int)v.w);
    }
    return make_int4(ldg_keep_i32(g.perm + 4 * i, pol_keep), ldg_keep_i32(g.perm + 4 * i + 1, pol_keep),
                     ldg_keep_i32(g.perm + 4 * i + 2, pol_keep), ldg_keep_i32(g.perm + 4 * i + 3, pol_keep));
  };
  int4 pv[kXPerm ? kPP : 1];
  if constexpr (kXPerm) {
#pragma unroll
    for (int k = 0; k < kPP; ++k) {
      const int i = threadIdx.x + k * blockDim.x;
      pv[k] = i < nq ? load_perm4(i) : make_int4(0, 0, 0, 0);
    }
  }
  // The activations may be written by the previous kernel in the stream
  // (programmatic dependent launch): wait for it before reading x.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const uint16_t* xg = g.x;
  if constexpr (kXS) {
    // stage x (natural order, M rows) in shared memory: coalesced copy, four
    // loads in flight per thread before their stores (one round trip for a
    // token of up to 4 * 16 * blockDim columns)
    const bool vec = (reinterpret_cast<uintptr_t>(xg) & 15) == 0;
    const int per_row = K / 8, total = MT * per_row;
    for (int i0 = threadIdx.x; i0 < total; i0 += 4 * blockDim.x) {
      uint4 v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = i0 + k * blockDim.x;
        v[k] = make_uint4(0, 0, 0, 0);
        if (i < total) {
          const int m = i / per_row, j = i - m * per_row;
          if (m < M) {
            if (vec) {
              v[k] = ldg_keep_v4(reinterpret_cast<const uint4*>(xg + (size_t)m * K) + j, pol_keep);
            } else {
              uint16_t h[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) h[e] = ldg_keep_u16(xg + (size_t)m * K + 8 * j + e, pol_keep);
              v[k] = make_uint4(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16),
                                h[4] | ((uint32_t)h[5] << 16), h[6] | ((uint32_t)h[7] << 16));
            }
          }
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = i0 + k * blockDim.x;
        if (i < total) *reinterpret_cast<uint4*>(xn + (size_t)i * 16) = v[k];
      }
    }
  }
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
  if constexpr (kXPerm) {
    // x in stored order: column j of token m is x[m][perm[j]] (an entry outside
    // 0..K-1, which a permutation never holds, reads column 0)
    auto permute4 = [&](int i, int4 p) {
      const uint32_t ku = (uint32_t)K;
      const int j0 = (uint32_t)p.x < ku ? p.x : 0, j1 = (uint32_t)p.y < ku ? p.y : 0;
      const int j2 = (uint32_t)p.z < ku ? p.z : 0, j3 = (uint32_t)p.w < ku ? p.w : 0;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const uint16_t* xr = reinterpret_cast<const uint16_t*>(xn + (size_t)m * K * 2);
        uint2 w;
        w.x = (uint32_t)xr[j0] | ((uint32_t)xr[j1] << 16);
        w.y = (uint32_t)xr[j2] | ((uint32_t)xr[j3] << 16);
        *reinterpret_cast<uint2*>(xp + (size_t)m * K * 2 + 8 * (size_t)i) = w;
      }
    };
#pragma unroll
    for (int k = 0; k < kPP; ++k) {
      const int i = threadIdx.x + k * blockDim.x;
      if (i < nq) permute4(i, pv[k]);
    }
    for (int i = threadIdx.x + kPP * blockDim.x; i < nq; i += blockDim.x) permute4(i, load_perm4(i));
    __syncthreads();
  }
  // activations of one x column for every token: from the staged copy or global memory
  auto gather_x = [&](int pj, uint16_t (&h)[MT]) {
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if constexpr (kXS) h[m] = reinterpret_cast<const uint16_t*>(xn + (size_t)m * K * 2)[pj];
      else h[m] = m < M ? ldg_keep_u16(xg + (size_t)m * K + pj, pol_keep) : (uint16_t)0;
    }
  };
  auto put_x = [&](unsigned char* slot, const uint16_t (&h)[MT]) {
#pragma unroll
    for (int m = 0; m < MT; ++m) reinterpret_cast<uint16_t*>(slot + m * xstride)[lane] = h[m];
  };
  if (!kXP && nfull > 0) {
    uint16_t h0[MT];
    gather_x(pj0, h0);
    put_x(xs, h0);
    __syncwarp();
  }

  float2 acc[2][MT];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[h][m] = make_float2(0.f, 0.f);

  auto park = [&](int tt) {
    // the warp leaves tile tt: park its sums (lanes beyond the tile park zeros)
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float* rr = red + (((size_t)wr * npw + (tt - t_first)) * MT + m) * kTileRows + 4 * lane;
      *reinterpret_cast<float4*>(rr) = make_float4(acc[0][m].x, acc[0][m].y, acc[1][m].x, acc[1][m].y);
      acc[0][m] = make_float2(0.f, 0.f);
      acc[1][m] = make_float2(0.f, 0.f);
    }
    const bool whole = un.tile_u0(tt) >= ua && un.tile_u1(tt) <= ub;
    tile_piece_done<MT>(g, un, c, tt, red, tcnt, rbt, ta, whole, G, npw, y_f32, lane);
  };

  // ---------------------------------------------------------------- full-tile units
  if (nfull > 0) {
    const FragK fk = frag_consts(one, BD, R);
    const uint32_t cb_base_q = (uint32_t)__cvta_generic_to_shared(cbs) + (uint32_t)(lane % R) * 16;
    uint32_t bm[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int h = 0; h < 2; ++h) bm[i][h] = ((lane >> 3) == i && ((lane >> 2) & 1) == h) ? 0xFFFFFFFFu : 0u;
    const uint32_t xw_off = 16u * ((lane >> 2) & 1) + 4u * (lane & 3);
    int tile_end = un.tile_u1(t);                      // first unit of the next tile
    uint32_t xo = 64u * (uint32_t)(u0 - un.tile_u0(t)); // (kXP) byte offset of unit i's 32 columns in x
    if (nfull > 4) {                                   // L2 prefetch of the second block of the range
      const uint8_t* pb = g.packed + (size_t)((u0 >> 2) + 1) * 4608;
      prefetch_l2(pb + lane * 128);
      if (lane < 4) prefetch_l2(pb + 4096 + lane * 128);
    }
    // unit i of the range: cur holds its codes; when MORE, the next unit's go
    // into nxt and its activations into the other x slot
    auto step = [&](QRegs& cur, QRegs& nxt, int i, auto more_tag) {
      constexpr bool kMore = decltype(more_tag)::value;
      const int u = u0 + i;
      const bool new_block = ((u + 1) & 3) == 0, new_tile = u + 1 == tile_end;
      [[maybe_unused]] int pj2 = 0;                    // x index of unit i+2 (kXM < 2)
      if constexpr (kMore) {
        load_unit(nxt, u + 1);
        if (new_block) {
          c8n = load_c8(u + 1);
          // L2 prefetch of the block after it (lines 0..31, then 32..35)
          const uint8_t* pb = g.packed + (size_t)(((u + 1) >> 2) + 1) * 4608;
          if (i + 5 < nfull) {
            prefetch_l2(pb + lane * 128);
            prefetch_l2(pb + 4096 + (lane & 3) * 128);
          }
        }
        if (new_tile) load_radius(t + 1);
        if constexpr (!kXP) {
          if (i + 2 < nfull) {
            if constexpr (kPerm) pj2 = ldg_keep_i32(g.perm + col2, pol_keep);
            else pj2 = col2;
          }
        }
      }
      const int A = u & 3;
      const uint32_t p5 = A == 0 ? c8.x : (A == 1 ? c8.y : (A == 2 ? c8.z : c8.w));
      const unsigned char* xq = kXP ? xp + xo : xs + (i & 1) * kXSlot;
      frag_quarter<MT>(cur.s, cur.p, p5, xq, xstride, cb_base_q, fk, bm, xw_off, scp, ofp, acc);
      if constexpr (kMore) {
        if (new_tile) {
          park(t);
          ++t;
          tile_end = un.tile_u1(t);
          radius_pairs(sc, of);
        }
        if constexpr (kXP) {
          xo = new_tile ? 0u : xo + 64u;
        } else {
          uint16_t h[MT];
          gather_x(pj1, h);
          __syncwarp();                                // all lanes done reading the slot about to be reused
          put_x(xs + ((i + 1) & 1) * kXSlot, h);
          __syncwarp();
          pj1 = pj2;
          col2 = col2 + 32 < K ? col2 + 32 : col2 + 32 - K;
        }
        if (new_block) c8 = c8n;
      } else {
        park(t);
      }
    };
    using More = std::integral_constant<bool, true>;
    using Last = std::integral_constant<bool, false>;
    int i = 0;
    for (; i + 2 < nfull; i += 2) {
      step(qa, qb, i, More{});
      step(qb, qa, i + 1, More{});
    }
    if (i + 1 < nfull) {                               // two units left
      step(qa, qb, i, More{});
      step(qb, qa, i + 1, Last{});
    } else {                                           // one unit left
      step(qa, qb, i, Last{});
    }
  }

  // ---------------------------------------------------------------- partial last tile (whole blocks)
  if (u1 > max(u0, un.ufull)) {                        // the warp's range reaches into the partial tile
    const CbShift cs_ = cb_shift(BD, R);
    const uint32_t CODEM = BR ? (((1u << BR) - 1u) << (23 - BR)) : 0u;
    const unsigned char* cbb = reinterpret_cast<const unsigned char*>(cbs);
    const uint32_t q16 = (uint32_t)(lane % R) * 16;
    const int tp = un.full_tiles, L = tile_lanes(N, tp);
    const int kb0 = max(u0, un.ufull) - un.ufull, kb1 = u1 - un.ufull;
    if (nfull > 0) {                                   // the warp moved on from a full tile: new radius parameters
      load_radius(tp);
      radius_pairs(sc, of);
    }
    const uint8_t* tbase = g.packed + tile_offset(K, tp);
    uint4 d0[kChunks], d1[kChunks];
    if (lane < L) load_block(d0, tbase + (size_t)kb0 * L * kLaneBlockBytes, L, lane, pol_stream);
    for (int k2 = kb0; k2 < kb1; ++k2) {
      if (k2 + 1 < kb1 && lane < L) load_block(d1, tbase + (size_t)(k2 + 1) * L * kLaneBlockBytes, L, lane, pol_stream);
      if constexpr (!kXP) {
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int col = k2 * kBlockCols + lane + 32 * j;
          const int pc = kPerm ? ldg_keep_i32(g.perm + col, pol_keep) : col;
          uint16_t h[MT];
          gather_x(pc, h);
#pragma unroll
          for (int m = 0; m < MT; ++m) reinterpret_cast<uint16_t*>(xs + m * xstride)[lane + 32 * j] = h[m];
        }
        __syncwarp();
      }
      const unsigned char* xb = kXP ? xp + (size_t)k2 * kBlockCols * 2 : xs;
      if (lane < L) process_block<MT>(d0, xb, xstride, cbb, q16, cs_, CODEM, scp, ofp, acc);
#pragma unroll
      for (int k = 0; k < kChunks; ++k) d0[k] = d1[k];
    }
    park(tp);
  }
}

// PM: 1 = every matrix of the launch has a permutation, 0 = none has, 2 = mixed
// (each CTA follows its own matrix).  XM: where every CTA of the launch keeps x
// (kXM of gemv_cta).  The uniform cases get kernels of their own so each is
// compiled (registers, schedule) for one path only.
template <int MT, int PM, int XM>
__global__ void __launch_bounds__(gemv_warps(MT) * 32, 1)
gemv_kernel(const __grid_constant__ GemvKParams P) {
  extern __shared__ __align__(1024) unsigned char smem[];
  int mi = 0;
  while (mi + 1 < P.n_mats && (int)blockIdx.x >= P.mats[mi + 1].cta_begin) ++mi;
  const GemvKMat& g = P.mats[mi];
  const int c = (int)blockIdx.x - g.cta_begin;
  if constexpr (PM == 1) gemv_cta<MT, true, XM>(g, c, smem, P.y_f32, P.one);
  else if constexpr (PM == 0) gemv_cta<MT, false, XM>(g, c, smem, P.y_f32, P.one);
  else if (g.perm) gemv_cta<MT, true, XM>(g, c, smem, P.y_f32, P.one);
  else gemv_cta<MT, false, XM>(g, c, smem, P.y_f32, P.one);
}

template <int MT, int PM, int XM>
cudaError_t launch_gemv_pm(const GemvKParams& p, int grid, size_t smem, cudaStream_t st) {
  static std::atomic<unsigned long long> attr_set{0};   // one bit per device (setting it twice is harmless)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !((attr_set.load(std::memory_order_acquire) >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(gemv_kernel<MT, PM, XM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  e = cudaLaunchKernelEx(&cfg, gemv_kernel<MT, PM, XM>, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

template <int MT, int XM>
cudaError_t launch_gemv_xm(const GemvKParams& p, int grid, size_t smem, cudaStream_t st) {
  int with = 0;
  for (int i = 0; i < p.n_mats; ++i) with += p.mats[i].perm != nullptr;
  if (with == p.n_mats) return launch_gemv_pm<MT, 1, XM>(p, grid, smem, st);
  if (with == 0) return launch_gemv_pm<MT, 0, XM>(p, grid, smem, st);
  return launch_gemv_pm<MT, 2, XM>(p, grid, smem, st);
}

template <int MT>
cudaError_t launch_gemv_mt(const GemvKParams& p, int grid, size_t smem, cudaStream_t st) {
  // every matrix of a launch keeps x alike (the planner makes it so)
  const int xm = p.mats[0].x_smem;
  for (int i = 1; i < p.n_mats; ++i)
    if (p.mats[i].x_smem != xm) return cudaErrorInvalidValue;
  if (xm == 2) return launch_gemv_xm<MT, 2>(p, grid, smem, st);
  if (xm == 1) return launch_gemv_xm<MT, 1>(p, grid, smem, st);
  return launch_gemv_xm<MT, 0>(p, grid, smem, st);
}

}  // namespace svq
