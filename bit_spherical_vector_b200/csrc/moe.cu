// moe.cu -- grouped SVQ GEMV over a device-side list of (matrix, token) items,
// for mixture-of-experts layers whose routing is produced on the GPU.
//
// Method ("SAGE", arXiv 2610.14745): each expert matrix is an SVQ matrix
// (Figure 2 caption) applied with its own ESG permutation (Figure 6 caption);
// the pages evaluate an MoE model (Qwen3-30B-A3B, abstract) but describe no
// MoE kernel.  Design here:
//   1. routing: count the items of every matrix, build the list of touched
//      matrices, group the item indices by matrix and estimate each matrix's
//      work -- on the device, no host round trip; every CTA of moe_kernel builds
//      these tables in shared memory when they are small, else route_kernel
//      (one CTA) writes them to the workspace first;
//   2. moe_kernel (persistent): one work unit = (touched matrix, 128-row tile);
//      each CTA takes a contiguous range of units, so the codebook and the
//      input rows of a matrix are staged once for all its tiles; the unit
//      decodes its weights once and applies them to all of that matrix's items
//      (up to MT tokens per pass, a one-token path when a matrix has a single
//      item), 8 warps splitting K, partial sums combined in shared memory in
//      warp order; the input row of an item is either fp16 x or, for a down
//      projection, fp16(silu(gate) * up) computed on the fly from an fp32
//      [gate | up] row;
//   3. combine_kernel (when accumulating): y[r] = sum of the items with
//      out_row r, in item order (deterministic); one CTA per output row
//      compacts its row's item list in item order, linear in the items.
// Item fields are range-checked on the device: an input row outside x is read
// as zeros, an output row outside y is not written, and either sets the device
// status word to SVQ_ERR_INVALID_ARG (svq_get_device_status).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "gemv_device.cuh"
#include "layout.cuh"
#include "moe_params.h"
#include "svq.h"

namespace svq {
namespace {

constexpr int kMoeWarps = 8;
constexpr int kMoeCostSmem = 2048;              // cost-prefix entries kept in shared memory
constexpr int kRouteThreads = 1024;

// Work of one row tile of a matrix with ni items, in decode passes of up to mt
// items: a pass over the codes costs about 19 instructions per subvector-row
// plus 6 per item of the pass width (1, 2 or mt).
__device__ __forceinline__ int moe_matrix_cost(int ni, int mt) {
  int cost = 0;
  for (int c0 = 0; c0 < ni; c0 += mt) {
    const int nc = min(mt, ni - c0);
    const int width = nc == 1 ? 1 : (nc == 2 ? 2 : mt);
    cost += 19 + 6 * width;
  }
  return cost;
}

__global__ void __launch_bounds__(kRouteThreads) route_kernel(MoeKParams p) {
  extern __shared__ int sh[];                   // [n_mats] counts, then scan scratch
  int* cnt = sh;
  for (int i = threadIdx.x; i < p.n_mats; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < p.n_items; i += blockDim.x) {
    const int m = p.items[i].matrix;
    if (m >= 0 && m < p.n_mats) atomicAdd(&cnt[m], 1);
    else atomicExch(p.status, SVQ_ERR_INVALID_ARG);
  }
  __syncthreads();
  // Exclusive scans of the counts (item offsets) and of the touched flags
  // (active list), in chunks of blockDim.x matrices.
  int base_items = 0, base_active = 0;
  for (int c0 = 0; c0 < p.n_mats; c0 += blockDim.x) {
    const int m = c0 + threadIdx.x;
    const int v = m < p.n_mats ? cnt[m] : 0;
    const int f = v > 0 ? 1 : 0;
    // pack (items, active) into one 64-bit scan value
    long long x = ((long long)v << 20) | f;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xFFFFFFFFu, x, o);
      if (lane >= o) x += y;
    }
    __shared__ long long s_w[kRouteThreads / 32];
    if (lane == 31) s_w[wid] = x;
    __syncthreads();
    if (wid == 0) {
      long long w = lane < (int)(blockDim.x / 32) ? s_w[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xFFFFFFFFu, w, o);
        if (lane >= o) w += y;
      }
      if (lane < (int)(blockDim.x / 32)) s_w[lane] = w;
    }
    __syncthreads();
    const long long incl = x + (wid > 0 ? s_w[wid - 1] : 0);
    const long long excl = incl - (((long long)v << 20) | f);
    if (m < p.n_mats) {
      p.offsets[m] = base_items + (int)(excl >> 20);
      p.cursor[m] = 0;
      if (f) p.active[base_active + (int)(excl & 0xFFFFF)] = m;
    }
    const long long tot = s_w[blockDim.x / 32 - 1];
    __syncthreads();
    base_items += (int)(tot >> 20);
    base_active += (int)(tot & 0xFFFFF);
  }
  if (threadIdx.x == 0) {
    p.offsets[p.n_mats] = base_items;
    *p.n_active = base_active;
  }
  __syncthreads();
  // Group item indices by matrix (order inside a matrix does not affect any
  // result: every item is computed on its own).
  for (int i = threadIdx.x; i < p.n_items; i += blockDim.x) {
    const int m = p.items[i].matrix;
    if (m < 0 || m >= p.n_mats) continue;
    const int slot = atomicAdd(&p.cursor[m], 1);
    p.sorted[p.offsets[m] + slot] = i;
  }
  // Work estimate of every touched matrix (its row tiles times the decode
  // passes over its items) and its exclusive prefix over the active list: the
  // MoE kernel gives each CTA an equal share of the total.
  const int na = base_active, R = num_tiles(p.N);
  int base_cost = 0;
  for (int c0 = 0; c0 < na; c0 += blockDim.x) {
    const int a = c0 + threadIdx.x;
    int v = 0;
    if (a < na) {
      const int m = p.active[a];
      v = R * moe_matrix_cost(p.offsets[m + 1] - p.offsets[m], p.mt);
    }
    int x = v;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
      if (lane >= o) x += y;
    }
    __shared__ int s_c[kRouteThreads / 32];
    if (lane == 31) s_c[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int w = lane < (int)(blockDim.x / 32) ? s_c[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, w, o);
        if (lane >= o) w += y;
      }
      if (lane < (int)(blockDim.x / 32)) s_c[lane] = w;
    }
    __syncthreads();
    const int incl = x + (wid > 0 ? s_c[wid - 1] : 0);
    if (a < na) p.costpre[a] = base_cost + incl - v;
    const int tot = s_c[blockDim.x / 32 - 1];
    __syncthreads();
    base_cost += tot;
  }
  if (threadIdx.x == 0) p.costpre[na] = base_cost;
}

// Input rows of items sorted[i0 .. i0 + nc) in permuted order into xs ([MT][K]
// fp16): x_mode 0 gathers fp16 x; x_mode 1 computes fp16(silu(gate) * up) from
// an fp32 [gate | up] row.  Each thread handles 8 consecutive columns: 8
// independent permutation loads, then 8 (or 16) independent gathers per row.
template <int MT>
__device__ __forceinline__ void stage_x(const MoeKParams& p, const svq_matrix& W, const int* sorted, int i0,
                                        int nc, unsigned char* xs, uint64_t pol_keep) {
  const int K = p.K;
  int xrow[MT];
  bool xok[MT];
#pragma unroll
  for (int c = 0; c < MT; ++c) {
    xrow[c] = c < nc ? p.items[sorted[i0 + c]].x_row : 0;
    // an input row outside x is reported (status word) and read as zeros
    xok[c] = xrow[c] >= 0 && xrow[c] < p.n_x_rows;
    if (c < nc && !xok[c] && threadIdx.x == 0) atomicExch(p.status, SVQ_ERR_INVALID_ARG);
    if (!xok[c]) xrow[c] = 0;
  }
  for (int j8 = threadIdx.x * 8; j8 < K; j8 += blockDim.x * 8) {
    int pj[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) pj[k] = W.perm ? ldg_keep_i32(W.perm + j8 + k, pol_keep) : j8 + k;
#pragma unroll
    for (int c = 0; c < MT; ++c) {
      if (c >= nc) break;
      uint32_t h[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (!xok[c]) {
        // zeros (the item was reported as invalid)
      } else if (p.x_mode == 0) {
        const uint16_t* xr = reinterpret_cast<const uint16_t*>(p.x) + (size_t)xrow[c] * K;
#pragma unroll
        for (int k = 0; k < 8; ++k) h[k] = ldg_keep_u16(xr + pj[k], pol_keep);
      } else {
        const float* xr = reinterpret_cast<const float*>(p.x) + (size_t)xrow[c] * 2 * K;
        float gv[8], uv[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) { gv[k] = __ldg(xr + pj[k]); uv[k] = __ldg(xr + K + pj[k]); }
#pragma unroll
        for (int k = 0; k < 8; ++k)
          h[k] = __half_as_ushort(__float2half_rn(gv[k] / (1.0f + expf(-gv[k])) * uv[k]));
      }
      *reinterpret_cast<uint4*>(xs + ((size_t)c * K + j8) * 2) =
          make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
    }
  }
}

// One (matrix, row tile) unit for the nc staged items: the 8 warps split the
// tile's blocks, their sums are combined in shared memory in warp order.
template <int NC, int MT>
__device__ __forceinline__ void moe_tile(const MoeKParams& p, const svq_matrix& W, const int* sorted, int t,
                                         int i0, int nc, const unsigned char* cbs, const unsigned char* xs,
                                         float* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = p.N, K = p.K, B = K / kBlockCols;
  const int BD = W.b_d, BR = 10 - BD;
  const int RR = cb_replicas(BD);
  const CbShift cs = cb_shift(BD);
  const uint32_t CODEM = BR ? (((1u << BR) - 1u) << (23 - BR)) : 0u;
  const int wb0 = (B * warp) / kMoeWarps, wb1 = (B * (warp + 1)) / kMoeWarps, nb = wb1 - wb0;
  const int L = tile_lanes(N, t);
  // matrices with a per-row radius table are not taken here: reported, decoded as zeros
  const bool lut_refused = W.radius_lut != nullptr;
  if (lut_refused && threadIdx.x == 0) atomicExch(p.status, SVQ_ERR_INVALID_ARG);
  const bool on = lane < L && !lut_refused;
  const int row0 = t * kTileRows + 4 * lane;
  const uint64_t pol_stream = policy_evict_first(), pol_keep = policy_evict_last();
  const uint8_t* tile_base = reinterpret_cast<const uint8_t*>(W.packed) + tile_offset(K, t);
  const size_t blk_bytes = (size_t)L * kLaneBlockBytes;
  float2 acc[2][NC];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int q = 0; q < NC; ++q) acc[h][q] = make_float2(0.f, 0.f);
  if (on && nb > 0) {
    uint4 d0[kChunks], d1[kChunks];
    load_block(d0, tile_base + (size_t)wb0 * blk_bytes, L, lane, pol_stream);
    float sc[4], of[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      sc[r] = __half2float(__ushort_as_half(ldg_keep_u16(W.radius_scale + row0 + r, pol_keep)));
      of[r] = __half2float(__ushort_as_half(ldg_keep_u16(W.radius_offset + row0 + r, pol_keep)));
    }
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
    const uint32_t q16 = (uint32_t)(lane % RR) * 16;
    for (int b = 0; b < nb; ++b) {
      if (b + 1 < nb) load_block(d1, tile_base + (size_t)(wb0 + b + 1) * blk_bytes, L, lane, pol_stream);
      process_block<NC>(d0, xs + (size_t)(wb0 + b) * kBlockCols * 2, K * 2, cbs, q16, cs, CODEM, scp, ofp, acc);
#pragma unroll
      for (int k = 0; k < kChunks; ++k) d0[k] = d1[k];
    }
  }
#pragma unroll
  for (int q = 0; q < NC; ++q) {
    float* rr = red + ((size_t)warp * MT + q) * kTileRows + 4 * lane;
    *reinterpret_cast<float4*>(rr) = make_float4(acc[0][q].x, acc[0][q].y, acc[1][q].x, acc[1][q].y);
  }
  __syncthreads();
  const int rows = L * 4;
  for (int e = threadIdx.x; e < rows * nc; e += blockDim.x) {
    const int c = e / rows, nl = e - c * rows;
    float v = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < kMoeWarps; ++w8) v += red[((size_t)w8 * MT + c) * kTileRows + nl];
    const int item = sorted[i0 + c];
    const svq_group_item it = p.items[item];
    const int n = t * kTileRows + nl;
    v *= it.out_scale;
    if (p.accumulate) {
      p.item_out[(size_t)item * N + n] = v;
    } else if (it.out_row >= 0 && it.out_row < p.n_out_rows) {
      p.y[(size_t)it.out_row * N + n] = v;
    } else if (e == threadIdx.x) {
      atomicExch(p.status, SVQ_ERR_INVALID_ARG);     // an output row outside y: reported, not written
    }
  }
  __syncthreads();                                   // red is reused by the next unit
}

// Exclusive scan of v over the CTA; *total receives the sum.  ws: 32 ints of
// shared scratch.  Every thread of the CTA must call it.
__device__ __forceinline__ int block_scan_excl(int v, int* ws, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) ws[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int w = lane < nw ? ws[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) ws[lane] = w;
  }
  __syncthreads();
  const int incl = x + (wid > 0 ? ws[wid - 1] : 0);
  *total = ws[nw - 1];
  __syncthreads();
  return incl - v;
}

// The routing tables of route_kernel, built by this CTA in shared memory:
// offsets [n_mats + 1], active [n_mats], cost prefix [n_mats + 1], sorted
// [n_items], cursors [n_mats].  Every CTA computes the same offsets, active
// list and cost prefix; the order of the items inside a matrix may differ
// between CTAs, which changes no result (each item is computed on its own).
__device__ void moe_local_route(const MoeKParams& p, int* rt, int& n_active) {
  __shared__ int s_ws[32];
  const int nm = p.n_mats, R = num_tiles(p.N);
  int* offs = rt;
  int* act = offs + nm + 1;
  int* cst = act + nm;
  int* srt = cst + nm + 1;
  int* cur = srt + p.n_items;
  for (int i = threadIdx.x; i < nm; i += blockDim.x) { offs[i] = 0; cur[i] = 0; }
  __syncthreads();
  for (int i = threadIdx.x; i < p.n_items; i += blockDim.x) {
    const int m = p.items[i].matrix;
    if (m >= 0 && m < nm) atomicAdd(&offs[m], 1);
    else if (blockIdx.x == 0) atomicExch(p.status, SVQ_ERR_INVALID_ARG);
  }
  __syncthreads();
  int base = 0, base_a = 0;
  for (int c0 = 0; c0 < nm; c0 += blockDim.x) {
    const int m = c0 + threadIdx.x;
    const int v = m < nm ? offs[m] : 0;
    const int f = v > 0 ? 1 : 0;
    int tv, tf;
    const int ev = block_scan_excl(v, s_ws, &tv);
    const int ef = block_scan_excl(f, s_ws, &tf);
    if (m < nm) {
      offs[m] = base + ev;
      if (f) act[base_a + ef] = m;
    }
    base += tv;
    base_a += tf;
  }
  if (threadIdx.x == 0) offs[nm] = base;
  __syncthreads();
  for (int i = threadIdx.x; i < p.n_items; i += blockDim.x) {
    const int m = p.items[i].matrix;
    if (m < 0 || m >= nm) continue;
    srt[offs[m] + atomicAdd(&cur[m], 1)] = i;
  }
  int bc = 0;
  for (int c0 = 0; c0 < base_a; c0 += blockDim.x) {
    const int a = c0 + threadIdx.x;
    int v = 0;
    if (a < base_a) {
      const int m = act[a];
      v = R * moe_matrix_cost(offs[m + 1] - offs[m], p.mt);
    }
    int tv;
    const int ev = block_scan_excl(v, s_ws, &tv);
    if (a < base_a) cst[a] = bc + ev;
    bc += tv;
  }
  if (threadIdx.x == 0) cst[base_a] = bc;
  __syncthreads();
  n_active = base_a;
}

// Persistent: CTA c takes a contiguous range of the (touched matrix, row tile)
// units holding an equal share of the estimated work, so consecutive units
// mostly share a matrix and its codebook and input rows stay staged in shared
// memory.
template <int MT>
__global__ void __launch_bounds__(kMoeWarps * 32, 1) moe_kernel(const __grid_constant__ MoeKParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int R = num_tiles(p.N);
  unsigned char* cbs = smem;
  unsigned char* xs = smem + (size_t)32 * 1024;                 // [MT][K] fp16 after the codebook
  float* red = reinterpret_cast<float*>(xs + (size_t)MT * p.K * 2);   // [8][MT][128]
  int* rt = reinterpret_cast<int*>(red + (size_t)kMoeWarps * MT * kTileRows);   // routing tables
  // Routing tables: built here (small tables) or read from route_kernel's
  // output, whose cost prefix is then copied to shared memory when it is short
  // (one parallel load instead of a chain of dependent loads in the search).
  const int *offs, *act, *srt, *cpre;
  int na;
  if (p.local_route) {
    moe_local_route(p, rt, na);
    offs = rt;
    act = offs + p.n_mats + 1;
    cpre = act + p.n_mats;
    srt = cpre + p.n_mats + 1;
  } else {
    na = *p.n_active;
    offs = p.offsets;
    act = p.active;
    srt = p.sorted;
    cpre = p.costpre;
    if (na + 1 <= kMoeCostSmem) {
      for (int i = threadIdx.x; i <= na; i += blockDim.x) rt[i] = p.costpre[i];
      __syncthreads();
      cpre = rt;
    }
  }
  // This CTA's share [lo, hi) of the total work; unit (a, t) (active matrix a,
  // row tile t) starts at costpre[a] + t * (its tile cost) and belongs to the
  // CTA whose share holds that start.
  const long long total = cpre[na];
  const long long lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
  int a_lo = 0, a_hi = na;                         // last a with costpre[a] <= lo
  while (a_hi - a_lo > 1) {
    const int mid = (a_lo + a_hi) >> 1;
    if (cpre[mid] <= lo) a_lo = mid; else a_hi = mid;
  }
  const uint64_t pol_keep = policy_evict_last();
  int cb_m = -1, x_m = -1, x_c0 = -1;
  for (int a = a_lo; a < na && cpre[a] < hi; ++a) {
    const int ca = cpre[a], tile_cost = (cpre[a + 1] - ca) / R;
    int t0 = 0;
    if (ca < lo) t0 = (int)((lo - ca + tile_cost - 1) / tile_cost);
    const long long t1l = (hi - ca + tile_cost - 1) / tile_cost;
    const int t1 = t1l < R ? (int)t1l : R;
    for (int t = t0; t < t1; ++t) {
    const int m = act[a];
    const svq_matrix W = p.mats[m];
    const int i0 = offs[m], ni = offs[m + 1] - i0;
    for (int c0 = 0; c0 < ni; c0 += MT) {
      const int nc = min(MT, ni - c0);
      if (cb_m != m || x_m != m || x_c0 != c0) {
        __syncthreads();                                 // everyone is done with the staged data
        if (cb_m != m) {
          const int RR = cb_replicas(W.b_d);
          const uint32_t cb_s = (uint32_t)__cvta_generic_to_shared(cbs);
          const uint4* cb = reinterpret_cast<const uint4*>(W.codebook);
          for (int i = threadIdx.x; i < (RR << W.b_d); i += blockDim.x)
            asm volatile("cp.async.ca.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(cb_s + 16u * i),
                         "l"(cb + i / RR), "l"(pol_keep)
                         : "memory");
          asm volatile("cp.async.commit_group;" ::: "memory");
          cb_m = m;
        }
        stage_x<MT>(p, W, srt, i0 + c0, nc, xs, pol_keep);
        x_m = m;
        x_c0 = c0;
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
      }
      if (MT > 1 && nc == 1) moe_tile<1, MT>(p, W, srt, t, i0 + c0, nc, cbs, xs, red);
      else if (MT > 2 && nc == 2) moe_tile<2, MT>(p, W, srt, t, i0 + c0, nc, cbs, xs, red);
      else moe_tile<MT, MT>(p, W, srt, t, i0 + c0, nc, cbs, xs, red);
    }
    }
  }
}

// y[r][n] = sum over items i with out_row r (ascending i) of item_out[i][n].
// One CTA per (output row, 256-column chunk): the CTA scans the item list once and compacts the
// indices of its row's items in item order (warp ballots, then a prefix over
// the warps), so the work is linear in the number of items per row; rows with
// more items than the shared list holds fall back to a scan per column.
constexpr int kCombineThreads = 256;
constexpr int kCombineList = 2048;
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const MoeKParams p) {
  __shared__ int list[kCombineList];
  __shared__ int s_warp[kCombineThreads / 32];
  __shared__ int s_count;
  const int r = blockIdx.x, lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (threadIdx.x == 0) s_count = 0;
  __syncthreads();
  for (int base = 0; base < p.n_items; base += kCombineThreads) {
    const int i = base + threadIdx.x;
    const bool hit = i < p.n_items && p.items[i].out_row == r;
    const unsigned bal = __ballot_sync(0xFFFFFFFFu, hit);
    if (lane == 0) s_warp[wid] = __popc(bal);
    __syncthreads();
    int before = s_count;
    for (int w = 0; w < wid; ++w) before += s_warp[w];
    const int pos = before + __popc(bal & ((1u << lane) - 1u));
    if (hit && pos < kCombineList) list[pos] = i;
    __syncthreads();
    if (threadIdx.x == 0) {
      int add = 0;
      for (int w = 0; w < kCombineThreads / 32; ++w) add += s_warp[w];
      s_count += add;
    }
    __syncthreads();
  }
  const int cnt = s_count;
  if (cnt == 0) return;                              // rows with no item are left untouched
  // this CTA's columns: chunk blockIdx.y of kCombineThreads columns
  for (int n = blockIdx.y * kCombineThreads + threadIdx.x; n < min(p.N, (int)(blockIdx.y + 1) * kCombineThreads);
       n += kCombineThreads) {
    float s = 0.f;
    if (cnt <= kCombineList) {
      for (int k = 0; k < cnt; ++k) s += p.item_out[(size_t)list[k] * p.N + n];
    } else {
      for (int i = 0; i < p.n_items; ++i)
        if (p.items[i].out_row == r) s += p.item_out[(size_t)i * p.N + n];
    }
    p.y[(size_t)r * p.N + n] = s;
  }
}

template <int MT>
cudaError_t launch_moe_mt(const MoeKParams& p, int grid, size_t smem, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(moe_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  moe_kernel<MT><<<grid, kMoeWarps * 32, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

bool moe_local_route(int n_mats, int n_items) { return n_mats <= 2048 && n_items <= 4096; }

size_t moe_smem_bytes(int max_b_d, int K, int mt, int n_mats, int n_items) {
  (void)max_b_d;                                   // replicas keep every codebook within 32 KB
  const size_t tables = moe_local_route(n_mats, n_items) ? (size_t)(4 * n_mats + 2 + n_items) * 4
                                                         : (size_t)kMoeCostSmem * 4;
  return (size_t)32 * 1024 + (size_t)mt * K * 2 + (size_t)kMoeWarps * mt * kTileRows * 4 + tables;
}

MoeWorkspace moe_workspace_layout(int n_mats, int n_items, int N, int accumulate) {
  MoeWorkspace w;
  auto up = [](size_t b) { return (b + 255) / 256 * 256; };
  size_t off = 0;
  w.offsets = off; off += up((size_t)(n_mats + 1) * 4);
  w.cursor = off; off += up((size_t)n_mats * 4);
  w.sorted = off; off += up((size_t)n_items * 4);
  w.active = off; off += up((size_t)n_mats * 4);
  w.n_active = off; off += 256;
  w.costpre = off; off += up((size_t)(n_mats + 1) * 4);
  w.item_out = off; off += accumulate ? up((size_t)n_items * N * 4) : 0;
  w.total = off;
  return w;
}

cudaError_t launch_moe(MoeKParams p, int mt, int n_out_rows, int num_sms, cudaStream_t st) {
  cudaError_t e = cudaSuccess;
  if (!p.local_route) {
    const size_t route_smem = (size_t)p.n_mats * 4;
    e = cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)route_smem);
    if (e != cudaSuccess) return e;
    route_kernel<<<1, kRouteThreads, route_smem, st>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const size_t smem = moe_smem_bytes(p.max_b_d, p.K, mt, p.n_mats, p.n_items);
  switch (mt) {
    case 1: e = launch_moe_mt<1>(p, num_sms, smem, st); break;
    case 2: e = launch_moe_mt<2>(p, num_sms, smem, st); break;
    default: e = launch_moe_mt<4>(p, num_sms, smem, st); break;
  }
  if (e != cudaSuccess) return e;
  if (p.accumulate) {
    const dim3 grid((unsigned)n_out_rows, (unsigned)((p.N + kCombineThreads - 1) / kCombineThreads));
    combine_kernel<<<grid, kCombineThreads, 0, st>>>(p);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace svq
