// gemm.cu -- SVQ prefill GEMM on the sm_100a tensor cores:
//   y[m][n] = sum_j W[n][j] * X[m][perm[j]],  W decoded from SVQ codes on chip.
//
// Method ("SAGE", arXiv 2610.14745): subvector = radius * signs (.) codeword
// (Figure 2 caption); activations are read in the ESG order (Figure 6 caption);
// the pages' prefill kernel is a "64-row GEMM loop" in which an mma adds
// A * B_j^T to an accumulator (Figure 6(b) caption) -- warp-level mma on the
// GPU it was written for.  Here the same contraction runs on tcgen05:
//
//   * pass 1 (permute kernel): X_p[m][j] = X[m][perm[j]] into the workspace, so
//     activation tiles become plain 2-D boxes for TMA;
//   * pass 2 (this kernel, persistent, one CTA per SM, 22 warps):
//       warp 0      TMA producer: X_p tiles [BN tokens x 64 k], 128-byte swizzle,
//                   into the A/B ring, and bulk copies of the packed-code
//                   blocks into a deeper ring of their own, issued ahead
//       warp 1      TMEM allocator and the single MMA-issuing thread:
//                   tcgen05.mma.cta_group::1.kind::f16, M = 128 weight rows,
//                   N = BN tokens, K = 16 per instruction, fp32 accumulators
//                   in TMEM (two buffers of BN columns)
//       warps 2..17 decoders: packed codes (bulk-copied into shared memory by
//                   the producer) -> 128 x 64 bf16/fp16 weight tile in shared
//                   memory (K-major, 128-byte swizzle), codebook from
//                   shared-memory replicas; the sixteen warps share every
//                   stage (one of its eight subvector groups, half the rows)
//       warps 18..21 epilogue: tcgen05.ld -> registers -> shared staging ->
//                   coalesced stores of y (or of the fp32 partials of a
//                   k-slice of a split tile)
//   * pass 3 (split tiles only): y = sum of the slices' partials in slice order.
//     Whole tiles fill complete rounds of the grid; the tiles of a last,
//     partial round (or, where that estimates faster, every tile) are split
//     along K so that their slices spread over all SMs.
//   * weights are the A operand (swap-AB), so small token counts still map to
//     the 128-row MMA; work units are (token tile, k-split, row tile).
// Weight rows are placed in the A tile in the order rho = lane + 32 * r (lane
// of the packed lane-block, r = its row 0..3), which makes the decoders'
// 16-byte swizzled stores conflict free; the epilogue maps TMEM lane rho back to
// weight row 4 * (rho % 32) + rho / 32.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>

#include "gemm_common.cuh"
#include "gemm_params.h"
#include "layout.cuh"
#include "sm100.cuh"
#include "svq_internal.h"

namespace svq {
namespace {

using namespace sm100;
using namespace gemm;

constexpr int kDecWarp0 = 2, kNumDec = 16;
constexpr int kEpiWarp0 = kDecWarp0 + kNumDec, kNumEpi = 4;
constexpr int kThreads = (kEpiWarp0 + kNumEpi) * 32;
constexpr int kATileBytes = 128 * 128;           // 128 rows x 64 k x 2 bytes
constexpr int kPTileBytes = 32 * kLaneBlockBytes; // packed codes of one 128-row x 128-column block
constexpr int kCbBytes = 32 * 1024;               // codebook replicas
constexpr int kStageCols = 32;                    // epilogue columns per round
constexpr int kStgBytes = kStageCols * 128 * 4;


// Packed-code ring: deeper than the A/B ring so the codes of a stage are
// requested several stages before its decode.
template <int NS>
__host__ __device__ constexpr int p_slots() { return NS + 3 <= 8 ? NS + 3 : 8; }

// DENSE (pre-decoded weights): no packed-code ring and no codebook, so the
// A/B ring can be deeper.
template <int BN, int NS, bool DENSE>
__host__ __device__ constexpr uint32_t smem_bytes() {
  return NS * kATileBytes + NS * BN * 128 + (DENSE ? 0 : p_slots<NS>() * kPTileBytes + kCbBytes) + kStgBytes +
         1024 /* barriers */ + 1024 /* align */;
}

struct Bars {
  uint64_t full_a[8], full_b[8], empty[8], full_p[8], empty_p[8], acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
  int abort_flag;
  int epi_ok;
};

// Decode decoder warp dw's share of one 64-column stage of one 128-row tile
// into the swizzled A tile: subvector group j = 8 * (kb & 1) + dw % 8 of the
// packed block, rows 2 * (dw / 8) and 2 * (dw / 8) + 1 of every lane (64 of
// the 128 rows).  The sixteen decoder warps together fill the stage.  Every decoder warp runs the same instructions (the group is
// a runtime value and the code words are read from the shared-memory copy of
// the packed block by computed address), so the warps share instruction-cache
// lines.
template <bool BF16>
__device__ __forceinline__ void decode_stage(const GemmKParams& p, int kb, const uint8_t* pk, uint8_t* a_tile,
                                             const uint8_t* cbs, int lane, int dw, int L, const float (&sc)[4],
                                             const float (&of)[4], int row_base) {
  if (lane >= L) return;
  const int kc = dw & 7;                               // 16-byte chunk within the 128-byte A row
  const int r0 = 2 * (dw >> 3);                        // this warp decodes rows r0, r0 + 1 of each lane
  const int j = 8 * (kb & 1) + kc;                     // subvector group within the packed block
  // word wi of this lane's lane-block: chunk wi / 4 at ((wi / 4) * L + lane) * 16, word wi % 4
  const uint8_t* lb = pk + lane * 16;
  const int cstride = L * 16;
  auto word = [&](int wi) -> uint32_t {
    return *reinterpret_cast<const uint32_t*>(lb + (wi >> 2) * cstride + (wi & 3) * 4);
  };
  const int bd = p.b_d;
  const uint32_t imask = (1u << bd) - 1u;
  const uint32_t cmask = (1u << (10 - bd)) - 1u;
  const int rep = p.cb_replicas;
  const uint8_t* cbq = cbs + (lane & (rep - 1)) * 16;
  const int cb_stride = rep * 16;                      // bytes per codebook entry (all replicas)
  // Fields of the lane's subvectors (row 4 * lane + r, group j) of this block:
  // sign masks of the four element pairs (bits 15 and 31, ready to XOR onto a
  // 16-bit pair), direction index, radius code.
  uint32_t smk[2][4], pidx[2], pcode[2];
  {
    // everything in the lane's own words (owner arrangement)
    const uint32_t S = word(j);
    uint32_t top[2] = {0u, 0u};
    if (j == 15) {
      // payloads 60..63 live in the top two bits of the 20 payload words (chunks
      // 4..8): read the five chunks whole (16-byte loads, conflict free)
      uint32_t pw[20];
#pragma unroll
      for (int c = 0; c < 5; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(lb + (4 + c) * cstride);
        pw[4 * c] = v.x; pw[4 * c + 1] = v.y; pw[4 * c + 2] = v.z; pw[4 * c + 3] = v.w;
      }
      uint32_t t4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int i = 0; i < 5; ++i) t4[r] |= (pw[5 * r + i] >> 30) << (8 - 2 * i);
      top[0] = r0 == 0 ? t4[0] : t4[2];
      top[1] = r0 == 0 ? t4[1] : t4[3];
    }
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int r = r0 + rr;
      const int v = 4 * j + r;
      uint32_t pay;
      if (j < 15) {
        const int wi = 16 + v / 3;
        pay = word(wi) >> (10 * (v - 3 * (wi - 16)));
      } else {
        pay = top[rr];
      }
      pidx[rr] = pay & imask;
      pcode[rr] = (pay >> bd) & cmask;
#pragma unroll
      for (int q = 0; q < 4; ++q) smk[rr][q] = (S << (4 * r + q)) & 0x80008000u;
    }
  }
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int r = r0 + rr;
    const uint32_t id = pidx[rr];
    const uint32_t code = pcode[rr];
    const uint4 cw = *reinterpret_cast<const uint4*>(cbq + id * cb_stride);
    const float scr = r0 == 0 ? sc[rr] : sc[2 + rr], ofr = r0 == 0 ? of[rr] : of[2 + rr];
    // the quantized radius: the row's table level (read through L1), or the affine form
    const bool real_row = row_base + r < p.N;          // padding rows of a ragged N decode as zeros
    const float rad = p.lut ? (real_row ? __half2float(__ushort_as_half(
                                             __ldg(p.lut + ((size_t)(row_base + r) << (10 - bd)) + code)))
                                       : 0.f)
                            : __fmaf_rn(scr, (float)code, ofr);
    const float2 rad2 = make_float2(rad, rad);
    const uint32_t c4[4] = {cw.x, cw.y, cw.z, cw.w};
    uint32_t o4[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 cf = __half22float2(*reinterpret_cast<const __half2*>(&c4[q]));
      const float2 pr = __fmul2_rn(rad2, cf);               // binary32 products r * c
      o4[q] = pack2<BF16>(pr.x, pr.y) ^ smk[rr][q];
    }
    const int rho = lane + 32 * r;                       // A-tile row of weight row 4 * lane + r
    uint8_t* dst = a_tile + (rho >> 3) * 1024 + (rho & 7) * 128 + ((kc ^ (rho & 7)) << 4);
    *reinterpret_cast<uint4*>(dst) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
  }
}

template <int BN, int NS, bool BF16, bool DENSE>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
            const __grid_constant__ GemmKParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* a_st = base;
  uint8_t* b_st = a_st + NS * kATileBytes;
  constexpr int NP = p_slots<NS>();
  uint8_t* p_st = b_st + NS * BN * 128;             // packed-code ring (NP slots; none when DENSE)
  uint8_t* cbs = p_st + (DENSE ? 0 : NP * kPTileBytes);
  float* stg = reinterpret_cast<float*>(cbs + (DENSE ? 0 : kCbBytes));
  Bars* bars = reinterpret_cast<Bars*>(reinterpret_cast<uint8_t*>(stg) + kStgBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t kTmemCols = (2 * BN) <= 32 ? 32 : (2 * BN) <= 64 ? 64 : (2 * BN) <= 128 ? 128
                                 : (2 * BN) <= 256 ? 256 : 512;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars->full_a[s], DENSE ? 1 : kNumDec);   // TMA bytes, or the decoders
      mbar_init(&bars->full_b[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int s = 0; s < NP; ++s) {
      mbar_init(&bars->full_p[s], 1);
      mbar_init(&bars->empty_p[s], kNumDec);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->acc_full[i], 1);
      mbar_init(&bars->acc_empty[i], kNumEpi);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_x);
    if (DENSE) prefetch_tmap(&tmap_w);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // Codebook replicas: entry e, replica q at 16-byte slot e * rep + q.
  if constexpr (!DENSE) {
    const int rep = p.cb_replicas;
    const int n = (1 << p.b_d) * rep;
    for (int i = threadIdx.x; i < n; i += kThreads)
      reinterpret_cast<uint4*>(cbs)[i] = __ldg(p.codebook + i / rep);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int n_units = p.F + p.rem * p.S;

  if (warp == 0) {
    // ---------------- TMA producer: activation tiles into the A/B ring (slot
    // freed by the MMA), packed codes into the P ring up to NP - 2 stages
    // ahead (slot freed by the decoders)
    if (lane == 0) {
      struct Cursor {
        int u, kb;
        Unit w;
      };
      auto start = [&](Cursor& c) {
        c.u = blockIdx.x;
        if (c.u < n_units) { c.w = unit_of(p, c.u); c.kb = c.w.kb0; }
      };
      auto advance = [&](Cursor& c) {
        if (++c.kb >= c.w.kb1) {
          c.u += gridDim.x;
          if (c.u < n_units) { c.w = unit_of(p, c.u); c.kb = c.w.kb0; }
        }
      };
      // X_p (and the decoded weights) come from the grids launched before this
      // one in the same call (programmatic dependent launch): wait for them
      asm volatile("griddepcontrol.wait;" ::: "memory");
      Cursor cb_, cp_;
      start(cb_);
      start(cp_);
      int itb = 0, itp = 0;
      bool ok = true;
      while (ok && cb_.u < n_units) {
        while (!DENSE && cp_.u < n_units && itp < itb + NP - 2) {
          const int s = itp % NP;
          const uint32_t ph = (itp / NP) & 1;
          if (itp >= NP && !wait_bar(&bars->empty_p[s], ph ^ 1, p, bars)) { ok = false; break; }
          const int L = tile_lanes(pad_rows(p.N), cp_.w.nt);
          const uint32_t pbytes = (uint32_t)L * kLaneBlockBytes;
          mbar_arrive_expect_tx(&bars->full_p[s], pbytes);
          bulk_load(p_st + s * kPTileBytes, p.packed + tile_offset(pad_cols(p.K), cp_.w.nt) + (size_t)(cp_.kb >> 1) * pbytes,
                    pbytes, &bars->full_p[s]);
          advance(cp_);
          ++itp;
        }
        if (!ok) break;
        const int s = itb % NS;
        const uint32_t ph = (itb / NS) & 1;
        if (itb >= NS && !wait_bar(&bars->empty[s], ph ^ 1, p, bars)) { ok = false; break; }
        if constexpr (DENSE) {
          // pre-decoded weights: the 128 x 64 tile of rows nt*128.. straight from the workspace
          mbar_arrive_expect_tx(&bars->full_a[s], kATileBytes);
          tma_load_2d(a_st + s * kATileBytes, &tmap_w, &bars->full_a[s], cb_.kb * 64, cb_.w.nt * kTileRows);
        }
        mbar_arrive_expect_tx(&bars->full_b[s], BN * 128);
        tma_load_2d(b_st + s * BN * 128, &tmap_x, &bars->full_b[s], cb_.kb * 64, cb_.w.mt * BN);
        advance(cb_);
        ++itb;
      }
      if (!ok) {
        // Let copies already issued land before the CTA exits.
        for (int k = std::max(0, itb - NS); k < itb; ++k) {
          mbar_wait(&bars->full_b[k % NS], (k / NS) & 1);
          if (DENSE) mbar_wait(&bars->full_a[k % NS], (k / NS) & 1);
        }
        for (int k = std::max(0, itp - NP); k < itp; ++k) mbar_wait(&bars->full_p[k % NP], (k / NP) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(BF16 ? 1 : 0, BN);
      int it = 0, acc_it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++acc_it) {
        const Unit w = unit_of(p, u);
        const int buf = acc_it & 1;
        const uint32_t aph = (acc_it >> 1) & 1;
        if (acc_it >= 2 && !wait_bar(&bars->acc_empty[buf], aph ^ 1, p, bars)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + buf * BN;
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const int s = it % NS;
          const uint32_t ph = (it / NS) & 1;
          if (!wait_bar(&bars->full_a[s], ph, p, bars) || !wait_bar(&bars->full_b[s], ph, p, bars)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = smem_desc_sw128(smem_u32(a_st + s * kATileBytes));
          const uint64_t bd = smem_desc_sw128(smem_u32(b_st + s * BN * 128));
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16)
            mma_f16(d_tmem, ad + 2 * k16, bd + 2 * k16, idesc, (kb > w.kb0 || k16 > 0) ? 1u : 0u);
          mma_commit(&bars->empty[s]);
        }
        if (!ok) break;
        mma_commit(&bars->acc_full[buf]);
      }
      // All MMAs issued by this thread are complete before TMEM is released.
      mma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0);
    }
  } else if (warp < kEpiWarp0) {
    // ---------------- decoders: all sixteen warps fill every stage together, so each
    // waits on every phase of every barrier in order (a warp that skipped
    // phases could alias an mbarrier parity).
    const int d = warp - kDecWarp0;
    int it = 0;
    bool ok = !DENSE;                        // pre-decoded weights: the decoders have nothing to do
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const Unit w = unit_of(p, u);
      // radius parameters of this lane's 4 rows of the unit's row tile
      const int L = tile_lanes(pad_rows(p.N), w.nt);
      float sc[4] = {0.f, 0.f, 0.f, 0.f}, of[4] = {0.f, 0.f, 0.f, 0.f};
      if (lane < L && !p.lut) {
        const int n0 = w.nt * kTileRows + 4 * lane;
#pragma unroll
        for (int r = 0; r < 4; ++r) {                  // rows past N (padding) decode with zeros
          sc[r] = n0 + r < p.N ? __half2float(__ushort_as_half(p.scale[n0 + r])) : 0.f;
          of[r] = n0 + r < p.N ? __half2float(__ushort_as_half(p.offset[n0 + r])) : 0.f;
        }
      }
      for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
        const int s = it % NS;
        const uint32_t ph = (it / NS) & 1;
        const int sp = it % NP;
        const uint32_t php = (it / NP) & 1;
        int good = 1;
        if (lane == 0) {
          if (it >= NS) good = wait_bar(&bars->empty[s], ph ^ 1, p, bars) ? 1 : 0;   // A slot free
          if (good) good = wait_bar(&bars->full_p[sp], php, p, bars) ? 1 : 0;       // packed codes landed
        }
        good = __shfl_sync(0xFFFFFFFFu, good, 0);
        if (!good) { ok = false; break; }
        decode_stage<BF16>(p, kb, p_st + sp * kPTileBytes, a_st + s * kATileBytes, cbs, lane, d, L, sc, of,
                           w.nt * kTileRows + 4 * lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars->full_a[s]);
          mbar_arrive(&bars->empty_p[sp]);
        }
      }
    }
  } else {
    // ---------------- epilogue
    const int q = warp & 3;                  // TMEM lane quadrant of this warp
    const int e = warp - kEpiWarp0;          // 0..3
    int acc_it = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++acc_it) {
      const Unit w = unit_of(p, u);
      const int buf = acc_it & 1;
      const uint32_t aph = (acc_it >> 1) & 1;
      if (threadIdx.x == kEpiWarp0 * 32) bars->epi_ok = wait_bar(&bars->acc_full[buf], aph, p, bars) ? 1 : 0;
      named_bar_sync(1, kNumEpi * 32);
      if (!bars->epi_ok) break;
      tc_fence_after();
      const int n0 = w.nt * kTileRows;
      const int rows = min(kTileRows, p.N - n0);
      const bool split = w.slot >= 0;
      float* part = split ? p.partial + (size_t)w.slot * BN * kTileRows : nullptr;
      for (int c0 = 0; c0 < BN; c0 += kStageCols) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + buf * BN + c0, v);
        tmem_ld_wait();
        // Weight row `row` of the tile is staged at position 4 L + ((row % 4) ^
        // x(L)), L = row / 4, x(L) = (L / 8) % 4: the reader lane L takes rows
        // 4L..4L+3 with one 16-byte load and undoes the swizzle in registers.
        // For decoded tiles (weight row 4 * lane + q in TMEM lane 32q + lane)
        // the lanes of a store that would share a bank (lane, lane + 8, ...)
        // get different offsets; pre-decoded tiles (row 32q + lane) store 32
        // distinct banks either way.
        const int row = DENSE ? 32 * q + lane : 4 * lane + q;
        const int rl = row >> 2;
        const int nl = 4 * rl + ((row & 3) ^ ((rl >> 3) & 3));
        const int xs = (lane >> 3) & 3;                // the reader's swizzle (rows 4 * lane ..)
#pragma unroll
        for (int i = 0; i < 32; ++i) stg[i * 128 + nl] = __uint_as_float(v[i]);
        named_bar_sync(1, kNumEpi * 32);
        for (int i = e * 8; i < e * 8 + 8; ++i) {
          const int m = w.mt * BN + c0 + i;
          if (m >= p.M || 4 * lane >= rows) continue;
          const float4 raw = *reinterpret_cast<const float4*>(stg + i * 128 + 4 * lane);
          const float rv[4] = {raw.x, raw.y, raw.z, raw.w};
          auto pick = [&](int t) -> float {                // rv[t ^ xs] without dynamic indexing
            const int k = t ^ xs;
            return k == 0 ? rv[0] : (k == 1 ? rv[1] : (k == 2 ? rv[2] : rv[3]));
          };
          const float4 val = make_float4(pick(0), pick(1), pick(2), pick(3));
          const int n = n0 + 4 * lane;
          const size_t o = (size_t)m * p.N + n;           // element of y
          if (split) {                                    // [token][row] of the tile's slot
            *reinterpret_cast<float4*>(part + (size_t)(c0 + i) * kTileRows + 4 * lane) = val;
          } else if ((p.N & 3) == 0) {                    // rows of 4 stay 16-byte aligned
            if (p.y_f32) {
              __stcs(reinterpret_cast<float4*>(reinterpret_cast<float*>(p.y) + o), val);   // streaming: y is not re-read
            } else {
              uint2 pk;
              pk.x = pack2<true>(val.x, val.y);
              pk.y = pack2<true>(val.z, val.w);
              __stcs(reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(p.y) + o), pk);
            }
          } else {                                        // ragged N: element by element, rows < N
            const float vv[4] = {val.x, val.y, val.z, val.w};
            for (int r = 0; r < 4 && n + r < p.N; ++r) {
              if (p.y_f32) reinterpret_cast<float*>(p.y)[o + r] = vv[r];
              else reinterpret_cast<uint16_t*>(p.y)[o + r] = __bfloat16_as_ushort(__float2bfloat16_rn(vv[r]));
            }
          }
        }
        named_bar_sync(1, kNumEpi * 32);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// X_p[m][j] = X[m][perm[j]] (16-bit values), eight columns per thread.
__global__ void permute_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm, int M, int K,
                               uint16_t* __restrict__ xp) {
  // the next grid of the call (dequantisation or GEMM) may start beside this one
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long per_row = K / 8;
  if (i >= (long long)M * per_row) return;
  const int m = (int)(i / per_row);
  const int j0 = (int)(i % per_row) * 8;
  const uint16_t* xr = x + (size_t)m * K;
  uint16_t v[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = xr[__ldg(perm + j0 + k)];
  uint4 o;
  o.x = v[0] | ((uint32_t)v[1] << 16);
  o.y = v[2] | ((uint32_t)v[3] << 16);
  o.z = v[4] | ((uint32_t)v[5] << 16);
  o.w = v[6] | ((uint32_t)v[7] << 16);
  *reinterpret_cast<uint4*>(xp + (size_t)m * K + j0) = o;
}

// The same gather with the row staged in shared memory: each CTA takes rows
// m = blockIdx.x, + gridDim.x, ...; row m is copied into one of two buffers by
// asynchronous 16-byte copies (cp.async) issued while the previous row is being
// gathered, then every thread gathers eight columns from shared memory and
// stores 16 bytes.  x, perm 16-byte aligned; 2 K 16-bit values of shared memory.
__device__ __forceinline__ void row_copy_async(uint4* dst, const uint4* src, int K8) {
  for (int c = threadIdx.x; c < K8; c += blockDim.x)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sm100::smem_u32(dst + c)), "l"(src + c)
                 : "memory");
}

__global__ void __launch_bounds__(256)
permute_rows_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm, int M, int K,
                    uint16_t* __restrict__ xp) {
  extern __shared__ uint4 prow[];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int K8 = K / 8;
  const uint32_t last = (uint32_t)K - 1u;
  int m = blockIdx.x;
  if (m < M) row_copy_async(prow, reinterpret_cast<const uint4*>(x + (size_t)m * K), K8);
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (int it = 0; m < M; m += gridDim.x, ++it) {
    const int mn = m + gridDim.x;
    if (mn < M) row_copy_async(prow + ((it + 1) & 1) * K8, reinterpret_cast<const uint4*>(x + (size_t)mn * K), K8);
    asm volatile("cp.async.commit_group;" ::: "memory");    // possibly empty: one group per row
    asm volatile("cp.async.wait_group 1;" ::: "memory");    // this row's copies have landed
    __syncthreads();
    const uint16_t* r16 = reinterpret_cast<const uint16_t*>(prow + (it & 1) * K8);
    uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)m * K);
    // indices clamped to the row: a malformed perm cannot read past the buffer
    auto at = [&](int j) -> uint32_t { return r16[min((uint32_t)j, last)]; };
    for (int c = threadIdx.x; c < K8; c += blockDim.x) {
      const int4 p0 = __ldg(reinterpret_cast<const int4*>(perm) + 2 * c);
      const int4 p1 = __ldg(reinterpret_cast<const int4*>(perm) + 2 * c + 1);
      uint4 o;
      o.x = at(p0.x) | (at(p0.y) << 16);
      o.y = at(p0.z) | (at(p0.w) << 16);
      o.z = at(p1.x) | (at(p1.y) << 16);
      o.w = at(p1.z) | (at(p1.w) << 16);
      dst[c] = o;
    }
    __syncthreads();                                        // this buffer is refilled two rows on
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Split-tile reduction: for each of the rem split tiles (tile F + i, rows
// nt * RM.., tokens mt * BN..), y = the sum of its S slot values in slice
// order (so the result does not depend on scheduling); slot s * rem + i holds
// BN x RM fp32 values [token][row].  Four outputs per thread, rows past N and
// tokens past M skipped, ragged N stored element by element.
__global__ void split_reduce_kernel(const float* __restrict__ partial, int S, int F, int rem, int n_tiles, int BN,
                                    int RM, int M, int N, void* __restrict__ y, int y_f32) {
  const int R4 = RM / 4;
  const long long total = (long long)rem * BN * R4;
  const long long stride = (long long)gridDim.x * blockDim.x;
  const size_t slot_el = (size_t)BN * RM;
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < total; q += stride) {
    const int i = (int)(q / ((long long)BN * R4));
    const int ml = (int)((q / R4) % BN), q4 = (int)(q % R4);
    const int t = F + i;
    const int m = (t / n_tiles) * BN + ml, n = (t % n_tiles) * RM + 4 * q4;
    if (m >= M || n >= N) continue;
    const size_t e = (size_t)ml * RM + 4 * q4;
    float4 acc = __ldcs(reinterpret_cast<const float4*>(partial + (size_t)i * slot_el + e));
    for (int s = 1; s < S; ++s) {
      const float4 v = __ldcs(reinterpret_cast<const float4*>(partial + ((size_t)s * rem + i) * slot_el + e));
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    const size_t o = (size_t)m * N + n;
    if ((N & 3) == 0) {
      if (y_f32) {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(y) + o) = acc;
      } else {
        uint2 pk;
        pk.x = pack2<true>(acc.x, acc.y);
        pk.y = pack2<true>(acc.z, acc.w);
        *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(y) + o) = pk;
      }
    } else {
      const float av[4] = {acc.x, acc.y, acc.z, acc.w};
      for (int r = 0; r < 4 && n + r < N; ++r) {
        if (y_f32) reinterpret_cast<float*>(y)[o + r] = av[r];
        else reinterpret_cast<uint16_t*>(y)[o + r] = __bfloat16_as_ushort(__float2bfloat16_rn(av[r]));
      }
    }
  }
}

template <int BN, int NS, bool BF16, bool DENSE = false>
cudaError_t launch_bn(const CUtensorMap& tm, const CUtensorMap& tw, const GemmKParams& p, int grid, bool pdl,
                      cudaStream_t st) {
  constexpr uint32_t smem = smem_bytes<BN, NS, DENSE>();
  static_assert(smem <= 227 * 1024, "shared memory");
  cudaError_t e = cudaFuncSetAttribute(gemm_kernel<BN, NS, BF16, DENSE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gemm_kernel<BN, NS, BF16, DENSE>, tm, tw, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <bool BF16>
cudaError_t launch_typed(int BN, const CUtensorMap& tm, const CUtensorMap& tw, const GemmKParams& p, int grid,
                         bool pdl, cudaStream_t st) {
  switch (BN) {
    case 16: return launch_bn<16, 6, BF16>(tm, tw, p, grid, pdl, st);
    case 32: return launch_bn<32, 6, BF16>(tm, tw, p, grid, pdl, st);
    case 64: return launch_bn<64, 5, BF16>(tm, tw, p, grid, pdl, st);
    case 128:
      return p.dense ? launch_bn<128, 6, BF16, true>(tm, tw, p, grid, pdl, st)
                     : launch_bn<128, 4, BF16>(tm, tw, p, grid, pdl, st);
    default:
      return p.dense ? launch_bn<256, 4, BF16, true>(tm, tw, p, grid, pdl, st)
                     : launch_bn<256, 3, BF16>(tm, tw, p, grid, pdl, st);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  // initialised once, thread-safely (function-local static)
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

}  // namespace

namespace {
std::atomic<uint32_t> g_wait_polls{kWaitPolls};
}  // namespace

uint32_t set_wait_polls(uint32_t polls) { return g_wait_polls.exchange(polls); }

GemmPlan plan_gemm(int N, int K, int M, int num_sms) {
  GemmPlan g{};
  g.BN = M >= 256 ? 256 : (M > 64 ? 128 : (M > 32 ? 64 : (M > 16 ? 32 : 16)));
  g.m_tiles = (M + g.BN - 1) / g.BN;
  // From two token tiles on (M > 128, except exactly 256: one tile of 256),
  // the matrix is decoded once into the workspace (N x K 16-bit values, the
  // activations' type) and the kernel loads weight tiles by TMA instead of
  // decoding every stage once per token tile; with one token tile the decode
  // pass would only add its own cost (at 256 tokens the decode pass of a
  // 2560 x 9728 matrix costs more than the on-chip decode it replaces).
  g.dense = g.m_tiles >= 2 ? 1 : 0;
  // Pre-decoded tiles of 256 rows (1.5x fewer L2 bytes per output) once they
  // still fill every SM at least once; below that 128-row tiles keep more SMs busy.
  const int nt256 = (pad_rows(N) + kDenseTileRows - 1) / kDenseTileRows;
  g.RM = g.dense && (long long)nt256 * g.m_tiles >= num_sms ? kDenseTileRows : kTileRows;
  g.n_tiles = g.RM == kTileRows ? num_tiles(pad_rows(N)) : nt256;
  const int T = g.n_tiles * g.m_tiles;
  const int KB = pad_cols(K) / 64;
  // Work split, by the estimated time: whole tiles round-robin over the SMs
  // (rounds of tiles times the k-blocks of a tile), optionally with every tile
  // split into S k-slices (more, shorter units), or with only the tiles of the
  // last, partial round split S ways so that they spread over all SMs.  A
  // 64-column k-block takes about 1 us with on-chip decode and 0.6 us with
  // pre-decoded tiles (set by the staging ring's latency, not the MMA); a split
  // adds the reduction pass over its S + 1 fp32 copies of the split tiles
  // (~4 TB/s) and one launch.
  const double t_kb = g.RM == kDenseTileRows ? 0.9e-6 : (g.dense ? 0.6e-6 : 1.0e-6);
  const double tile_bytes = (double)g.BN * g.RM * 4.0;
  auto red = [&](int S, int tiles) { return (double)(S + 1) * tiles * tile_bytes / 4.0e12 + 3.0e-6; };
  g.S = 1; g.F = T; g.rem = 0;
  double best = std::ceil((double)T / num_sms) * KB * t_kb;
  for (int S = 2; S <= std::min(16, std::max(1, KB / 8)); ++S) {
    const double est = std::ceil((double)T * S / num_sms) * std::ceil((double)KB / S) * t_kb + red(S, T);
    if (est < best * 0.97) { best = est; g.S = S; g.F = 0; g.rem = T; }
  }
  const int rem = T % num_sms;
  if (T > num_sms && rem > 0) {
    for (int S = 2; S <= std::min(num_sms / rem, std::max(1, KB / 4)); ++S) {
      const double est = (double)(T / num_sms) * KB * t_kb + std::ceil((double)KB / S) * t_kb + red(S, rem);
      if (est < best * 0.97) { best = est; g.S = S; g.F = T - rem; g.rem = rem; }
    }
  }
  g.grid = std::min(g.F + g.rem * g.S, num_sms);
  const size_t xp = ((size_t)M * K * 2 + 255) / 256 * 256;
  const size_t wdec = g.dense ? ((size_t)N * K * 2 + 255) / 256 * 256 : 0;
  g.xp_offset = 0;
  g.wdec_offset = xp;
  g.partial_offset = xp + wdec;
  const size_t part = g.rem > 0 ? (size_t)g.S * g.rem * (size_t)g.BN * g.RM * 4 : 0;
  g.ws_bytes = xp + wdec + part;
  return g;
}

cudaError_t launch_gemm(const GemmMatDesc& d, const GemmPlan& g, void* ws, int* status, cudaStream_t st) {
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  // X[:, perm] into the workspace, or X itself when it is already in stored
  // column order (perm NULL)
  const uint16_t* xp = d.x;
  if (d.perm) {
    uint16_t* xw = reinterpret_cast<uint16_t*>(wsb + g.xp_offset);
    const size_t row_smem = (size_t)4 * d.K;           // two staged rows
    const bool al16 = ((reinterpret_cast<uintptr_t>(d.x) | reinterpret_cast<uintptr_t>(d.perm)) & 15) == 0;
    if (al16 && row_smem <= 96 * 1024) {
      static std::atomic<bool> attr_set{false};
      if (!attr_set.load(std::memory_order_acquire)) {
        const cudaError_t ea = cudaFuncSetAttribute(permute_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                    96 * 1024);
        if (ea != cudaSuccess) return ea;
        attr_set.store(true, std::memory_order_release);
      }
      const int ctas = std::max(1, std::min(d.M, 148 * 4));
      permute_rows_kernel<<<ctas, 256, row_smem, st>>>(d.x, d.perm, d.M, d.K, xw);
    } else {
      const long long work = (long long)d.M * (d.K / 8);
      permute_kernel<<<(unsigned)((work + 255) / 256), 256, 0, st>>>(d.x, d.perm, d.M, d.K, xw);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    xp = xw;
  }
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tm;
  const cuuint64_t dims[2] = {(cuuint64_t)d.K, (cuuint64_t)d.M};
  const cuuint64_t strides[1] = {(cuuint64_t)d.K * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)g.BN};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(&tm, d.x_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                         const_cast<uint16_t*>(xp),
                         dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  // pre-decoded weights (dense plan): the matrix decoded once, in the stored
  // column order and the activations' 16-bit type, tiles of 128 rows x 64 columns
  CUtensorMap tw = tm;
  if (g.dense) {
    uint16_t* wdec = reinterpret_cast<uint16_t*>(wsb + g.wdec_offset);
    // after the permute it runs beside it (programmatic dependent launch)
    cudaError_t e = d.perm ? launch_dequant_chained(d.packed, d.N, d.K, d.b_d, d.codebook, d.scale, d.offset, d.lut,
                                                    d.x_bf16, wdec, st)
                           : launch_dequant(d.packed, d.N, d.K, d.b_d, d.codebook, d.scale, d.offset, d.lut,
                                            d.x_bf16, wdec, st);
    if (e != cudaSuccess) return e;
    const cuuint64_t wdims[2] = {(cuuint64_t)d.K, (cuuint64_t)d.N};
    const cuuint32_t wbox[2] = {64, (cuuint32_t)g.RM};
    const CUresult rw = enc(&tw, d.x_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                            wdec, wdims, strides, wbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (rw != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  GemmKParams p{};
  p.packed = reinterpret_cast<const uint8_t*>(d.packed);
  p.codebook = reinterpret_cast<const uint4*>(d.codebook);
  p.scale = d.scale;
  p.offset = d.offset;
  p.lut = d.lut;
  p.N = d.N; p.K = d.K; p.b_d = d.b_d; p.M = d.M;
  p.n_tiles = g.n_tiles; p.m_tiles = g.m_tiles; p.S = g.S; p.F = g.F; p.rem = g.rem;
  p.cb_replicas = d.b_d <= 8 ? 8 : (d.b_d == 9 ? 4 : 2);
  p.y = d.y;
  p.y_f32 = d.y_f32;
  p.partial = g.rem > 0 ? reinterpret_cast<float*>(wsb + g.partial_offset) : nullptr;
  p.status = status;
  p.wait_polls = g_wait_polls.load(std::memory_order_relaxed);
  p.dense = g.dense;
  // A grid of this call precedes the GEMM (permute and/or dequantisation): let
  // the GEMM's prologue start beside it; its producer waits before reading.
  const bool pdl = d.perm != nullptr || g.dense;
  cudaError_t e = g.RM == kDenseTileRows ? launch_gemm_dense256(tm, tw, p, g.grid, d.x_bf16, pdl, st)
                  : d.x_bf16 ? launch_typed<true>(g.BN, tm, tw, p, g.grid, pdl, st)
                             : launch_typed<false>(g.BN, tm, tw, p, g.grid, pdl, st);
  if (e != cudaSuccess || g.rem == 0) return e;
  const long long work = (long long)g.rem * g.BN * (g.RM / 4);
  const long long blocks = std::max<long long>(1, std::min<long long>((work + 255) / 256, 148LL * 8));
  split_reduce_kernel<<<(unsigned)blocks, 256, 0, st>>>(p.partial, g.S, g.F, g.rem, g.n_tiles, g.BN, g.RM, d.M, d.N,
                                                        d.y, d.y_f32);
  return cudaGetLastError();
}

}  // namespace svq
