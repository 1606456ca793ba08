// gemm_dense.cu -- the prefill GEMM on weights already decoded into the
// workspace (N x K values of the activations' 16-bit type, written by the
// dequantisation pass), with 256-row x 256-token tiles per CTA:
//   y[m][n] = sum_j Wdec[n][j] * X_p[m][j].
//
// Once the weights need no on-chip decode the kernel is a plain tensor-core
// GEMM whose speed is set by how many operand bytes each SM pulls from L2 per
// MMA: a 128 x 256 tile takes 48 KB per 64-column k-block, a 256 x 256 tile
// 64 KB for twice the outputs (1.5x fewer bytes per output), with every CTA
// loading its own tiles (no clusters).  Per CTA (persistent, one per SM, 18 warps):
//   warp 0      TMA producer: per k-block one 256-row box of the decoded
//               weights and one 256-token box of X_p (128-byte swizzle) into a
//               three-stage ring, both completing on the stage's barrier
//   warp 1      TMEM allocator (all 512 columns) and the single MMA-issuing
//               thread: two tcgen05.mma.cta_group::1.kind::f16 per 16-column
//               step, rows 0..127 into TMEM columns 0..255 and rows 128..255
//               into columns 256..511 (M = 128, N = 256 each), same B operand
//   warps 2..17 drain: each warp owns the TMEM lanes of its quadrant (warp % 4)
//               and 64 of the 256 token columns of both halves; tcgen05.ld 32
//               columns, then per token one 32-row coalesced store of y (or of
//               the fp32 partial of a k-slice)
// The accumulator fills TMEM, so the next unit's MMAs wait for the drain; the
// producer keeps loading meanwhile, so the ring is full when they resume.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gemm_common.cuh"
#include "gemm_params.h"
#include "layout.cuh"
#include "sm100.cuh"

namespace svq {
namespace {

using namespace sm100;
using namespace gemm;

constexpr int kRM = kDenseTileRows;              // weight rows per tile
constexpr int kBN = 256;                         // tokens per tile
constexpr int kNS = 3;                           // ring stages
constexpr int kDrainWarp0 = 2, kNumDrain = 16;
constexpr int kThreads = (kDrainWarp0 + kNumDrain) * 32;
constexpr int kABytes = kRM * 128;               // 256 rows x 64 k x 2 bytes
constexpr int kBBytes = kBN * 128;
constexpr uint32_t kTmemCols = 512;

struct DBars {
  uint64_t full[kNS], empty[kNS], acc_full, acc_empty, drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr uint32_t kSmemBytes = kNS * (kABytes + kBBytes) + 1024 /* barriers */ + 1024 /* align */;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

template <bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
gemm_dense_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                  const __grid_constant__ GemmKParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* a_st = base;
  uint8_t* b_st = a_st + kNS * kABytes;
  DBars* bars = reinterpret_cast<DBars*>(b_st + kNS * kBBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNS; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, kNumDrain);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_x);
    prefetch_tmap(&tmap_w);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int n_units = p.F + p.rem * p.S;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      // the decoded weights and X_p come from the grids launched before this one
      // in the same call (programmatic dependent launch): wait for them
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const Unit w = unit_of(p, u);
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const int s = it % kNS;
          const uint32_t ph = (it / kNS) & 1;
          if (it >= kNS && !wait_bar(&bars->empty[s], ph ^ 1, p, bars)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars->full[s], kABytes + kBBytes);
          tma_load_2d(a_st + s * kABytes, &tmap_w, &bars->full[s], kb * 64, w.nt * kRM);
          tma_load_2d(b_st + s * kBBytes, &tmap_x, &bars->full[s], kb * 64, w.mt * kBN);
        }
      }
      if (!ok) {
        // Let copies already issued land before the CTA exits.
        for (int k = it > kNS ? it - kNS : 0; k < it; ++k) mbar_wait(&bars->full[k % kNS], (k / kNS) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(BF16 ? 1 : 0, kBN);
      int it = 0, acc_it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++acc_it) {
        const Unit w = unit_of(p, u);
        // the previous unit's accumulator has been read out
        if (acc_it >= 1 && !wait_bar(&bars->acc_empty, (acc_it - 1) & 1, p, bars)) { ok = false; break; }
        tc_fence_after();
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const int s = it % kNS;
          const uint32_t ph = (it / kNS) & 1;
          if (!wait_bar(&bars->full[s], ph, p, bars)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(a_st + s * kABytes);
          const uint64_t ad0 = smem_desc_sw128(a0);
          const uint64_t ad1 = smem_desc_sw128(a0 + kABytes / 2);   // rows 128..255
          const uint64_t bd = smem_desc_sw128(smem_u32(b_st + s * kBBytes));
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16) {
            const uint32_t acc = (kb > w.kb0 || k16 > 0) ? 1u : 0u;
            mma_f16(tmem, ad0 + 2 * k16, bd + 2 * k16, idesc, acc);
            mma_f16(tmem + kBN, ad1 + 2 * k16, bd + 2 * k16, idesc, acc);
          }
          mma_commit(&bars->empty[s]);
        }
        if (!ok) break;
        mma_commit(&bars->acc_full);
      }
      // All MMAs issued by this thread are complete before TMEM is released.
      mma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0);
    }
  } else {
    // ---------------- drain: TMEM -> y (or a k-slice's partial slot)
    const int q = warp & 3;                          // TMEM lane quadrant of this warp
    const int e = (warp - kDrainWarp0) >> 2;         // token columns 64 e .. 64 e + 63
    int acc_it = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++acc_it) {
      const Unit w = unit_of(p, u);
      int good = 1;
      if (lane == 0) good = wait_bar(&bars->acc_full, acc_it & 1, p, bars) ? 1 : 0;
      good = __shfl_sync(0xFFFFFFFFu, good, 0);
      if (!good) break;
      tc_fence_after();
      float* part = w.slot >= 0 ? p.partial + (size_t)w.slot * kBN * kRM : nullptr;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int rt = h * 128 + 32 * q + lane;      // row within the tile (TMEM lane 32 q + lane of half h)
        const int n = w.nt * kRM + rt;
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          const int c0 = e * 64 + cc * 32;
          uint32_t v[32];
          tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + h * kBN + c0, v);
          tmem_ld_wait();
          const int m0 = w.mt * kBN + c0;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (m0 + i >= p.M) break;
            const float val = __uint_as_float(v[i]);
            if (part) {
              part[(size_t)(c0 + i) * kRM + rt] = val;                  // [token][row] of the slot
            } else if (n < p.N) {
              const size_t o = (size_t)(m0 + i) * p.N + n;
              // streaming stores: y is not re-read here, the operand tiles are
              if (p.y_f32) __stcs(reinterpret_cast<float*>(p.y) + o, val);
              else __stcs(reinterpret_cast<unsigned short*>(p.y) + o, __bfloat16_as_ushort(__float2bfloat16_rn(val)));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <bool BF16>
cudaError_t launch_dense(const CUtensorMap& tm, const CUtensorMap& tw, const GemmKParams& p, int grid, bool pdl,
                         cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(gemm_dense_kernel<BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gemm_dense_kernel<BF16>, tm, tw, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_dense256(const CUtensorMap& tm, const CUtensorMap& tw, const GemmKParams& p, int grid,
                                 int x_bf16, bool pdl, cudaStream_t st) {
  return x_bf16 ? launch_dense<true>(tm, tw, p, grid, pdl, st) : launch_dense<false>(tm, tw, p, grid, pdl, st);
}

}  // namespace svq
