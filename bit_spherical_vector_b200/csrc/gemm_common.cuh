// gemm_common.cuh -- pieces shared by the two tensor-core GEMM kernels (on-chip
// decode with 128-row tiles in gemm.cu, pre-decoded weights with 256-row tiles
// in gemm_dense.cu): the work-unit mapping, bounded mbarrier waits and the
// 16-bit pair conversion.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

#include "gemm_params.h"
#include "layout.cuh"
#include "sm100.cuh"

namespace svq {
namespace gemm {

// Record a timed-out wait: the status word, and the CTA's abort flag so that
// the other roles stop waiting too.
template <class Bars>
__device__ __forceinline__ void record_timeout(const GemmKParams& p, Bars* bars) {
  atomicExch(p.status, 5 /* SVQ_ERR_TIMEOUT */);
  atomicExch(&bars->abort_flag, 1);
}

// Wait that gives up on timeout or when another role has aborted.
template <class Bars>
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const GemmKParams& p, Bars* bars) {
  for (uint32_t i = 0; i < p.wait_polls; ++i) {
    if (sm100::mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 63 && *(volatile int*)&bars->abort_flag) return false;
  }
  record_timeout(p, bars);
  return false;
}

struct Unit {
  int nt, mt, s, kb0, kb1;
  int slot;             // < 0: whole tile, stored to y; else the partial slot of a k-slice
};

// Units 0..F-1 are whole tiles; the rem tiles after them are split into S
// k-slices, unit F + s * rem + i being slice s of tile F + i.  Tile index t
// runs over row tiles fastest: nt = t % n_tiles, mt = t / n_tiles.
__device__ __forceinline__ Unit unit_of(const GemmKParams& p, int u) {
  Unit w;
  const int KB = pad_cols(p.K) / 64;                  // 64-column blocks of the (padded) layout
  int t;
  if (u < p.F) {
    t = u;
    w.s = 0; w.kb0 = 0; w.kb1 = KB; w.slot = -1;
  } else {
    const int v = u - p.F;
    const int i = v % p.rem;
    t = p.F + i;
    w.s = v / p.rem;
    w.kb0 = (int)(((long long)KB * w.s) / p.S);
    w.kb1 = (int)(((long long)KB * (w.s + 1)) / p.S);
    w.slot = v;
  }
  w.nt = t % p.n_tiles;
  w.mt = t / p.n_tiles;
  return w;
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t r;
  if constexpr (BF16) {
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  } else {
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  }
  return r;
}

}  // namespace gemm
}  // namespace svq
