// gemv_params.h -- kernel parameter block of the GEMV launch (shared by the
// planner in gemv.cu and the per-batch-width kernel translation units).
#pragma once
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "svq_internal.h"

namespace svq {

struct GemvKMat {
  const uint8_t* packed;
  const uint4* codebook;
  const uint16_t* scale;
  const uint16_t* offset;
  const int32_t* perm;    // [K]
  const uint16_t* lut;    // per-row radius table [N][2^b_r], or null
  const uint16_t* x;      // fp16 [M][K], natural input order
  void* y;                // [M][N]
  float* partial;         // [n_tiles][kmax][MT][128] when kmax > 1
  unsigned* counters;     // [n_tiles]
  int N, K, b_d, M;
  int ctas, cta_begin, kmax, npw;
};

struct GemvKParams {
  GemvKMat mats[kGemvMaxMats];
  int n_mats;
  int y_f32;
};

constexpr size_t kGemvSmemMax = 220 * 1024;

template <int MT>
cudaError_t launch_gemv_mt(const GemvKParams& p, int grid, size_t smem, cudaStream_t st);

}  // namespace svq
