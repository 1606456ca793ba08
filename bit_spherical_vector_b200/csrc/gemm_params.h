// gemm_params.h -- parameter block and launch plan of the tensor-core GEMM.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace svq {

// Weight rows per tile of the pre-decoded 256 x 256-tile kernel (the on-chip
// decode kernel and the 128 x 256 pre-decoded variant use 128).
constexpr int kDenseTileRows = 256;

struct GemmKParams {
  const uint8_t* packed;
  const uint4* codebook;
  const uint16_t* scale;
  const uint16_t* offset;
  const uint16_t* lut;  // per-row radius table [N][2^b_r], or null (affine radius)
  int N, K, b_d, M;
  int n_tiles, m_tiles, S;
  int F;                // units 0..F-1: whole tiles (tile index = unit), stored to y directly
  int rem;              // tiles F..F+rem-1: split into S k-slices each, as units F + s * rem + i
  int cb_replicas;
  void* y;
  int y_f32;
  float* partial;       // split tiles: fp32 slot s * rem + i of BN x RM values ([token][row]), or null
  int* status;          // device status word (bounded-wait timeouts)
  uint32_t wait_polls;  // polls before a bounded wait gives up (svq_debug_set_wait_polls)
  int dense;            // 1: weight tiles come pre-decoded from the workspace by TMA (decoders idle)
};

struct GemmPlan {
  int BN, m_tiles, n_tiles, S, grid;
  int RM;               // weight rows per tile: 128, or 256 (pre-decoded 256 x 256 tiles)
  int F, rem;           // whole-tile units, then rem tiles split S ways (rem = 0: no split)
  int dense;            // decode the whole matrix once into the workspace, then a dense GEMM
  size_t xp_offset, wdec_offset, partial_offset, ws_bytes;
};

struct GemmMatDesc {
  int N, K, b_d, M;
  const void* packed;
  const uint16_t* codebook;
  const uint16_t* scale;
  const uint16_t* offset;
  const uint16_t* lut;  // per-row radius table or null
  const int32_t* perm;
  const uint16_t* x;    // [M][K], fp16 or bf16 (x_bf16)
  int x_bf16;
  void* y;              // [M][N], fp32 (y_f32) or bf16
  int y_f32;
};

GemmPlan plan_gemm(int N, int K, int M, int num_sms);
// Poll bound of the GEMM's bounded waits for subsequent launches (tests set 0
// to make a wait give up at once); returns the previous value.
uint32_t set_wait_polls(uint32_t polls);
cudaError_t launch_gemm(const GemmMatDesc& d, const GemmPlan& g, void* ws, int* status, cudaStream_t st);
// The dequantisation pass of the pre-decoded plan (repack.cu), launched as a
// programmatic dependent of the activation permute before it: it runs beside
// that grid and completes only after it.
cudaError_t launch_dequant_chained(const void* packed, int N, int K, int b_d, const uint16_t* codebook,
                                   const uint16_t* scale, const uint16_t* offset, const uint16_t* lut, int out_bf16,
                                   uint16_t* out, cudaStream_t st);
// The 256 x 256-tile kernel on pre-decoded weights (gemm_dense.cu); tm: 256-token
// boxes of X_p, tw: 256-row boxes of the decoded weights, both 64 columns wide.
cudaError_t launch_gemm_dense256(const CUtensorMap& tm, const CUtensorMap& tw, const GemmKParams& p, int grid,
                                 int x_bf16, bool pdl, cudaStream_t st);

}  // namespace svq
