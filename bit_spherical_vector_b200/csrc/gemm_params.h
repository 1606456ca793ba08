// gemm_params.h -- parameter block and launch plan of the tensor-core GEMM.
#pragma once
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace svq {

struct GemmKParams {
  const uint8_t* packed;
  const uint4* codebook;
  const uint16_t* scale;
  const uint16_t* offset;
  const uint16_t* lut;  // per-row radius table [N][2^b_r], or null (affine radius)
  int N, K, b_d, M;
  int n_tiles, m_tiles, S;
  int cb_replicas;
  void* y;
  int y_f32;
  float* partial;       // [S][part_stride] when S > 1 (slice s: [M][N] row-major)
  long long part_stride;  // elements between partial slices (M N rounded up to 4)
  int* status;          // device status word (bounded-wait timeouts)
  uint32_t wait_polls;  // polls before a bounded wait gives up (svq_debug_set_wait_polls)
  int dense;            // 1: weight tiles come pre-decoded from the workspace by TMA (decoders idle)
};

struct GemmPlan {
  int BN, m_tiles, n_tiles, S, grid;
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

}  // namespace svq
