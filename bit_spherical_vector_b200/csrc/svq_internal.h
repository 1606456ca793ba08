// svq_internal.h -- declarations shared by the library's translation units
// (kernel launchers and the GEMV plan).  Not part of the public ABI.
#pragma once
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace svq {

cudaError_t launch_repack(const uint8_t* canon, int N, int K, int b_d, void* out, cudaStream_t st);
cudaError_t launch_unpack(const void* packed, int N, int K, int b_d, uint8_t* signs, uint16_t* idx,
                          uint16_t* code, cudaStream_t st);
cudaError_t launch_dequant(const void* packed, int N, int K, int b_d, const uint16_t* codebook,
                           const uint16_t* scale, const uint16_t* offset, int out_bf16, uint16_t* out,
                           cudaStream_t st);

// ---------------------------------------------------------------- GEMV
constexpr int kGemvMaxMats = 8;
constexpr int kGemvWarps = 4;            // warps per CTA; they split the k-slice of one 128-row tile
constexpr int kGemvMaxTokens = 8;        // tokens per pass (more are split into passes)

struct GemvMatDesc {                      // host-side description of one matrix of a launch
  int N, K, b_d;
  const void* packed;
  const uint16_t* codebook;
  const uint16_t* scale;
  const uint16_t* offset;
  const int32_t* perm;
  const uint16_t* x;                     // fp16 [M][K]
  void* y;                               // [M][N]
};

struct GemvPlanMat {
  int S;                                 // k-splits
  int n_rc;                              // 128-row tiles (one CTA per tile and k-slice)
  int ctas;                              // S * n_rc
  size_t ws_offset;                      // gathered x, partials, counters; 256-byte aligned
  size_t xp_bytes, part_bytes;
  size_t ws_bytes;
};

struct GemvPlan {
  int n_mats, M, mt;                     // tokens per pass (1, 2, 4 or 8)
  GemvPlanMat m[kGemvMaxMats];
  size_t ws_total;
  int total_ctas;
};

// Deterministic launch plan (k-splits, CTA counts, workspace layout) for a group.
bool plan_gemv(const GemvMatDesc* mats, int n_mats, int M, int num_sms, GemvPlan* plan);
cudaError_t launch_gemv(const GemvMatDesc* mats, const GemvPlan& plan, int y_f32, void* ws,
                        cudaStream_t st);

}  // namespace svq
