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
// Per-row radius tables (svq_matrix.radius_lut): at most 2^kLutMaxBits levels.
constexpr int kLutMaxBits = 4;

cudaError_t launch_dequant(const void* packed, int N, int K, int b_d, const uint16_t* codebook,
                           const uint16_t* scale, const uint16_t* offset, const uint16_t* lut, int out_bf16,
                           uint16_t* out, cudaStream_t st);

// ---------------------------------------------------------------- producers
constexpr int kMaxProducerOuts = 8;
cudaError_t launch_rmsnorm_permute(const uint16_t* h, int h_bf16, const uint16_t* gamma, float eps, int M, int K,
                                   const int32_t* const* perms, uint16_t* const* outs, int n_out,
                                   cudaStream_t st);
cudaError_t launch_swiglu_permute(const float* gate, const float* up, int M, int I, const int32_t* perm,
                                  uint16_t* out, cudaStream_t st);

// ---------------------------------------------------------------- GEMV
constexpr int kGemvMaxMats = 8;
constexpr int kGemvMaxTokens = 8;        // tokens per pass (more are split into passes)

// Warps per CTA of the GEMV (one CTA per SM): fewer for wider passes, whose
// per-lane accumulators and activations take more registers.
__host__ __device__ constexpr int gemv_warps(int mt) { return mt <= 2 ? 12 : 8; }

// Codebook replicas in the GEMV's shared memory: 8 (conflict-free gathers) up to
// 512 entries (64 KB), 4 for 1024 entries (64 KB).
__host__ __device__ constexpr int gemv_cb_replicas(int b_d) { return b_d <= 9 ? 8 : 4; }

struct GemvMatDesc {                      // host-side description of one matrix of a launch
  int N, K, b_d;
  const void* packed;
  const uint16_t* codebook;
  const uint16_t* scale;
  const uint16_t* offset;
  const int32_t* perm;
  const uint16_t* lut;                   // per-row radius table [N][2^b_r] or null
  const uint16_t* x;                     // fp16 [M][K]
  void* y;                               // [M][N]
};

// A matrix's blocks (128-row tile t, 128-column block kb) are numbered
// q = t * (K / 128) + kb.  Its ctas CTAs take equal contiguous ranges of q.
// Workspace of a GEMV launch: completion counters (one per shared-capable row
// tile) in a fixed region at its start, then the partial sums of each matrix.
// The counter region never moves, so counters left at zero by one call are
// zero for the next, whatever its shapes.
constexpr size_t kGemvCounterBytes = 64 * 1024;
constexpr int kGemvMaxCounters = (int)(kGemvCounterBytes / sizeof(unsigned));

struct GemvPlanMat {
  int ctas;                              // CTA c covers q in [c*T/ctas, (c+1)*T/ctas), T = blocks
  int n_tiles;                           // 128-row tiles
  int kmax;                              // most CTAs sharing one tile (1: no cross-CTA sums)
  int npw;                               // most tiles that one warp's range touches
  int counter0;                          // first counter of this matrix's tiles
  size_t part_offset, part_bytes;        // partial sums [n_tiles][kmax][mt][128] (kmax > 1)
};

struct GemvPlan {
  int n_mats, M, mt;                     // tokens per pass (1, 2, 4 or 8)
  GemvPlanMat m[kGemvMaxMats];
  size_t ws_total;
  int total_ctas;
  size_t smem;                           // dynamic shared memory per CTA
};

// Deterministic launch plan (k-splits, CTA counts, workspace layout) for a group.
bool plan_gemv(const GemvMatDesc* mats, int n_mats, int M, int num_sms, GemvPlan* plan);
cudaError_t launch_gemv(const GemvMatDesc* mats, const GemvPlan& plan, int y_f32, void* ws,
                        cudaStream_t st);

}  // namespace svq
