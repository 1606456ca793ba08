// calib.h -- launchers of the calibration kernels (calib.cu): ESG, radius grid,
// encoder, ABS.  Not part of the public ABI.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

namespace svq {

constexpr int kAbsMaxCandidates = 64;
cudaError_t launch_esg(const float* x, int T, int K, double gamma, double* energy, int32_t* perm, float* weights,
                       cudaStream_t st);
cudaError_t launch_radius_grid(const float* W, int N, int K, const int32_t* perm, int b_d, uint16_t* scale,
                               uint16_t* offset, cudaStream_t st);
cudaError_t launch_encode(const float* W, int N, int K, int b_d, const int32_t* perm, const float* weights,
                          const uint16_t* codebook, const uint16_t* scale, const uint16_t* offset,
                          const uint16_t* lut, uint8_t* canonical, double* row_err, cudaStream_t st);
cudaError_t launch_abs_select(const double* row_err, int n_cand, int N, double* totals, int32_t* best,
                              cudaStream_t st);

}  // namespace svq
