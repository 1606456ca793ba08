// gather.cu -- x_p = x[:, perm] for the matrices of one GEMV launch.
//
// The ESG permutation (SAGE, arXiv 2610.14745, Figure 6 caption: each subvector
// multiplies eight reordered activations) is applied once per matrix and call
// here, so the decode kernel's CTAs read their slice of x_p with contiguous
// 16-byte copies instead of each gathering it through perm.
#include <cuda_runtime.h>

#include <cstdint>

#include "gemv_params.h"

namespace svq {
namespace {

// x_p[m][j] = x[m][perm[j]] for every matrix of the launch (2048 elements per
// CTA, eight independent gathers in flight per thread).
__global__ void __launch_bounds__(256) gather_kernel(const __grid_constant__ GatherParams P) {
  int mi = 0;
  while (mi + 1 < P.n_mats && (int)blockIdx.x >= P.mats[mi + 1].cta_begin) ++mi;
  const GatherMat& g = P.mats[mi];
  const long long e0 = (long long)((int)blockIdx.x - g.cta_begin) * 2048;
  const long long total = (long long)g.M * g.K;
  int pj[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const long long e = e0 + k * 256 + threadIdx.x;
    pj[k] = e < total ? __ldg(g.perm + (int)(e % g.K)) : 0;
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");       // x may come from the previous kernel
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  uint16_t v[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const long long e = e0 + k * 256 + threadIdx.x;
    v[k] = e < total ? g.x[(e / g.K) * g.K + pj[k]] : 0;
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const long long e = e0 + k * 256 + threadIdx.x;
    if (e < total) g.xp[e] = v[k];
  }
}

}  // namespace

cudaError_t launch_gather(const GatherParams& p, int grid, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, gather_kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace svq
