// producers.cu -- the kernels that produce a decoder layer's SVQ inputs, written
// directly in each consumer matrix's stored column order.
//
// Each subvector of an SVQ matrix multiplies eight reordered activations
// ("SAGE", arXiv 2610.14745, Figure 6 caption).  When the kernel that produces
// x writes it already reordered, the consumer is called with perm NULL: the
// GEMV reads x without the permutation lookups and the GEMM skips its
// permutation pass.  In a Qwen3-style decoder layer (the models the pages
// evaluate) those producers are the RMS normalisation in front of q|k|v and
// gate|up, and the SiLU-gated product in front of down.
//
// Both kernels are launched as programmatic dependents: they wait for the
// previous kernel on the stream before reading their input, and let the next
// kernel (a GEMV or GEMM, whose prologue reads only weights) start as soon as
// their own input has been read.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "svq_internal.h"

namespace svq {
namespace {

constexpr int kProdThreads = 256;
constexpr int kProdCols = kProdThreads * 2;       // columns written by one CTA (2 per thread)
constexpr int kSumStride = kProdThreads * 8;      // the sum of squares reads 8 columns per thread and step

struct NormParams {
  const uint16_t* h;
  const uint16_t* gamma;
  const int32_t* perm[kMaxProducerOuts];
  uint16_t* out[kMaxProducerOuts];
  float eps;
  int K;
  int h_bf16;
};

__device__ __forceinline__ float act_to_f32(uint16_t v, int bf16) {
  return bf16 ? __bfloat162float(__ushort_as_bfloat16(v)) : __half2float(__ushort_as_half(v));
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  return (uint32_t)__half_as_ushort(__float2half_rn(a)) | ((uint32_t)__half_as_ushort(__float2half_rn(b)) << 16);
}

// grid (ceil(K / 512), consumers, M).  Every CTA of a row computes the row's
// sum of squares in the same fixed order (8 consecutive elements per thread and
// step, butterfly over the warp, warps in index order), so all consumers of a
// row see the same scale; then it writes 512 columns of its consumer, two per
// thread (small CTAs spread the permutation gathers over many SMs):
//   x_g[m][j] = fp16( (h[m][s] * inv) * gamma[s] ),  s = p_g[j] (or j),
//   inv = 1 / sqrt(sum_k h[m][k]^2 / K + eps)   (fp32).
__global__ void __launch_bounds__(kProdThreads) rmsnorm_permute_kernel(const __grid_constant__ NormParams p) {
  __shared__ float wsum[kProdThreads / 32];
  const int m = blockIdx.z, g = blockIdx.y;
  const int K = p.K;
  const uint16_t* hr = p.h + (size_t)m * K;
  const int j2 = blockIdx.x * kProdCols + threadIdx.x * 2;
  const bool act = j2 < K;                       // K is a multiple of 8: j2 + 1 < K as well
  const int32_t* pm = p.perm[g];
  // The permutation and gamma are weights, not written by the previous kernel:
  // read them before waiting for it, so only the h loads follow the wait.
  int s0 = j2, s1 = j2 + 1;
  float gm0 = 0.f, gm1 = 0.f;
  if (act) {
    if (pm) {
      s0 = __ldg(pm + j2);
      s1 = __ldg(pm + j2 + 1);
      gm0 = __half2float(__ushort_as_half(__ldg(p.gamma + s0)));
      gm1 = __half2float(__ushort_as_half(__ldg(p.gamma + s1)));
    } else {
      const uint32_t gw = __ldg(reinterpret_cast<const unsigned int*>(p.gamma + j2));
      gm0 = __half2float(__ushort_as_half((uint16_t)(gw & 0xFFFFu)));
      gm1 = __half2float(__ushort_as_half((uint16_t)(gw >> 16)));
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // this thread's two inputs are loaded together with the sum-of-squares loads
  float h0 = 0.f, h1 = 0.f;
  if (act) {
    if (pm) {
      h0 = act_to_f32(hr[s0], p.h_bf16);
      h1 = act_to_f32(hr[s1], p.h_bf16);
    } else {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(hr + j2);
      h0 = act_to_f32((uint16_t)(w & 0xFFFFu), p.h_bf16);
      h1 = act_to_f32((uint16_t)(w >> 16), p.h_bf16);
    }
  }
  float ss = 0.f;
  for (int i8 = threadIdx.x * 8; i8 < K; i8 += kSumStride) {
    const uint4 v = *reinterpret_cast<const uint4*>(hr + i8);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a = act_to_f32((uint16_t)(w[k] & 0xFFFFu), p.h_bf16);
      const float b = act_to_f32((uint16_t)(w[k] >> 16), p.h_bf16);
      ss = fmaf(a, a, ss);
      ss = fmaf(b, b, ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kProdThreads / 32; ++w) tot += wsum[w];
  const float inv = 1.0f / sqrtf(tot / (float)K + p.eps);
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (!act) return;
  *reinterpret_cast<uint32_t*>(p.out[g] + (size_t)m * K + j2) = pack_h2(h0 * inv * gm0, h1 * inv * gm1);
}

// grid (ceil(I / 512), M): x[m][j] = fp16( silu(gate[m][s]) * up[m][s] ),
// s = perm[j] (or j), silu(v) = v / (1 + e^-v) in fp32 -- the same expression
// the MoE kernel evaluates for its fused down-projection input.  Two columns
// per thread.
__global__ void __launch_bounds__(kProdThreads) swiglu_permute_kernel(const float* __restrict__ gate,
                                                                      const float* __restrict__ up,
                                                                      const int32_t* __restrict__ perm,
                                                                      uint16_t* __restrict__ out, int I) {
  const int m = blockIdx.y;
  const int j2 = blockIdx.x * kProdCols + threadIdx.x * 2;
  const bool act = j2 < I;                       // I is a multiple of 8
  int s0 = j2, s1 = j2 + 1;
  if (act && perm) {                             // weights: read before the wait
    s0 = __ldg(perm + j2);
    s1 = __ldg(perm + j2 + 1);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (!act) return;
  const float* gr = gate + (size_t)m * I;
  const float* ur = up + (size_t)m * I;
  float g0, g1, u0, u1;
  if (perm) {
    g0 = gr[s0]; g1 = gr[s1];
    u0 = ur[s0]; u1 = ur[s1];
  } else {
    const float2 gv = *reinterpret_cast<const float2*>(gr + j2), uv = *reinterpret_cast<const float2*>(ur + j2);
    g0 = gv.x; g1 = gv.y; u0 = uv.x; u1 = uv.y;
  }
  const float x0 = g0 / (1.0f + expf(-g0)) * u0;
  const float x1 = g1 / (1.0f + expf(-g1)) * u1;
  *reinterpret_cast<uint32_t*>(out + (size_t)m * I + j2) = pack_h2(x0, x1);
}

template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kern, dim3 grid, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kProdThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rmsnorm_permute(const uint16_t* h, int h_bf16, const uint16_t* gamma, float eps, int M, int K,
                                   const int32_t* const* perms, uint16_t* const* outs, int n_out,
                                   cudaStream_t st) {
  NormParams p = {};
  p.h = h;
  p.gamma = gamma;
  for (int g = 0; g < n_out; ++g) {
    p.perm[g] = perms ? perms[g] : nullptr;
    p.out[g] = outs[g];
  }
  p.eps = eps;
  p.K = K;
  p.h_bf16 = h_bf16;
  const dim3 grid((unsigned)((K + kProdCols - 1) / kProdCols), (unsigned)n_out, (unsigned)M);
  return launch_pdl(rmsnorm_permute_kernel, grid, st, p);
}

cudaError_t launch_swiglu_permute(const float* gate, const float* up, int M, int I, const int32_t* perm,
                                  uint16_t* out, cudaStream_t st) {
  const dim3 grid((unsigned)((I + kProdCols - 1) / kProdCols), (unsigned)M);
  return launch_pdl(swiglu_permute_kernel, grid, st, gate, up, perm, out, I);
}

}  // namespace svq
