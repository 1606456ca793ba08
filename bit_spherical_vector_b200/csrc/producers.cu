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
constexpr int kProdCols = kProdThreads * 8;       // columns written by one CTA

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

// grid (ceil(K / 2048), consumers, M).  Every CTA of a row computes the row's
// sum of squares in the same fixed order (8 consecutive elements per thread,
// butterfly over the warp, warps in index order), so all consumers of a row
// see the same scale; then it writes 2048 columns of its consumer:
//   x_g[m][j] = fp16( (h[m][s] * inv) * gamma[s] ),  s = p_g[j] (or j),
//   inv = 1 / sqrt(sum_k h[m][k]^2 / K + eps)   (fp32).
__global__ void __launch_bounds__(kProdThreads) rmsnorm_permute_kernel(const __grid_constant__ NormParams p) {
  __shared__ float wsum[kProdThreads / 32];
  const int m = blockIdx.z, g = blockIdx.y;
  const int K = p.K;
  const uint16_t* hr = p.h + (size_t)m * K;
  const int j8 = blockIdx.x * kProdCols + threadIdx.x * 8;
  const bool act = j8 < K;
  const int32_t* pm = p.perm[g];
  // The permutation and gamma are weights, not written by the previous kernel:
  // read them before waiting for it, so only the h loads follow the wait.
  int s[8];
  float gm[8];
  if (act) {
    if (pm) {
#pragma unroll
      for (int k = 0; k < 8; ++k) s[k] = __ldg(pm + j8 + k);
#pragma unroll
      for (int k = 0; k < 8; ++k) gm[k] = __half2float(__ushort_as_half(__ldg(p.gamma + s[k])));
    } else {
      const uint4 gv = __ldg(reinterpret_cast<const uint4*>(p.gamma + j8));
      const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        s[2 * k] = j8 + 2 * k;
        s[2 * k + 1] = j8 + 2 * k + 1;
        gm[2 * k] = __half2float(__ushort_as_half((uint16_t)(gw[k] & 0xFFFFu)));
        gm[2 * k + 1] = __half2float(__ushort_as_half((uint16_t)(gw[k] >> 16)));
      }
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // this thread's 8 inputs (gathered through the permutation) are loaded
  // together with the row's sum-of-squares loads
  float hv[8];
  if (act) {
    if (pm) {
#pragma unroll
      for (int k = 0; k < 8; ++k) hv[k] = act_to_f32(hr[s[k]], p.h_bf16);
    } else {
      const uint4 v = *reinterpret_cast<const uint4*>(hr + j8);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        hv[2 * k] = act_to_f32((uint16_t)(w[k] & 0xFFFFu), p.h_bf16);
        hv[2 * k + 1] = act_to_f32((uint16_t)(w[k] >> 16), p.h_bf16);
      }
    }
  }
  float ss = 0.f;
  for (int i8 = threadIdx.x * 8; i8 < K; i8 += kProdCols) {
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
  float x[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) x[k] = hv[k] * inv * gm[k];
  uint4 o;
  o.x = pack_h2(x[0], x[1]);
  o.y = pack_h2(x[2], x[3]);
  o.z = pack_h2(x[4], x[5]);
  o.w = pack_h2(x[6], x[7]);
  *reinterpret_cast<uint4*>(p.out[g] + (size_t)m * K + j8) = o;
}

// grid (ceil(I / 2048), M): x[m][j] = fp16( silu(gate[m][s]) * up[m][s] ),
// s = perm[j] (or j), silu(v) = v / (1 + e^-v) in fp32 -- the same expression
// the MoE kernel evaluates for its fused down-projection input.
__global__ void __launch_bounds__(kProdThreads) swiglu_permute_kernel(const float* __restrict__ gate,
                                                                      const float* __restrict__ up,
                                                                      const int32_t* __restrict__ perm,
                                                                      uint16_t* __restrict__ out, int I) {
  const int m = blockIdx.y;
  const int j8 = blockIdx.x * kProdCols + threadIdx.x * 8;
  const bool act = j8 < I;
  int s[8];
  if (act && perm) {                                   // weights: read before the wait
#pragma unroll
    for (int k = 0; k < 8; ++k) s[k] = __ldg(perm + j8 + k);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (!act) return;
  const float* gr = gate + (size_t)m * I;
  const float* ur = up + (size_t)m * I;
  float gv[8], uv[8];
  if (perm) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      gv[k] = gr[s[k]];
      uv[k] = ur[s[k]];
    }
  } else {
    const float4 g0 = *reinterpret_cast<const float4*>(gr + j8), g1 = *reinterpret_cast<const float4*>(gr + j8 + 4);
    const float4 u0 = *reinterpret_cast<const float4*>(ur + j8), u1 = *reinterpret_cast<const float4*>(ur + j8 + 4);
    gv[0] = g0.x; gv[1] = g0.y; gv[2] = g0.z; gv[3] = g0.w; gv[4] = g1.x; gv[5] = g1.y; gv[6] = g1.z; gv[7] = g1.w;
    uv[0] = u0.x; uv[1] = u0.y; uv[2] = u0.z; uv[3] = u0.w; uv[4] = u1.x; uv[5] = u1.y; uv[6] = u1.z; uv[7] = u1.w;
  }
  float x[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) x[k] = gv[k] / (1.0f + expf(-gv[k])) * uv[k];
  uint4 o;
  o.x = pack_h2(x[0], x[1]);
  o.y = pack_h2(x[2], x[3]);
  o.z = pack_h2(x[4], x[5]);
  o.w = pack_h2(x[6], x[7]);
  *reinterpret_cast<uint4*>(out + (size_t)m * I + j8) = o;
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
