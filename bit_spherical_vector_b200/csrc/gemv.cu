// gemv.cu -- launch planning for the fused SVQ decode-and-multiply for small batches (1..8 tokens per
// pass), y = W x[perm], over a group of up to eight independent matrices in one
// launch.
//
// Method ("SAGE", arXiv 2610.14745): a subvector of eight weights is
// r * sign (.) c_idx (Figure 2 caption: signs, direction index, quantized
// radius); it multiplies eight reordered activations x[perm[8g..8g+7]]
// (Figure 6 caption); weights are reconstructed on demand, never stored dense
// (Figures 1 and 5).
//
// B200 mapping:
//   * a CTA of 8 warps works on one matrix, one k-slice and up to 8 row tiles;
//     each warp owns a 128-row tile and each lane owns 4 complete rows, so a
//     row's partial sum never leaves its thread (no shuffles in the hot loop);
//   * packed codes stream from HBM with 16-byte coalesced loads
//     (ld.global.nc.L1::no_allocate), one block (9 loads per lane) ahead;
//   * the fp16 codebook sits in shared memory as 8 replicas, entry e of
//     replica q at 16-byte slot 8e + q, and lane l reads replica l % 8: the 8
//     lanes of each quarter-warp phase of an LDS.128 hit 8 different bank
//     groups whatever the indices, so the random gather is conflict free;
//   * each warp gathers x[perm] for its blocks itself, one block ahead of the
//     decode, into two small shared-memory slots read with broadcast loads;
//   * signs are applied by XOR on fp16 sign bits; the eight products of a
//     subvector are summed in fp16x2, then scaled by the radius and
//     accumulated across subvectors in fp32;
//   * split-K partials go to the workspace; the last CTA of a row chunk (found
//     with a counter) sums them in a fixed order, so results are reproducible.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "gemv_params.h"
#include "layout.cuh"
#include "svq_internal.h"

namespace svq {
namespace {

// codebook replicas (at most 32 KB) + two x slots per warp + cross-warp reduction buffer
size_t cta_smem(int b_d, int mt, int K, int S) {
  (void)K;
  (void)S;
  const int R = b_d <= 8 ? 8 : (b_d == 9 ? 4 : 2);
  return ((size_t)16 * R << b_d) + (size_t)kGemvWarps * 2 * mt * kBlockCols * 2 +
         (size_t)kGemvWarps * mt * kTileRows * sizeof(float);
}

size_t up256(size_t b) { return (b + 255) / 256 * 256; }

}  // namespace

bool plan_gemv(const GemvMatDesc* mats, int n_mats, int M, int num_sms, GemvPlan* plan) {
  if (n_mats < 1 || n_mats > kGemvMaxMats || M < 1) return false;
  const int mt = M >= 5 ? 8 : (M >= 3 ? 4 : M);
  plan->n_mats = n_mats;
  plan->M = M;
  plan->mt = mt;
  // 4 CTAs (16 warps) per SM for 1-2 tokens per pass, 2 for wider passes
  // (register-limited); shared memory per CTA is capped accordingly.
  const int per_sm = mt <= 2 ? 4 : 2;
  const size_t smem_cap = (227 * 1024) / per_sm - 1024;
  const int slots = num_sms * per_sm;
  // One CTA per (128-row tile, k-slice).  Start with the fewest slices shared
  // memory allows, then repeatedly split the matrix whose CTAs carry the most
  // blocks while the grid still fits in one wave.
  int S[kGemvMaxMats], R[kGemvMaxMats], B[kGemvMaxMats];
  int total = 0;
  for (int i = 0; i < n_mats; ++i) {
    R[i] = num_tiles(mats[i].N);
    B[i] = mats[i].K / kBlockCols;
    S[i] = 1;
    while (S[i] < B[i] && cta_smem(mats[i].b_d, mt, mats[i].K, S[i]) > smem_cap) ++S[i];
    if (cta_smem(mats[i].b_d, mt, mats[i].K, S[i]) > smem_cap) return false;
    total += R[i] * S[i];
  }
  for (;;) {
    int best = -1;
    double worst = 0;
    for (int i = 0; i < n_mats; ++i) {
      const double per_cta = (double)B[i] / S[i];
      if (S[i] < B[i] && per_cta > worst) { worst = per_cta; best = i; }
    }
    if (best < 0 || total + R[best] > slots) break;
    ++S[best];
    total += R[best];
  }
  size_t off = 0;
  int ctas = 0;
  for (int i = 0; i < n_mats; ++i) {
    const GemvMatDesc& d = mats[i];
    GemvPlanMat& pm = plan->m[i];
    pm.S = S[i];
    pm.n_rc = R[i];
    pm.ctas = S[i] * R[i];
    pm.ws_offset = off;
    pm.xp_bytes = 0;
    pm.part_bytes = S[i] > 1 ? up256((size_t)S[i] * mt * d.N * sizeof(float)) : 0;
    pm.ws_bytes = pm.xp_bytes + pm.part_bytes + (S[i] > 1 ? up256((size_t)R[i] * sizeof(unsigned)) : 0);
    off += pm.ws_bytes;
    ctas += pm.ctas;
  }
  plan->ws_total = off;
  plan->total_ctas = ctas;
  return true;
}

cudaError_t launch_gemv(const GemvMatDesc* mats, const GemvPlan& plan, int y_f32, void* ws, cudaStream_t st) {
  const int mt = plan.mt;
  const int passes = (plan.M + mt - 1) / mt;
  for (int p = 0; p < passes; ++p) {
    const int m0 = p * mt, Mp = std::min(mt, plan.M - m0);
    GemvKParams kp{};
    kp.n_mats = plan.n_mats;
    kp.y_f32 = y_f32;
    size_t smem = 0;
    int cta = 0;
    for (int i = 0; i < plan.n_mats; ++i) {
      const GemvMatDesc& d = mats[i];
      const GemvPlanMat& pm = plan.m[i];
      char* base = reinterpret_cast<char*>(ws) + pm.ws_offset;
      GemvKMat& g = kp.mats[i];
      g.packed = reinterpret_cast<const uint8_t*>(d.packed);
      g.codebook = reinterpret_cast<const uint4*>(d.codebook);
      g.scale = d.scale;
      g.offset = d.offset;
      g.perm = d.perm;
      g.x = d.x + (size_t)m0 * d.K;
      g.y = reinterpret_cast<char*>(d.y) + (size_t)m0 * d.N * (y_f32 ? 4 : 2);
      if (pm.S > 1) {
        g.partial = reinterpret_cast<float*>(base + pm.xp_bytes);
        g.counters = reinterpret_cast<unsigned*>(base + pm.xp_bytes + pm.part_bytes);
      } else {
        g.partial = nullptr;
        g.counters = nullptr;
      }
      g.N = d.N; g.K = d.K; g.b_d = d.b_d; g.S = pm.S; g.n_rc = pm.n_rc; g.cta_begin = cta; g.M = Mp;
      cta += pm.ctas;
      smem = std::max(smem, cta_smem(d.b_d, mt, d.K, pm.S));
    }
    cudaError_t e;
    switch (mt) {
      case 1: e = launch_gemv_mt<1>(kp, cta, smem, st); break;
      case 2: e = launch_gemv_mt<2>(kp, cta, smem, st); break;
      case 4: e = launch_gemv_mt<4>(kp, cta, smem, st); break;
      default: e = launch_gemv_mt<8>(kp, cta, smem, st); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace svq
