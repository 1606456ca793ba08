// gemv.cu -- launch planning for the fused SVQ decode-and-multiply for small
// batches (1..8 tokens per pass), y = W x[perm], over a group of up to eight
// independent matrices in one launch.
//
// Method ("SAGE", arXiv 2610.14745): a subvector of eight weights is
// r * sign (.) c_idx (Figure 2 caption: signs, direction index, quantized
// radius); it multiplies eight reordered activations x[perm[8g..8g+7]]
// (Figure 6 caption); weights are reconstructed on demand, never stored dense
// (Figures 1 and 5).
//
// Work split: one CTA per SM.  Each matrix gets a number of CTAs by a greedy
// min-max over the estimated time of its slowest CTA (rounds of blocks per
// warp, plus the cross-CTA hand-off when it cannot overlap other work), and
// each of its CTAs a contiguous range of its blocks in
// storage order (tile-major), which may cross tile boundaries.  Inside a CTA
// the warps split the range again contiguously.  Partial sums are combined in
// a fixed order: warps of a CTA in shared memory (the last warp to leave a tile
// adds them in range order), CTAs sharing a tile through the workspace (the
// last CTA to finish the tile sums the slots in CTA order).
// The workspace starts with a fixed region of completion counters, then the
// partial sums of the matrices that have tiles shared by several CTAs.

#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "gemv_params.h"
#include "layout.cuh"
#include "svq_internal.h"

namespace svq {
namespace {

size_t up256(size_t b) { return (b + 255) / 256 * 256; }

// CTA of block q when T blocks are split into G contiguous ranges [c*T/G, (c+1)*T/G).
long long cta_of(long long q, long long T, long long G) { return ((q + 1) * G - 1) / T; }

// codebook replicas + two x slots per warp + per-warp partial sums of npw tiles
// + 36 ints (warp range boundaries and first tiles) + one completion counter per tile of a CTA's
// range (at most ntc tiles)
size_t cta_smem(int b_d, int mt, int npw, int ntc, bool lut) {
  const int R = gemv_cb_replicas(b_d);
  const int W = gemv_warps(mt);
  // (lut) the radius levels of the CTA's tiles, fp32 [tile][code][4][32]
  const size_t lut_bytes = lut ? ((size_t)ntc << (10 - b_d)) * kTileRows * sizeof(float) : 0;
  return ((size_t)16 * R << b_d) + (size_t)W * 2 * mt * kBlockCols * 2 +
         (size_t)W * npw * mt * kTileRows * sizeof(float) + 144 + ((size_t)ntc * 4 + 15) / 16 * 16 + lut_bytes;
}

}  // namespace

bool plan_gemv(const GemvMatDesc* mats, int n_mats, int M, int num_sms, GemvPlan* plan) {
  // a grouped launch either gives every matrix a radius table or none (one kernel per case)
  for (int i = 1; i < n_mats; ++i)
    if ((mats[i].lut != nullptr) != (mats[0].lut != nullptr)) return false;
  if (n_mats < 1 || n_mats > kGemvMaxMats || M < 1 || num_sms < 1) return false;
  const int mt = M >= 5 ? 8 : (M >= 3 ? 4 : M);
  const int W = gemv_warps(mt);
  plan->n_mats = n_mats;
  plan->M = M;
  plan->mt = mt;
  long long T[kGemvMaxMats], total_blocks = 0;
  int B[kGemvMaxMats];
  for (int i = 0; i < n_mats; ++i) {
    B[i] = pad_cols(mats[i].K) / kBlockCols;                    // the (padded) layout's blocks
    T[i] = (long long)num_tiles(pad_rows(mats[i].N)) * B[i];
    if (T[i] < 1 || T[i] > (1LL << 30)) return false;
    total_blocks += T[i];
  }
  // One wave of one CTA per SM if the partial-sum buffers fit in shared memory,
  // else more (shorter) ranges.
  for (int mult = 1; mult <= 64; mult *= 2) {
    const long long G = std::min<long long>((long long)num_sms * mult, total_blocks);
    if (G < n_mats) return false;
    int ctas[kGemvMaxMats];
    long long used = 0;
    for (int i = 0; i < n_mats; ++i) { ctas[i] = 1; ++used; }
    // Estimated time of a matrix's slowest CTA, in block times of one warp: the
    // rounds of blocks its warps run (range length / W, rounded up), plus about
    // 0.6 when the CTA range holds no whole row tile besides the ones it shares
    // at its ends, so the cross-CTA hand-off of those tiles ends the CTA instead
    // of overlapping its other work.  Greedy min-max: the next CTA goes to the
    // matrix with the largest estimate (ties: more blocks per CTA).
    auto est = [&](int i) -> double {
      const long long n = (T[i] + ctas[i] - 1) / ctas[i];
      const double rounds = (double)((n + W - 1) / W);
      const bool exposed = ctas[i] > 1 && 2LL * B[i] > n;
      return rounds + (exposed ? 0.6 : 0.0);
    };
    while (used < G) {
      int best = -1;
      double worst = -1.0, worst_per = 0.0;
      for (int i = 0; i < n_mats; ++i) {
        if (ctas[i] >= T[i]) continue;
        const double e = est(i), per = (double)T[i] / ctas[i];
        if (e > worst + 1e-9 || (e > worst - 1e-9 && per > worst_per)) { worst = e; worst_per = per; best = i; }
      }
      if (best < 0) break;
      ++ctas[best];
      ++used;
    }
    size_t smem = 0, off = kGemvCounterBytes;
    int total = 0, counters = 0;
    for (int i = 0; i < n_mats; ++i) {
      GemvPlanMat& pm = plan->m[i];
      const long long Gi = ctas[i], Ti = T[i];
      const long long cta_len = (Ti + Gi - 1) / Gi;                // longest CTA range
      const long long warp_len = (cta_len + W - 1) / W;            // longest warp range
      pm.ctas = ctas[i];
      pm.n_tiles = num_tiles(pad_rows(mats[i].N));
      pm.npw = (int)((warp_len - 1 + B[i] - 1) / B[i] + 1);
      int kmax = 1;
      for (int t = 0; t < pm.n_tiles; ++t) {
        const long long c0 = cta_of((long long)t * B[i], Ti, Gi), c1 = cta_of((long long)(t + 1) * B[i] - 1, Ti, Gi);
        kmax = std::max<int>(kmax, (int)(c1 - c0 + 1));
      }
      pm.kmax = kmax;
      pm.counter0 = counters;
      pm.part_offset = off;
      pm.part_bytes = 0;
      if (kmax > 1) {
        counters += pm.n_tiles;
        pm.part_bytes = up256((size_t)pm.n_tiles * kmax * mt * kTileRows * sizeof(float));
        off += pm.part_bytes;
      }
      total += pm.ctas;
      const int ntc = (int)((cta_len - 1 + B[i] - 1) / B[i] + 1);
      smem = std::max(smem, cta_smem(mats[i].b_d, mt, pm.npw, ntc, mats[i].lut != nullptr));
    }
    if (counters > kGemvMaxCounters) return false;
    if (counters == 0) off = 0;
    if (smem <= kGemvSmemMax) {
      plan->ws_total = off;
      plan->total_ctas = total;
      plan->smem = smem;
      return true;
    }
  }
  return false;
}

cudaError_t launch_gemv(const GemvMatDesc* mats, const GemvPlan& plan, int y_f32, void* ws, cudaStream_t st) {
  const int mt = plan.mt;
  const int passes = (plan.M + mt - 1) / mt;
  for (int p = 0; p < passes; ++p) {
    const int m0 = p * mt, Mp = std::min(mt, plan.M - m0);
    GemvKParams kp{};
    kp.n_mats = plan.n_mats;
    kp.y_f32 = y_f32;
    int cta = 0;
    for (int i = 0; i < plan.n_mats; ++i) {
      const GemvMatDesc& d = mats[i];
      const GemvPlanMat& pm = plan.m[i];
      GemvKMat& g = kp.mats[i];
      g.packed = reinterpret_cast<const uint8_t*>(d.packed);
      g.codebook = reinterpret_cast<const uint4*>(d.codebook);
      g.scale = d.scale;
      g.offset = d.offset;
      g.perm = d.perm;
      g.lut = d.lut;
      g.x = d.x + (size_t)m0 * d.K;
      g.y = reinterpret_cast<char*>(d.y) + (size_t)m0 * d.N * (y_f32 ? 4 : 2);
      if (pm.kmax > 1) {
        g.partial = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + pm.part_offset);
        g.counters = reinterpret_cast<unsigned*>(ws) + pm.counter0;
      } else {
        g.partial = nullptr;
        g.counters = nullptr;
      }
      g.N = d.N; g.K = d.K; g.b_d = d.b_d; g.M = Mp;
      g.ctas = pm.ctas; g.cta_begin = cta; g.kmax = pm.kmax; g.npw = pm.npw;
      cta += pm.ctas;
    }
    const size_t smem = plan.smem;
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
