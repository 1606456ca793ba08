"""Host logic of the GEMV launch plan (no GPU): the library's own plan_gemv, linked from the in-tree
objects into a small host program, on the decoder layer at every batch width and on seeded groups of
one to eight matrices (ragged shapes, every b_d, with and without radius tables), 148 SMs.

The kernel gives CTA c of a matrix the blocks [c T / G, (c + 1) T / G) (T = row tiles x 128-column
blocks, G = its CTAs) and splits them into gemv_warps(mt) warp ranges the same way; it sizes its
per-warp tile sums by npw, the cross-CTA partial sums by kmax and one completion counter per tile.
Checked with those formulas: every warp range touches at most npw tiles; every tile is shared by at
most kmax CTAs (counted from the ranges); partial-sum regions and counters are disjoint, inside
the workspace and sized for kmax; the CTA count is the sum over matrices; shared memory is within the
limit; tokens per pass follow M; a group mixing matrices with and without tables is refused."""
import os
import shutil
import subprocess

import pytest

from bit_spherical_vector_b200 import build as svq_build

HARNESS = r"""
#include <cstdio>
#include <cstdint>
#include <random>
#include <vector>
#include "svq_internal.h"
#include "gemv_params.h"
#include "layout.cuh"
using namespace svq;

static long long bad = 0, cases = 0, shared_tiles = 0;
static const uint16_t kDummy = 0;

static void check(const std::vector<GemvMatDesc>& d, int M) {
  GemvPlan p;
  if (!plan_gemv(d.data(), (int)d.size(), M, 148, &p)) { ++bad; printf("refused n=%zu M=%d\n", d.size(), M); return; }
  ++cases;
  const int mt = M >= 5 ? 8 : (M >= 3 ? 4 : M);
  if (p.mt != mt) { ++bad; printf("mt M=%d\n", M); }
  const int W = gemv_warps(p.mt);
  if (p.smem > kGemvSmemMax) { ++bad; printf("smem\n"); }
  long long total = 0;
  std::vector<int> counter_used(kGemvMaxCounters, 0);
  std::vector<std::pair<size_t, size_t>> parts;
  for (size_t i = 0; i < d.size(); ++i) {
    const GemvPlanMat& pm = p.m[i];
    const long long B = pad_cols(d[i].K) / kBlockCols, tiles = num_tiles(pad_rows(d[i].N)), T = tiles * B, G = pm.ctas;
    total += G;
    if (G < 1 || G > T || pm.n_tiles != tiles) { ++bad; printf("ctas i=%zu\n", i); continue; }
    std::vector<int> ctas_of_tile(tiles, 0);            // CTAs whose block range reaches into each tile
    for (long long c = 0; c < G; ++c) {
      const long long qa = c * T / G, qb = (c + 1) * T / G, n = qb - qa;
      if (n < 1) { ++bad; printf("empty cta\n"); continue; }
      for (long long t = qa / B; t <= (qb - 1) / B; ++t) ctas_of_tile[t]++;
      for (int r = 0; r < W; ++r) {
        const long long rb = qa + n * r / W, re = qa + n * (r + 1) / W;
        if (re > rb && (re - 1) / B - rb / B + 1 > pm.npw) { ++bad; printf("npw i=%zu\n", i); }
      }
    }
    for (long long t = 0; t < tiles; ++t) {
      if (ctas_of_tile[t] < 1 || ctas_of_tile[t] > pm.kmax) { ++bad; printf("kmax i=%zu\n", i); }
      if (ctas_of_tile[t] > 1) ++shared_tiles;
    }
    if (pm.kmax > 1) {
      if (pm.part_bytes < (size_t)tiles * pm.kmax * p.mt * kTileRows * sizeof(float)) { ++bad; printf("part\n"); }
      if (pm.part_offset < kGemvCounterBytes || pm.part_offset % 256 || pm.part_offset + pm.part_bytes > p.ws_total) {
        ++bad; printf("part range\n");
      }
      parts.push_back({pm.part_offset, pm.part_offset + pm.part_bytes});
      for (long long t = 0; t < tiles; ++t) {
        const long long k = pm.counter0 + t;
        if (k < 0 || k >= kGemvMaxCounters || counter_used[k]++) { ++bad; printf("counter\n"); break; }
      }
    }
  }
  for (size_t a = 0; a < parts.size(); ++a)
    for (size_t b = a + 1; b < parts.size(); ++b)
      if (parts[a].first < parts[b].second && parts[b].first < parts[a].second) { ++bad; printf("overlap\n"); }
  if (total != p.total_ctas) { ++bad; printf("total\n"); }
}

static GemvMatDesc mat(int N, int K, int b_d, bool lut) {
  GemvMatDesc m = {};
  m.N = N; m.K = K; m.b_d = b_d;
  m.lut = lut ? &kDummy : nullptr;
  return m;
}

int main() {
  const int layer[7][3] = {{4096, 2560, 6}, {1024, 2560, 7}, {1024, 2560, 8}, {2560, 4096, 9},
                           {9728, 2560, 6}, {9728, 2560, 7}, {2560, 9728, 8}};
  for (int M = 1; M <= 16; ++M) {
    std::vector<GemvMatDesc> d;
    for (auto& s : layer) d.push_back(mat(s[0], s[1], s[2], false));
    check(d, M);
    for (auto& m : d) m.lut = &kDummy, m.b_d = m.b_d < 6 ? 6 : m.b_d;
    check(d, M);
  }
  std::mt19937 rng(7);
  const int Ns[] = {4, 6, 130, 257, 1024, 1030, 2560, 4098, 9726, 9728, 32768};
  const int Ks[] = {8, 128, 136, 1000, 2552, 2560, 4096, 9728};
  for (int it = 0; it < 3000; ++it) {
    const int n = 1 + (int)(rng() % 8), M = 1 + (int)(rng() % 16);
    const bool lut = rng() % 3 == 0;
    std::vector<GemvMatDesc> d;
    for (int i = 0; i < n; ++i) {
      const int b_d = lut ? 6 + (int)(rng() % 5) : 1 + (int)(rng() % 10);
      d.push_back(mat(Ns[rng() % 11], Ks[rng() % 8], b_d, lut));
    }
    check(d, M);
  }
  std::vector<GemvMatDesc> mixed = {mat(256, 256, 7, true), mat(256, 256, 7, false)};
  GemvPlan p;
  if (plan_gemv(mixed.data(), 2, 1, 148, &p)) { ++bad; printf("mixed accepted\n"); }
  printf("SUMMARY %lld %lld %lld\n", cases, bad, shared_tiles);
  return bad != 0;
}
"""


def _nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not available")
def test_gemv_plan_sizes_every_buffer_the_kernel_uses(tmp_path):
    svq_build.build()
    objs = [os.path.join(svq_build.BUILD, f) for f in
            ("gemv.o", "gemv_mt1.o", "gemv_mt2.o", "gemv_mt4.o", "gemv_mt8.o")]
    src = tmp_path / "gemv_plan_check.cu"
    src.write_text(HARNESS)
    exe = tmp_path / "gemv_plan_check"
    cc = subprocess.run([_nvcc(), *svq_build.ARCH, "-O2", "-std=c++17", "--expt-relaxed-constexpr",
                         "-I", svq_build.INCLUDE, "-I", svq_build.CSRC, str(src), *objs, "-o", str(exe)],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0, run.stdout[-2000:]
    cases, bad, shared = map(int, run.stdout.splitlines()[-1].split()[1:])
    assert cases >= 3000 and bad == 0
    assert shared > 0                                   # cross-CTA tiles are exercised
