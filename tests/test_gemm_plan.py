"""Host logic of the prefill GEMM's work split (no GPU): the library's own plan_gemm, linked from the
in-tree objects into a small host program, over ~26k (N, K, M) shapes on a 148-SM part.

The kernels take unit u < F as whole tile u and unit F + s * rem + i as k-slice s of tile F + i, slice
s covering 64-column blocks [KB s / S, KB (s + 1) / S).  Checked: every (tile, k-block) pair is covered
exactly once; no slice is empty (an empty slice would leave its accumulator unwritten); the partial
slots of split tiles fit the workspace the plan sizes; F is a whole number of rounds over the grid when
only the last round is split; 256-row tiles appear only with pre-decoded weights, whose token tiles
have an instantiated kernel (128 or 256); the plans that the prefill benchmark and the GPU tests rely
on (the 2048-token gate|up and down projections, the 256-token case) come out as documented."""
import os
import shutil
import subprocess

import pytest

from bit_spherical_vector_b200 import build as svq_build

HARNESS = r"""
#include <cstdio>
#include <vector>
#include "gemm_params.h"
#include "layout.cuh"
using namespace svq;
int main() {
  long long bad = 0, cases = 0, tails = 0, splits = 0, rm256 = 0;
  const int Ns[] = {6, 130, 257, 1024, 1028, 1030, 2560, 4096, 4098, 9728, 8192, 768, 2048, 32768};
  const int Ks[] = {8, 136, 200, 512, 1032, 2560, 2568, 4096, 9728, 768, 2048};
  for (int N : Ns) for (int K : Ks) for (int M = 1; M <= 4100; M += (M < 64 ? 1 : 37)) {
    const GemmPlan g = plan_gemm(N, K, M, 148);
    ++cases;
    const int T = g.n_tiles * g.m_tiles, KB = pad_cols(K) / 64;
    if (g.rem > 0 && g.F > 0) ++tails;
    if (g.rem > 0 && g.F == 0) ++splits;
    if (g.RM == 256) ++rm256;
    std::vector<int> cover((size_t)T * KB, 0);
    const int nu = g.F + g.rem * g.S;
    size_t slots = 0;
    for (int u = 0; u < nu; ++u) {
      int t, kb0, kb1;
      if (u < g.F) { t = u; kb0 = 0; kb1 = KB; }
      else {
        const int v = u - g.F, s = v / g.rem;
        t = g.F + v % g.rem;
        kb0 = (int)(((long long)KB * s) / g.S);
        kb1 = (int)(((long long)KB * (s + 1)) / g.S);
        slots = (size_t)v + 1 > slots ? (size_t)v + 1 : slots;
      }
      if (kb1 <= kb0 || t < 0 || t >= T) { ++bad; printf("slice N=%d K=%d M=%d\n", N, K, M); }
      for (int k = kb0; k < kb1 && t >= 0 && t < T; ++k) cover[(size_t)t * KB + k]++;
    }
    for (size_t i = 0; i < cover.size(); ++i)
      if (cover[i] != 1) { ++bad; printf("cover N=%d K=%d M=%d\n", N, K, M); break; }
    if (g.partial_offset + slots * g.BN * g.RM * 4 > g.ws_bytes) { ++bad; printf("ws N=%d K=%d M=%d\n", N, K, M); }
    if (g.grid < 1 || g.grid > 148 || g.grid > nu) { ++bad; printf("grid N=%d K=%d M=%d\n", N, K, M); }
    if (g.F + g.rem != T) { ++bad; printf("F+rem N=%d K=%d M=%d\n", N, K, M); }
    if (g.rem > 0 && g.F > 0 && g.F % g.grid != 0) { ++bad; printf("rounds N=%d K=%d M=%d\n", N, K, M); }
    if (g.RM == 256 && !g.dense) { ++bad; printf("rm N=%d K=%d M=%d\n", N, K, M); }
    if (g.dense && g.BN != 128 && g.BN != 256) { ++bad; printf("bn N=%d K=%d M=%d\n", N, K, M); }
  }
  const int show[][3] = {{9728, 2560, 2048}, {2560, 9728, 2048}, {9728, 2560, 256}};
  for (auto& c : show) {
    const GemmPlan g = plan_gemm(c[0], c[1], c[2], 148);
    printf("PLAN %d %d %d RM=%d BN=%d T=%d dense=%d S=%d F=%d rem=%d\n", c[0], c[1], c[2], g.RM, g.BN,
           g.n_tiles * g.m_tiles, g.dense, g.S, g.F, g.rem);
  }
  printf("SUMMARY %lld %lld %lld %lld %lld\n", cases, bad, tails, splits, rm256);
  return bad != 0;
}
"""


def _nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not available")
def test_gemm_work_split_covers_every_tile_once(tmp_path):
    svq_build.build()
    objs = [os.path.join(svq_build.BUILD, f) for f in ("gemm.o", "gemm_dense.o", "repack.o")]
    src = tmp_path / "plan_check.cu"
    src.write_text(HARNESS)
    exe = tmp_path / "plan_check"
    cc = subprocess.run([_nvcc(), *svq_build.ARCH, "-O2", "-std=c++17", "--expt-relaxed-constexpr",
                         "-I", svq_build.INCLUDE, "-I", svq_build.CSRC, str(src), *objs, "-o", str(exe)],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0, run.stdout[-2000:]
    lines = run.stdout.splitlines()
    cases, bad, tails, splits, rm256 = map(int, lines[-1].split()[1:])
    assert cases > 20000 and bad == 0
    assert tails > 0 and splits > 0 and rm256 > 0          # all three split kinds are exercised
    plans = {tuple(map(int, ln.split()[1:4])): dict(kv.split("=") for kv in ln.split()[4:])
             for ln in lines if ln.startswith("PLAN")}
    gate = plans[(9728, 2560, 2048)]
    assert gate["RM"] == "256" and gate["dense"] == "1" and gate["F"] == "296" and gate["rem"] == "8"
    down = plans[(2560, 9728, 2048)]
    assert down["RM"] == "128" and down["dense"] == "1" and down["F"] == "148" and down["rem"] == "12"
    assert plans[(9728, 2560, 256)]["dense"] == "0"      # one 256-token tile decodes on chip
