// calib.cu -- the calibration side of SAGE on the GPU: Energy-Stratified
// Grouping (channel energies, the tier permutation, fitting weights), the
// per-row radius grid, the activation-weighted SVQ encoder and the Adaptive
// Bit Split choice.
//
// "SAGE" (arXiv 2610.14745), abstract and Figure 2 caption: each subvector of
// eight weights is encoded as signs, a direction index and a quantized radius;
// ESG puts channels of different energy tiers into each subvector and weights
// the fit by activation energy; Figure 4(a): the energy enters through an
// exponent gamma; ABS encodes a matrix under each candidate direction/radius
// split of the 18-bit budget and keeps the split with the lowest
// activation-weighted reconstruction error.  Readings (the pages give no
// formulas): energy e_k = mean_t x[t][k]^2; tiers = channels sorted by energy
// (highest first, ties to the lower index) cut into 8 runs of K/8, subvector g
// taking the g-th channel of every tier; the encoder takes s_i = (w_i < 0) and
// the (direction, radius code) pair minimising sum_i e_i (|w_i| - r c_i)^2,
// ties to the lowest direction, then the lowest code; the radius grid of a row
// is uniform between its smallest and largest subvector norm.
//
// Every integer these kernels produce (the permutation, signs, directions,
// radius codes, the chosen split) is decided from fp64 values formed with one
// rounding per operation in a fixed order -- the operations a plain fp64 loop
// performs -- so the results are reproducible bit for bit.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>

#include "calib.h"

namespace svq {
namespace {

constexpr int kCalThreads = 256;

__device__ __forceinline__ double h2d(uint16_t h) { return (double)__half2float(__ushort_as_half(h)); }

// binary64 -> binary16, one round-to-nearest-even step (IEEE 754): the value
// is cut to a multiple of the fp16 quantum of its binade (2^(e-10) for normal
// results, 2^-24 below 2^-14) with ties to an even multiple; a carry into the
// next binade and overflow to infinity follow from the encoding.
__device__ uint16_t f64_to_f16_rne(double v) {
  const unsigned long long b = (unsigned long long)__double_as_longlong(v);
  const uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
  const int ex = (int)((b >> 52) & 0x7FF);
  const unsigned long long man = b & ((1ull << 52) - 1);
  if (ex == 0x7FF) return (uint16_t)(sign | (man ? 0x7E00u : 0x7C00u));
  if (ex == 0) return sign;                             // |v| < 2^-1022: rounds to zero
  const int e = ex - 1023;                              // v = 1.m * 2^e
  if (e > 15) return (uint16_t)(sign | 0x7C00u);
  const unsigned long long m = man | (1ull << 52);      // v = m * 2^(e - 52)
  const int qe = (e < -14 ? -14 : e) - 10;              // exponent of the fp16 quantum
  const int shift = qe - (e - 52);                      // >= 42
  if (shift > 53) return sign;                          // below half the smallest subnormal
  unsigned long long q = m >> shift;
  const unsigned long long rem = m & ((1ull << shift) - 1), half = 1ull << (shift - 1);
  if (rem > half || (rem == half && (q & 1))) ++q;
  unsigned bits;
  if (qe == -24) bits = (unsigned)q;                    // subnormal (q = 1024 is the smallest normal)
  else bits = ((unsigned)(e + 15) << 10) + (unsigned)(q - 1024);   // q = 2048 carries into the exponent
  if (bits >= 0x7C00u) bits = 0x7C00u;
  return (uint16_t)(sign | bits);
}

// ---------------------------------------------------------------- ESG
// e_k = (sum_t x[t][k]^2) / T, t ascending.
__global__ void esg_energy_kernel(const float* __restrict__ x, int T, int K, double* __restrict__ energy) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  double s = 0.0;
  for (int t = 0; t < T; ++t) {
    const double v = (double)x[(size_t)t * K + k];
    const double sq = __dmul_rn(v, v);
    s = t == 0 ? sq : __dadd_rn(s, sq);
  }
  energy[k] = __ddiv_rn(s, (double)T);
}

// Channel k's place in the energy order is its rank: the channels of higher
// energy plus the lower-indexed channels of equal energy.  perm[8g + t] takes
// the channel of rank t * K/8 + g; weights[k] = e_k ^ gamma.
constexpr int kRankTile = 2048;
__global__ void esg_perm_kernel(const double* __restrict__ energy, int K, double gamma, int32_t* __restrict__ perm,
                                float* __restrict__ weights) {
  __shared__ double tile[kRankTile];
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  const double ek = k < K ? energy[k] : 0.0;
  int rank = 0;
  for (int j0 = 0; j0 < K; j0 += kRankTile) {
    const int n = min(kRankTile, K - j0);
    __syncthreads();
    for (int j = threadIdx.x; j < n; j += blockDim.x) tile[j] = energy[j0 + j];
    __syncthreads();
    if (k < K) {
      for (int j = 0; j < n; ++j) {
        const double ej = tile[j];
        rank += (ej > ek || (ej == ek && j0 + j < k)) ? 1 : 0;
      }
    }
  }
  if (k >= K) return;
  const int G = K / 8;
  perm[8 * (rank % G) + rank / G] = k;
  if (weights) weights[k] = (float)pow(ek, gamma);
}

// ---------------------------------------------------------------- radius grid
// One warp per row: subvector norms of the stored-order row (squares summed in
// element order), their minimum lo and maximum hi; offset = fp16(lo), scale =
// fp16((hi - lo) / (2^b_r - 1)) (0 when b_r = 0).
__global__ void radius_grid_kernel(const float* __restrict__ W, int N, int K, const int32_t* __restrict__ perm,
                                   int b_d, uint16_t* __restrict__ scale, uint16_t* __restrict__ offset) {
  const int n = (int)((blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
  if (n >= N) return;
  const int G = K / 8;
  const float* Wr = W + (size_t)n * K;
  double lo = INFINITY, hi = -INFINITY;
  for (int g = lane; g < G; g += 32) {
    double sq = 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int col = perm ? perm[8 * g + i] : 8 * g + i;
      const double v = (double)Wr[col];
      const double p = __dmul_rn(v, v);
      sq = i == 0 ? p : __dadd_rn(sq, p);
    }
    const double nr = __dsqrt_rn(sq);
    lo = fmin(lo, nr);
    hi = fmax(hi, nr);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fmin(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
    hi = fmax(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
  }
  if (lane == 0) {
    const int levels = (1 << (10 - b_d)) - 1;
    const double sc = levels > 0 ? __ddiv_rn(__dsub_rn(hi, lo), (double)levels) : 0.0;
    scale[n] = f64_to_f16_rne(sc);
    offset[n] = f64_to_f16_rne(lo);
  }
}

// ---------------------------------------------------------------- encoder
// One warp per row, one lane per subvector (chunks of 32 subvectors).  For
// each subvector the exact error of a candidate (d, c) is
//   X(d, c) = sum_i e_i (a_i - r_c c_{d,i})^2,   a_i = |w_i|,
// formed term by term (product r_c c, difference, e * diff * diff, running
// sum, i ascending).  Evaluating X for all 1024 (d, c) pairs costs 40 fp64
// operations each; instead a filter
//   F(d, c) = E - 2 r_c D_d + r_c^2 Q_d,   E = sum e a^2, D_d = sum e a c, Q_d = sum e c^2
// (two FMAs per pair) is computed with a rigorous bound |F - X| <= delta_d:
// both differ from the real-valued error by at most 26u (E + r^2 Q) (X: the
// product, difference and square of each term plus an 8-term sum) and 24u
// (E + r^2 Q) (F: the three sums and two FMAs, using 2|r| D <= E + r^2 Q by
// Cauchy-Schwarz), u = 2^-53; delta_d = 2^-47 (E + rmax^2 Q_d) (64u) covers
// both.  The pairs are scanned in the order (d ascending, then c ascending)
// keeping M = the least F + delta seen so far; a pair is evaluated exactly
// only when F - delta <= M, and the best exact value wins on a strict
// improvement.  A skipped pair has X >= F - delta > M >= min X, so it can
// neither win nor tie; the exact minimiser always passes the test; the scan
// order makes the lowest (d, c) win a tie.  The result is the brute-force
// choice, bit for bit.
constexpr int kEncWarps = 8;
constexpr double kFilterRel = 0x1p-47;
constexpr double kFilterAbs = 1e-290;     // covers underflow in products of tiny values

struct EncodeArgs {
  const float* W;              // [N][K] natural column order
  const int32_t* perm;         // [K] or null
  const float* weights;        // [K] natural order, or null (all 1)
  const uint16_t* codebook;    // fp16 [2^b_d][8]
  const uint16_t* scale;       // fp16 [N] (affine radius), or
  const uint16_t* offset;      // fp16 [N]
  const uint16_t* lut;         // fp16 [N][2^b_r] per-row radius table (when not null)
  uint8_t* canonical;          // [N][row_bytes]
  double* row_err;             // [N] or null
  int N, K, b_d;
  size_t row_bytes;
};

template <int BR>
__global__ void __launch_bounds__(kEncWarps * 32, 1) encode_kernel(const EncodeArgs a) {
  constexpr int NR = 1 << BR;
  constexpr bool kRegR = NR <= 16;              // radius levels in registers, else in shared memory
  extern __shared__ double smem_d[];
  const int BD = a.b_d, nd = 1 << BD;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  double* cbd = smem_d;                          // [nd][8] codeword entries
  double* cb2 = cbd + (size_t)nd * 8;            // [nd][8] their squares
  double* rts = cb2 + (size_t)nd * 8 + (size_t)warp * (kRegR ? 0 : NR);
  __shared__ uint32_t codes_s[kEncWarps][32];
  for (int i = threadIdx.x; i < nd * 8; i += blockDim.x) {
    const double c = h2d(a.codebook[i]);
    cbd[i] = c;
    cb2[i] = __dmul_rn(c, c);
  }
  __syncthreads();
  const int n = blockIdx.x * kEncWarps + warp;
  if (n >= a.N) return;
  const int G = a.K / 8;
  // radius levels of this row: r_c = fma(scale, c, offset) in fp32, or the table
  // level lut[n][c]; widened exactly
  const uint16_t* lrow = a.lut ? a.lut + ((size_t)n << BR) : nullptr;
  const float scf = lrow ? 0.f : __half2float(__ushort_as_half(a.scale[n]));
  const float off = lrow ? 0.f : __half2float(__ushort_as_half(a.offset[n]));
  auto level = [&](int c) -> double {
    return lrow ? h2d(lrow[c]) : (double)__fmaf_rn(scf, (float)c, off);
  };
  double rr[kRegR ? NR : 1];
  if constexpr (kRegR) {
#pragma unroll
    for (int c = 0; c < NR; ++c) rr[c] = level(c);
  } else {
    for (int c = lane; c < NR; c += 32) rts[c] = level(c);
    __syncwarp();
  }
  auto rad = [&](int c) -> double {
    if constexpr (kRegR) return rr[c];
    else return rts[c];
  };
  // the largest r_c^2: at an end of the affine levels (monotone in c), over all table levels
  double rm2 = 0.0;
  if (lrow) {
    for (int c = 0; c < NR; ++c) { const double v = level(c); rm2 = fmax(rm2, __dmul_rn(v, v)); }
  } else {
    const double r_lo = level(0), r_hi = level(NR - 1);
    rm2 = fmax(__dmul_rn(r_lo, r_lo), __dmul_rn(r_hi, r_hi));
  }
  const double rmax2 = rm2 * (1.0 + 0x1p-50);
  const float* Wr = a.W + (size_t)n * a.K;
  double row_acc = 0.0;
  for (int g0 = 0; g0 < G; g0 += 32) {
    const int g = g0 + lane;
    const bool act = g < G;
    double w[8], e[8], av[8], ea[8];
    uint32_t s = 0;
    double E = 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int col = act ? (a.perm ? a.perm[8 * g + i] : 8 * g + i) : 0;
      w[i] = act ? (double)Wr[col] : 0.0;
      e[i] = (act && a.weights) ? (double)a.weights[col] : 1.0;
      if (w[i] < 0.0) s |= 1u << i;
      av[i] = fabs(w[i]);
      ea[i] = e[i] * av[i];
      E = fma(ea[i], av[i], E);
    }
    double M = INFINITY, best = INFINITY;
    int bd = 0, bc = 0;
    for (int d = 0; d < nd; ++d) {
      const double2* cp = reinterpret_cast<const double2*>(cbd + (size_t)d * 8);
      const double2* cq = reinterpret_cast<const double2*>(cb2 + (size_t)d * 8);
      double c[8], D = 0.0, Q = 0.0;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const double2 v = cp[h], v2 = cq[h];
        c[2 * h] = v.x; c[2 * h + 1] = v.y;
        D = fma(ea[2 * h], v.x, D);
        D = fma(ea[2 * h + 1], v.y, D);
        Q = fma(e[2 * h], v2.x, Q);
        Q = fma(e[2 * h + 1], v2.y, Q);
      }
      const double delta = fma(kFilterRel, fma(rmax2, Q, E), kFilterAbs);
      const double h0 = -2.0 * D;
#pragma unroll(kRegR ? NR : 1)
      for (int cc = 0; cc < NR; ++cc) {
        const double r = rad(cc);
        const double F = fma(r, fma(r, Q, h0), E);
        M = fmin(M, F + delta);
        if (F - delta <= M) {
          double X = 0.0;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const double p = __dmul_rn(r, c[i]);
            const double diff = __dsub_rn(av[i], p);
            X = __dadd_rn(X, __dmul_rn(__dmul_rn(e[i], diff), diff));
          }
          if (X < best) { best = X; bd = d; bc = cc; }
        }
      }
    }
    // the chosen code and, for ABS, this subvector's share of
    // sum_j e_j (w_j - What_j)^2 (What exact: a binary32 radius times a binary16 entry)
    double sub = 0.0;
    {
      const double r = rad(bc);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const double wh = __dmul_rn(r, cbd[(size_t)bd * 8 + i]);
        const double diff = __dsub_rn(w[i], ((s >> i) & 1u) ? -wh : wh);
        sub = __dadd_rn(sub, __dmul_rn(e[i], __dmul_rn(diff, diff)));
      }
    }
    if (!act) sub = 0.0;
    codes_s[warp][lane] = act ? (s | ((uint32_t)bd << 8) | ((uint32_t)bc << (8 + BD))) : 0u;
    __syncwarp();
    // chunk bytes: 18 bits per subvector, LSB first; 32 subvectors = 72 bytes
    const int nact = min(32, G - g0);
    const int nbytes = (18 * nact + 7) / 8;
    uint8_t* out = a.canonical + (size_t)n * a.row_bytes + (size_t)g0 * 18 / 8;
    for (int b = lane; b < nbytes; b += 32) {
      const int bit = 8 * b, L = bit / 18, o = bit - 18 * L;
      uint32_t v = codes_s[warp][L] >> o;
      if (o > 10 && L + 1 < 32) v |= codes_s[warp][L + 1] << (18 - o);
      out[b] = (uint8_t)(v & 0xFFu);
    }
    __syncwarp();
    // fixed-order sum of the chunk's 32 shares, then chunks in order
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sub = __dadd_rn(sub, __shfl_xor_sync(0xFFFFFFFFu, sub, o));
    row_acc = g0 == 0 ? sub : __dadd_rn(row_acc, sub);
  }
  if (lane == 0 && a.row_err) a.row_err[n] = row_acc;
}

// ---------------------------------------------------------------- ABS
// totals[k] = sum_n row_err[k][n] (fixed order: thread t sums n = t, t + 1024,
// ... in turn, then a fixed tree), best = the first candidate with the least
// total.
constexpr int kAbsThreads = 1024;
__global__ void __launch_bounds__(kAbsThreads) abs_select_kernel(const double* __restrict__ row_err, int n_cand,
                                                                 int N, double* __restrict__ totals,
                                                                 int32_t* __restrict__ best) {
  __shared__ double part[kAbsThreads];
  __shared__ double tot_s[64];
  for (int k = 0; k < n_cand; ++k) {
    double s = 0.0;
    for (int r = threadIdx.x; r < N; r += kAbsThreads)
      s = r == (int)threadIdx.x ? row_err[(size_t)k * N + r] : __dadd_rn(s, row_err[(size_t)k * N + r]);
    part[threadIdx.x] = s;
    __syncthreads();
    for (int w = kAbsThreads / 2; w > 0; w >>= 1) {
      if ((int)threadIdx.x < w) part[threadIdx.x] = __dadd_rn(part[threadIdx.x], part[threadIdx.x + w]);
      __syncthreads();
    }
    if (threadIdx.x == 0) {
      tot_s[k] = part[0];
      if (totals) totals[k] = part[0];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    int b = 0;
    for (int k = 1; k < n_cand; ++k)
      if (tot_s[k] < tot_s[b]) b = k;
    *best = b;
  }
}

template <int BR>
cudaError_t launch_encode_br(const EncodeArgs& a, cudaStream_t st) {
  constexpr int NR = 1 << BR;
  const size_t smem = (size_t)(2 * 8 << a.b_d) * sizeof(double) + (NR > 16 ? (size_t)kEncWarps * NR * sizeof(double) : 0);
  static std::atomic<bool> attr{false};             // setting it twice is harmless
  if (!attr.load(std::memory_order_acquire)) {
    const cudaError_t e = cudaFuncSetAttribute(encode_kernel<BR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)(160 * 1024));
    if (e != cudaSuccess) return e;
    attr.store(true, std::memory_order_release);
  }
  const int grid = (a.N + kEncWarps - 1) / kEncWarps;
  encode_kernel<BR><<<grid, kEncWarps * 32, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_esg(const float* x, int T, int K, double gamma, double* energy, int32_t* perm, float* weights,
                       cudaStream_t st) {
  const int grid = (K + kCalThreads - 1) / kCalThreads;
  esg_energy_kernel<<<grid, kCalThreads, 0, st>>>(x, T, K, energy);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  esg_perm_kernel<<<grid, kCalThreads, 0, st>>>(energy, K, gamma, perm, weights);
  return cudaGetLastError();
}

cudaError_t launch_radius_grid(const float* W, int N, int K, const int32_t* perm, int b_d, uint16_t* scale,
                               uint16_t* offset, cudaStream_t st) {
  const long long threads = (long long)N * 32;
  const int grid = (int)((threads + kCalThreads - 1) / kCalThreads);
  radius_grid_kernel<<<grid, kCalThreads, 0, st>>>(W, N, K, perm, b_d, scale, offset);
  return cudaGetLastError();
}

cudaError_t launch_encode(const float* W, int N, int K, int b_d, const int32_t* perm, const float* weights,
                          const uint16_t* codebook, const uint16_t* scale, const uint16_t* offset,
                          const uint16_t* lut, uint8_t* canonical, double* row_err, cudaStream_t st) {
  EncodeArgs a;
  a.W = W; a.perm = perm; a.weights = weights; a.codebook = codebook; a.scale = scale; a.offset = offset;
  a.lut = lut;
  a.canonical = canonical; a.row_err = row_err; a.N = N; a.K = K; a.b_d = b_d;
  a.row_bytes = ((size_t)(K / 8) * 18 + 7) / 8;
  switch (10 - b_d) {
    case 0: return launch_encode_br<0>(a, st);
    case 1: return launch_encode_br<1>(a, st);
    case 2: return launch_encode_br<2>(a, st);
    case 3: return launch_encode_br<3>(a, st);
    case 4: return launch_encode_br<4>(a, st);
    case 5: return launch_encode_br<5>(a, st);
    case 6: return launch_encode_br<6>(a, st);
    case 7: return launch_encode_br<7>(a, st);
    case 8: return launch_encode_br<8>(a, st);
    default: return launch_encode_br<9>(a, st);
  }
}

cudaError_t launch_abs_select(const double* row_err, int n_cand, int N, double* totals, int32_t* best,
                              cudaStream_t st) {
  abs_select_kernel<<<1, kAbsThreads, 0, st>>>(row_err, n_cand, N, totals, best);
  return cudaGetLastError();
}

}  // namespace svq
