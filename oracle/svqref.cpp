// svqref.cpp -- CPU oracle for SAGE spherical vector quantization (SVQ).
//
// TEST INFRASTRUCTURE ONLY.  This file is the independent, slow, obviously
// correct definition that the CUDA library is checked against.  Only the test
// suite, the smoke check and the benchmark's CPU-baseline leg may load it; the
// product path never does.  It shares no code, header, table or helper with the
// CUDA sources.
//
// What it follows ("SAGE: Pushing 2-Bit Vector-Quantized LLMs toward Real-World
// Usability", arXiv 2610.14745):
//   * Figure 2 caption: every weight subvector is encoded by signs, a direction
//     index and a quantized radius, 18 bits per eight weights, with a per-matrix
//     split of the 10 non-sign bits between direction index and radius (ABS).
//   * Figure 6 caption: the kernel multiplies by eight reordered activations
//     (the ESG permutation), x_sub = x[perm[8g .. 8g+7]].
//   * Figure 1 / Figure 5 captions: weights are reconstructed on demand, i.e.
//     the layer computes y = W x with W decoded from the codes.
// The pages print no bit layout, sign convention or radius formula; the
// readings used here (bit order, sign bit meaning, affine per-row radius,
// rounding of the exported fp16/bf16 weights) are listed with the code below.
//
// Every routine is a plain loop; floating point is IEEE fp32 where the format
// fixes it (the radius and the exported weights) and fp64 everywhere else.
// Build: g++ -O2 -std=c++17 -fopenmp -ffp-contract=off -fPIC -shared.

#include <cmath>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <cstdint>
#include <cstring>
#include <vector>

extern "C" {

// ---------------------------------------------------------------------------
// IEEE 754 binary16 and bfloat16 conversions, written from the definitions.
// ---------------------------------------------------------------------------

// binary16 -> binary32.  Exact: every binary16 value is a binary32 value.
float svqref_h2f(uint16_t h) {
  const int sign = h >> 15;
  const int e = (h >> 10) & 0x1f;
  const int m = h & 0x3ff;
  double v;
  if (e == 0x1f) {
    if (m) return std::nanf("");
    v = INFINITY;
  } else if (e == 0) {
    v = std::ldexp((double)m, -24);                 // subnormal: m * 2^-24
  } else {
    v = std::ldexp((double)(1024 + m), e - 25);     // (1 + m/1024) * 2^(e-15)
  }
  return (float)(sign ? -v : v);
}

// bfloat16 -> binary32: the bfloat16 bits are the top half of a binary32.
float svqref_bf2f(uint16_t b) {
  const int sign = b >> 15;
  const int e = (b >> 7) & 0xff;
  const int m = b & 0x7f;
  double v;
  if (e == 0xff) {
    if (m) return std::nanf("");
    v = INFINITY;
  } else if (e == 0) {
    v = std::ldexp((double)m, -133);                // subnormal: m * 2^-133
  } else {
    v = std::ldexp((double)(128 + m), e - 134);     // (1 + m/128) * 2^(e-127)
  }
  return (float)(sign ? -v : v);
}

// Round a non-negative finite double to the nearest multiple of `ulp`
// (a power of two), ties to the even multiple.  Exact in double for the
// inputs used here (binary32 values and power-of-two spacings).
static double round_to_grid_rne(double a, double ulp) {
  const double q = a / ulp;          // exact: division by a power of two
  const double fl = std::floor(q);
  const double frac = q - fl;        // exact
  double r = fl;
  if (frac > 0.5) r = fl + 1.0;
  else if (frac == 0.5) r = (std::fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
  return r * ulp;
}

// Generic round-to-nearest-even into a binary format with `mant` stored
// mantissa bits, exponent bias `bias` and `ebits` exponent bits.  Returns the
// bit pattern.  NaN maps to a quiet NaN with the input's sign.
static uint16_t encode_rne(float x, int mant, int bias, int ebits) {
  const uint32_t sign = std::signbit(x) ? 1u : 0u;
  const uint32_t emax_field = (1u << ebits) - 1u;
  const uint16_t sbit = (uint16_t)(sign << (mant + ebits));
  if (std::isnan(x)) return (uint16_t)(sbit | (emax_field << mant) | (1u << (mant - 1)));
  const double a = std::fabs((double)x);
  if (std::isinf(x)) return (uint16_t)(sbit | (emax_field << mant));
  if (a == 0.0) return sbit;
  const int emin = 1 - bias;                         // smallest normal exponent
  int E;
  std::frexp(a, &E);                                 // a in [2^(E-1), 2^E)
  int e = E - 1;
  if (e < emin) e = emin;                            // subnormal range shares emin's spacing
  const double ulp = std::ldexp(1.0, e - mant);
  const double r = round_to_grid_rne(a, ulp);
  // Largest finite value: (2 - 2^-mant) * 2^emax.
  const int emax = (int)emax_field - 1 - bias;
  if (r >= std::ldexp(1.0, emax + 1)) return (uint16_t)(sbit | (emax_field << mant));
  if (r == 0.0) return sbit;
  // Encode the (exactly representable) rounded value.
  int Er;
  std::frexp(r, &Er);
  const int er = Er - 1;
  if (er < emin) {
    const uint32_t m = (uint32_t)(r / std::ldexp(1.0, emin - mant));   // subnormal
    return (uint16_t)(sbit | m);
  }
  const uint32_t m = (uint32_t)(r / std::ldexp(1.0, er - mant)) - (1u << mant);
  const uint32_t field = (uint32_t)(er + bias);
  return (uint16_t)(sbit | (field << mant) | m);
}

uint16_t svqref_f2h_rne(float x) { return encode_rne(x, 10, 15, 5); }
uint16_t svqref_f2bf_rne(float x) { return encode_rne(x, 7, 127, 8); }

// Array forms (used by the exhaustive conversion pins).
void svqref_f2h_rne_array(const float* x, uint16_t* out, int64_t n) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = svqref_f2h_rne(x[i]);
}
void svqref_f2bf_rne_array(const float* x, uint16_t* out, int64_t n) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = svqref_f2bf_rne(x[i]);
}
void svqref_h2f_array(const uint16_t* h, float* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = svqref_h2f(h[i]);
}

// ---------------------------------------------------------------------------
// The canonical code stream (Figure 2 caption: 18 bits per eight weights).
//
// Reading of the layout (the pages give only the bit count and the three
// fields): row n of an N x K matrix starts at byte n * row_bytes with
// row_bytes = ceil(18 * (K/8) / 8).  Subvector g of the row occupies stream
// bits [18g, 18g + 18); stream bit b is bit (b mod 8) of byte floor(b/8)
// (least significant bit first).  Inside the 18-bit code word:
//   bits 0..7            sign bits, bit i belongs to element i, 1 = negative
//   bits 8..8+b_d-1      direction index into the codebook (b_d bits)
//   bits 8+b_d..17       radius code (b_r = 10 - b_d bits)
// Pad bits at the end of a row are zero when written and ignored when read.
// ---------------------------------------------------------------------------

int64_t svqref_row_bytes(int K) { return ((int64_t)(K / 8) * 18 + 7) / 8; }

static uint32_t read_bits(const uint8_t* row, int64_t bit, int nbits) {
  uint32_t v = 0;
  for (int k = 0; k < nbits; ++k) {
    const int64_t b = bit + k;
    v |= (uint32_t)((row[b >> 3] >> (b & 7)) & 1u) << k;
  }
  return v;
}

static void write_bits(uint8_t* row, int64_t bit, int nbits, uint32_t v) {
  for (int k = 0; k < nbits; ++k) {
    const int64_t b = bit + k;
    const uint8_t mask = (uint8_t)(1u << (b & 7));
    if ((v >> k) & 1u) row[b >> 3] |= mask;
    else row[b >> 3] &= (uint8_t)~mask;
  }
}

// Pack per-subvector fields [N][K/8] into the canonical stream (N*row_bytes).
// Returns 0, or -1 if a field does not fit its width.
int svqref_pack(int N, int K, int b_d, const uint8_t* signs, const uint16_t* idx,
                const uint16_t* code, uint8_t* out) {
  const int G = K / 8, b_r = 10 - b_d;
  const int64_t rb = svqref_row_bytes(K);
  std::memset(out, 0, (size_t)(N * rb));
  for (int n = 0; n < N; ++n) {
    uint8_t* row = out + n * rb;
    for (int g = 0; g < G; ++g) {
      const int64_t f = (int64_t)n * G + g;
      if (idx[f] >> b_d) return -1;
      if (b_r < 16 && (code[f] >> b_r)) return -1;
      const uint32_t word = (uint32_t)signs[f] | ((uint32_t)idx[f] << 8) |
                            ((uint32_t)code[f] << (8 + b_d));
      write_bits(row, (int64_t)g * 18, 18, word);
    }
  }
  return 0;
}

// Unpack the canonical stream into per-subvector fields [N][K/8].
void svqref_unpack(int N, int K, int b_d, const uint8_t* in, uint8_t* signs, uint16_t* idx,
                   uint16_t* code) {
  const int G = K / 8;
  const int64_t rb = svqref_row_bytes(K);
  for (int n = 0; n < N; ++n) {
    const uint8_t* row = in + n * rb;
    for (int g = 0; g < G; ++g) {
      const int64_t f = (int64_t)n * G + g;
      const int64_t bit = (int64_t)g * 18;
      signs[f] = (uint8_t)read_bits(row, bit, 8);
      idx[f] = (uint16_t)read_bits(row, bit + 8, b_d);
      code[f] = (uint16_t)read_bits(row, bit + 8 + b_d, 10 - b_d);
    }
  }
}

// ---------------------------------------------------------------------------
// Radius (Figure 2 caption: "a quantized radius").  Reading: per-row affine
// dequantisation r = offset_n + scale_n * code with fp16 scale and offset,
// evaluated in binary32 with one rounding (a fused multiply-add).
// ---------------------------------------------------------------------------
float svqref_radius(uint16_t scale_h, uint16_t offset_h, uint32_t code) {
  return std::fmaf(svqref_h2f(scale_h), (float)code, svqref_h2f(offset_h));
}

// Radius of (row n, code) under either form of the quantized radius: the
// affine pair above, or (lut != NULL) a per-row table of 2^b_r fp16 levels,
// r = fp32(lut[n][code]) -- the levels the pages optimise ("SAGE", Figure 2
// caption: a quantized radius; the pages fit the levels, not a formula).
static float row_radius(const uint16_t* scale, const uint16_t* offset, const uint16_t* lut, int b_d, int n,
                        uint32_t code) {
  if (lut) return svqref_h2f(lut[((size_t)n << (10 - b_d)) + code]);
  return svqref_radius(scale[n], offset[n], code);
}

// Exact decoded weights in fp64, W[n][j] in the stored (permuted) column
// order: W[n][8g+i] = (-1)^{s_i} * r * c_{idx,i}.  The product of a binary32
// radius and a binary16 codebook entry is exact in fp64.
void svqref_decode_exact(int N, int K, int b_d, const uint8_t* canon, const uint16_t* codebook,
                         const uint16_t* scale, const uint16_t* offset, const uint16_t* lut, double* W) {
  const int G = K / 8;
  std::vector<uint8_t> s((size_t)N * G);
  std::vector<uint16_t> id((size_t)N * G), cd((size_t)N * G);
  svqref_unpack(N, K, b_d, canon, s.data(), id.data(), cd.data());
  // rows are independent: decoded in parallel (the values do not depend on the thread count)
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    for (int g = 0; g < G; ++g) {
      const int64_t f = (int64_t)n * G + g;
      const double r = (double)row_radius(scale, offset, lut, b_d, n, cd[f]);
      for (int i = 0; i < 8; ++i) {
        const double c = (double)svqref_h2f(codebook[(size_t)id[f] * 8 + i]);
        const double w = r * c;
        W[(int64_t)n * K + 8 * g + i] = ((s[f] >> i) & 1u) ? -w : w;
      }
    }
  }
}

// Exported low-precision weights (the bit-exact dequantisation).
//   fp16: w16 = RNE_fp16(r * c) with the product in binary32, then the sign
//         bit is set from the code (so a zero component may become -0).
//   bf16: same, rounding the binary32 product to bfloat16.
// out_kind: 0 = fp16, 1 = bf16.  Output bit patterns [N][K].
void svqref_dequant(int N, int K, int b_d, const uint8_t* canon, const uint16_t* codebook,
                    const uint16_t* scale, const uint16_t* offset, const uint16_t* lut, int out_kind,
                    uint16_t* out) {
  const int G = K / 8;
  std::vector<uint8_t> s((size_t)N * G);
  std::vector<uint16_t> id((size_t)N * G), cd((size_t)N * G);
  svqref_unpack(N, K, b_d, canon, s.data(), id.data(), cd.data());
  for (int n = 0; n < N; ++n) {
    for (int g = 0; g < G; ++g) {
      const int64_t f = (int64_t)n * G + g;
      const float r = row_radius(scale, offset, lut, b_d, n, cd[f]);
      for (int i = 0; i < 8; ++i) {
        const float c = svqref_h2f(codebook[(size_t)id[f] * 8 + i]);
        const float p = r * c;                              // one binary32 rounding
        uint16_t bits = out_kind == 0 ? svqref_f2h_rne(p) : svqref_f2bf_rne(p);
        if ((s[f] >> i) & 1u) bits = (uint16_t)(bits ^ 0x8000u);
        out[(int64_t)n * K + 8 * g + i] = bits;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// The layer (Figure 6 caption: eight reordered activations per subvector;
// Figures 1 and 5: weights reconstructed on demand).
//   y[m][n] = sum_j W[n][j] * x[m][perm[j]]          (fp64)
//   den[m][n] = sum_j |W[n][j]| * |x[m][perm[j]]|     (error scale)
// x holds M rows of K 16-bit values; x_kind 0 = fp16, 1 = bf16.
// ---------------------------------------------------------------------------
void svqref_linear(int N, int K, int b_d, const uint8_t* canon, const uint16_t* codebook,
                   const uint16_t* scale, const uint16_t* offset, const uint16_t* lut, const int32_t* perm,
                   const uint16_t* x, int x_kind, int M, double* y, double* den) {
  std::vector<double> W((size_t)N * K);
  svqref_decode_exact(N, K, b_d, canon, codebook, scale, offset, lut, W.data());
  std::vector<double> xp((size_t)M * K);
  for (int m = 0; m < M; ++m)
    for (int j = 0; j < K; ++j) {
      const uint16_t v = x[(int64_t)m * K + perm[j]];
      xp[(size_t)m * K + j] = (double)(x_kind == 0 ? svqref_h2f(v) : svqref_bf2f(v));
    }
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    const double* w = W.data() + (size_t)n * K;
    for (int m = 0; m < M; ++m) {
      const double* xr = xp.data() + (size_t)m * K;
      double acc = 0.0, mag = 0.0;
      for (int j = 0; j < K; ++j) {
        acc += w[j] * xr[j];
        mag += std::fabs(w[j]) * std::fabs(xr[j]);
      }
      y[(int64_t)m * N + n] = acc;
      if (den) den[(int64_t)m * N + n] = mag;
    }
  }
}

// ---------------------------------------------------------------------------
// Brute-force encoder (test tool).  Figure 2 caption: the fit is weighted by
// activation energies.  Reading: sign s_i = (w_i < 0); then the joint argmin
// over (idx, code) of sum_i e_i (|w_i| - r_code * c_{idx,i})^2 in fp64, with
// r_code the dequantised radius of this row.  Ties go to the lowest idx, then
// the lowest code.  energy may be NULL (all weights 1).
// ---------------------------------------------------------------------------
void svqref_encode(int N, int K, int b_d, const double* W, const uint16_t* codebook,
                   const uint16_t* scale, const uint16_t* offset, const uint16_t* lut, const double* energy,
                   uint8_t* signs, uint16_t* idx, uint16_t* code) {
  const int G = K / 8, b_r = 10 - b_d;
  const int n_dir = 1 << b_d, n_rad = 1 << b_r;
  std::vector<double> cb((size_t)n_dir * 8);
  for (int e = 0; e < n_dir * 8; ++e) cb[e] = (double)svqref_h2f(codebook[e]);
  for (int n = 0; n < N; ++n) {
    std::vector<double> rad(n_rad);
    for (int c = 0; c < n_rad; ++c) rad[c] = (double)row_radius(scale, offset, lut, b_d, n, c);
    for (int g = 0; g < G; ++g) {
      const double* w = W + (int64_t)n * K + 8 * g;
      const double* e = energy ? energy + 8 * g : nullptr;
      uint8_t s = 0;
      for (int i = 0; i < 8; ++i)
        if (w[i] < 0.0) s = (uint8_t)(s | (1u << i));
      double best = INFINITY;
      int bi = 0, bc = 0;
      for (int d = 0; d < n_dir; ++d) {
        for (int c = 0; c < n_rad; ++c) {
          double err = 0.0;
          for (int i = 0; i < 8; ++i) {
            const double diff = std::fabs(w[i]) - rad[c] * cb[(size_t)d * 8 + i];
            err += (e ? e[i] : 1.0) * diff * diff;
          }
          if (err < best) { best = err; bi = d; bc = c; }
        }
      }
      const int64_t f = (int64_t)n * G + g;
      signs[f] = s;
      idx[f] = (uint16_t)bi;
      code[f] = (uint16_t)bc;
    }
  }
}

int svqref_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// Thread count of the later parallel loops (timing only: results do not depend
// on it, every output is computed by one thread in a fixed order).
void svqref_set_threads(int n) {
#ifdef _OPENMP
  omp_set_num_threads(n > 0 ? n : 1);
#else
  (void)n;
#endif
}

}  // extern "C"
