// repack.cu -- canonical stream -> device layout, its inverse (field export)
// and the bit-exact dense dequantisation.
//
// One thread owns one lane-block (4 rows x 16 subvectors, 144 bytes); see
// layout.cuh.  These kernels run once per matrix (repack) or in tests and
// exports (unpack, dequantize), so they favour plainness over speed.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "layout.cuh"
#include "svq_internal.h"

namespace svq {
namespace {

// Read an 18-bit code word: stream bits [18g, 18g+18) of one row segment.
__device__ __forceinline__ uint32_t read_code(const uint8_t* seg, int g) {
  const int bit = 18 * g;
  const int byte = bit >> 3, sh = bit & 7;
  // 18 bits starting at bit `sh` span at most 4 bytes (sh + 18 <= 25).
  uint32_t v = (uint32_t)seg[byte] | ((uint32_t)seg[byte + 1] << 8) | ((uint32_t)seg[byte + 2] << 16);
  if (sh + 18 > 24) v |= (uint32_t)seg[byte + 3] << 24;
  return (v >> sh) & 0x3FFFFu;
}


// Build the 36 words of a lane-block from 64 (signs, payload) pairs,
// indexed [j][r] (subvector j of the block, row r of the lane).
__device__ void build_words(const uint8_t s[16][4], const uint32_t p[16][4], uint32_t w[kWords]) {
  for (int j = 0; j < 16; ++j) {
    uint32_t S = 0;
    for (int r = 0; r < 4; ++r)
      for (int q = 0; q < 4; ++q) {
        const int t = 4 * r + q;
        S |= (uint32_t)((s[j][r] >> (2 * q)) & 1u) << (15 - t);
        S |= (uint32_t)((s[j][r] >> (2 * q + 1)) & 1u) << (31 - t);
      }
    w[j] = S;
  }
  for (int k = 0; k < 20; ++k) w[16 + k] = 0;
  for (int v = 0; v < 64; ++v) {
    const uint32_t pay = p[v >> 2][v & 3];
    if (v < 60) {
      w[16 + v / 3] |= pay << (10 * (v % 3));
    } else {
      const int a = v - 60;
      for (int i = 0; i < 5; ++i) w[16 + 5 * a + i] |= ((pay >> (8 - 2 * i)) & 3u) << 30;
    }
  }
}

__device__ void split_words(const uint32_t w[kWords], uint8_t s[16][4], uint32_t p[16][4]) {
  for (int j = 0; j < 16; ++j)
    for (int r = 0; r < 4; ++r) {
      uint32_t sv = 0;
      for (int q = 0; q < 4; ++q) {
        const int t = 4 * r + q;
        sv |= ((w[j] >> (15 - t)) & 1u) << (2 * q);
        sv |= ((w[j] >> (31 - t)) & 1u) << (2 * q + 1);
      }
      s[j][r] = (uint8_t)sv;
    }
  for (int v = 0; v < 64; ++v) {
    uint32_t pay;
    if (v < 60) {
      pay = (w[16 + v / 3] >> (10 * (v % 3))) & 0x3FFu;
    } else {
      const int a = v - 60;
      pay = 0;
      for (int i = 0; i < 5; ++i) pay |= (w[16 + 5 * a + i] >> 30) << (8 - 2 * i);
    }
    p[v >> 2][v & 3] = pay;
  }
}

struct LaneBlockId {
  int t, b, l;
  bool valid;
};

// Enumerate lane-blocks: tiles in order, blocks, lanes.  Full tiles have 32
// lanes; the last tile may have fewer.
__device__ LaneBlockId lane_block_id(int N, int K, long long id) {
  const int B = K / kBlockCols;
  const int full = N / kTileRows;
  const long long per_full = (long long)B * 32;
  LaneBlockId r;
  if (id < (long long)full * per_full) {
    r.t = (int)(id / per_full);
    const long long rem = id % per_full;
    r.b = (int)(rem / 32);
    r.l = (int)(rem % 32);
    r.valid = true;
    return r;
  }
  const long long rem = id - (long long)full * per_full;
  const int L = tile_lanes(N, full);
  r.t = full;
  if (L == 0 || rem >= (long long)B * L) { r.valid = false; r.b = r.l = 0; return r; }
  r.b = (int)(rem / L);
  r.l = (int)(rem % L);
  r.valid = true;
  return r;
}

__device__ __forceinline__ long long num_lane_blocks(int N, int K) {
  return (long long)(N / kRowsPerLane) * (K / kBlockCols);
}

__global__ void repack_kernel(const uint8_t* __restrict__ canon, int N, int K, int b_d,
                              uint8_t* __restrict__ out) {
  const int Np = pad_rows(N), Kp = pad_cols(K), G = K / 8;
  const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= num_lane_blocks(Np, Kp)) return;
  const LaneBlockId lb = lane_block_id(Np, Kp, id);
  if (!lb.valid) return;
  const size_t rb = ((size_t)G * 18 + 7) / 8;         // canonical row bytes
  uint8_t s[16][4];
  uint32_t p[16][4];
  for (int r = 0; r < 4; ++r) {
    const int n = lb.t * kTileRows + 4 * lb.l + r;
    const uint8_t* seg = canon + (size_t)n * rb + (size_t)lb.b * 36;   // 16 codes = 36 bytes
    for (int j = 0; j < 16; ++j) {
      // padding (row >= N or subvector >= K/8): a zero code
      const uint32_t code = (n < N && lb.b * 16 + j < G) ? read_code(seg, j) : 0u;
      s[j][r] = (uint8_t)(code & 0xFFu);
      p[j][r] = code >> 8;                              // idx | radius << b_d
    }
  }
  (void)b_d;
  uint32_t w[kWords];
  build_words(s, p, w);
  for (int c = 0; c < kChunks; ++c) {
    uint4 v = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
    *reinterpret_cast<uint4*>(out + chunk_offset(Np, Kp, lb.t, lb.b, c, lb.l)) = v;
  }
  // A GEMV launched next on the stream may start (programmatic dependent launch)
  // as soon as every block of this grid has exited, and it reads the packed codes
  // before it waits for this grid: make the stores visible before exiting.
  __threadfence();
}

// (N, K: the padded layout dimensions)
__device__ void load_words(const uint8_t* packed, int N, int K, const LaneBlockId& lb, uint32_t w[kWords]) {
  for (int c = 0; c < kChunks; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(packed + chunk_offset(N, K, lb.t, lb.b, c, lb.l));
    w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
  }
}

__global__ void unpack_kernel(const uint8_t* __restrict__ packed, int N, int K, int b_d,
                              uint8_t* __restrict__ signs, uint16_t* __restrict__ idx,
                              uint16_t* __restrict__ code) {
  const int Np = pad_rows(N), Kp = pad_cols(K);
  const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= num_lane_blocks(Np, Kp)) return;
  const LaneBlockId lb = lane_block_id(Np, Kp, id);
  if (!lb.valid) return;
  uint32_t w[kWords];
  load_words(packed, Np, Kp, lb, w);
  uint8_t s[16][4];
  uint32_t p[16][4];
  split_words(w, s, p);
  const int G = K / 8;
  const uint32_t imask = (1u << b_d) - 1u;
  for (int r = 0; r < 4; ++r) {
    const int n = lb.t * kTileRows + 4 * lb.l + r;
    if (n >= N) break;
    for (int j = 0; j < 16; ++j) {
      if (lb.b * 16 + j >= G) break;
      const size_t f = (size_t)n * G + (size_t)lb.b * 16 + j;
      signs[f] = s[j][r];
      idx[f] = (uint16_t)(p[j][r] & imask);
      code[f] = (uint16_t)(p[j][r] >> b_d);
    }
  }
}

// Dense export, bit-exact: r = fmaf(scale, code, offset); w = RNE(r * c) in the
// output format; sign bit set from the code afterwards.
__global__ void dequant_kernel(const uint8_t* __restrict__ packed, int N, int K, int b_d,
                               const uint16_t* __restrict__ codebook,
                               const uint16_t* __restrict__ scale, const uint16_t* __restrict__ offset,
                               const uint16_t* __restrict__ lut, int out_bf16, uint16_t* __restrict__ out) {
  const int Np = pad_rows(N), Kp = pad_cols(K), G = K / 8;
  const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= num_lane_blocks(Np, Kp)) return;
  const LaneBlockId lb = lane_block_id(Np, Kp, id);
  if (!lb.valid) return;
  uint32_t w[kWords];
  load_words(packed, Np, Kp, lb, w);
  uint8_t s[16][4];
  uint32_t p[16][4];
  split_words(w, s, p);
  const uint32_t imask = (1u << b_d) - 1u;
  for (int r = 0; r < 4; ++r) {
    const int n = lb.t * kTileRows + 4 * lb.l + r;
    if (n >= N) break;
    const float sc = lut ? 0.f : __half2float(__ushort_as_half(scale[n]));
    const float of = lut ? 0.f : __half2float(__ushort_as_half(offset[n]));
    for (int j = 0; j < 16; ++j) {
      if (lb.b * 16 + j >= G) break;
      const uint32_t id_ = p[j][r] & imask;
      const uint32_t cd = p[j][r] >> b_d;
      // the quantized radius: per-row table level, or the affine form
      const float rad = lut ? __half2float(__ushort_as_half(lut[((size_t)n << (10 - b_d)) + cd]))
                            : __fmaf_rn(sc, (float)cd, of);
      uint16_t vals[8];
      for (int i = 0; i < 8; ++i) {
        const float c = __half2float(__ushort_as_half(codebook[id_ * 8 + i]));
        const float prod = __fmul_rn(rad, c);
        uint16_t bits = out_bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(prod))
                                 : __half_as_ushort(__float2half_rn(prod));
        if ((s[j][r] >> i) & 1u) bits ^= 0x8000u;
        vals[i] = bits;
      }
      uint4 v;
      v.x = vals[0] | ((uint32_t)vals[1] << 16);
      v.y = vals[2] | ((uint32_t)vals[3] << 16);
      v.z = vals[4] | ((uint32_t)vals[5] << 16);
      v.w = vals[6] | ((uint32_t)vals[7] << 16);
      *reinterpret_cast<uint4*>(out + (size_t)n * K + (size_t)lb.b * kBlockCols + 8 * j) = v;
    }
  }
}

inline unsigned grid_for(long long work, int threads) {
  return (unsigned)((work + threads - 1) / threads);
}

}  // namespace

cudaError_t launch_repack(const uint8_t* canon, int N, int K, int b_d, void* out, cudaStream_t st) {
  const long long work = (long long)(pad_rows(N) / kRowsPerLane) * (pad_cols(K) / kBlockCols);
  repack_kernel<<<grid_for(work, 128), 128, 0, st>>>(canon, N, K, b_d, (uint8_t*)out);
  return cudaGetLastError();
}

cudaError_t launch_unpack(const void* packed, int N, int K, int b_d, uint8_t* signs, uint16_t* idx,
                          uint16_t* code, cudaStream_t st) {
  const long long work = (long long)(pad_rows(N) / kRowsPerLane) * (pad_cols(K) / kBlockCols);
  unpack_kernel<<<grid_for(work, 128), 128, 0, st>>>((const uint8_t*)packed, N, K, b_d, signs, idx, code);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const void* packed, int N, int K, int b_d, const uint16_t* codebook,
                           const uint16_t* scale, const uint16_t* offset, const uint16_t* lut, int out_bf16,
                           uint16_t* out, cudaStream_t st) {
  const long long work = (long long)(pad_rows(N) / kRowsPerLane) * (pad_cols(K) / kBlockCols);
  dequant_kernel<<<grid_for(work, 128), 128, 0, st>>>((const uint8_t*)packed, N, K, b_d, codebook, scale,
                                                      offset, lut, out_bf16, out);
  return cudaGetLastError();
}

}  // namespace svq
