// repack.cu -- canonical stream -> device layout, its inverse (field export)
// and the bit-exact dense dequantisation.
//
// In repack and unpack one thread owns one lane-block (4 rows x 16 subvectors,
// 144 bytes; see layout.cuh).  They run once per matrix (repack) or in tests
// and exports (unpack), so they favour plainness over speed; dequantize is
// organised per warp (below) since the GEMM runs it per call.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>

#include "gemm_params.h"
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

// Dense export, bit-exact: r = fmaf(scale, code, offset) (or the row's table
// level); w = RNE(r * c) in the output format; sign bit set from the code
// afterwards.  It also runs on every call of the GEMM's pre-decoded plan, so it
// is written for bandwidth: one warp per (tile, block, row r of the lanes)
// item, dealt round-robin over the CTAs; the 32 lanes load their lane-blocks
// with coalesced 16-byte loads, decode row r of their four into a shared-memory
// stage (rows of 16 x 16 bytes, the column XOR the row, so that both the
// decoders' column writes and the row reads below are conflict free), and the
// warp stores two 256-byte output rows per instruction.
constexpr int kDqWarps = 8;
constexpr int kDqStageU4 = 32 * 16;                 // 32 rows x 16 subvectors of 16 bytes per warp

__device__ __forceinline__ uint32_t payload_of(const uint32_t w[kWords], int v) {
  if (v < 60) return (w[16 + v / 3] >> (10 * (v % 3))) & 0x3FFu;
  const int a = v - 60;
  uint32_t pay = 0;
#pragma unroll
  for (int i = 0; i < 5; ++i) pay |= (w[16 + 5 * a + i] >> 30) << (8 - 2 * i);
  return pay;
}

// One element pair: RNE(r * c) of both halves in the output format (binary32
// products, then one conversion), then the two sign bits of pair t (bit 15 - t:
// low element, bit 31 - t: high element).
template <bool BF16>
__device__ __forceinline__ uint32_t dq_pair(float2 rad2, uint32_t cw, uint32_t S, int t) {
  const float2 pr = __fmul2_rn(rad2, __half22float2(*reinterpret_cast<const __half2*>(&cw)));
  uint32_t bits;
  if constexpr (BF16) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(pr.x, pr.y);
    bits = *reinterpret_cast<const uint32_t*>(&h);
  } else {
    const __half2 h = __floats2half2_rn(pr.x, pr.y);
    bits = *reinterpret_cast<const uint32_t*>(&h);
  }
  return bits ^ ((S << t) & 0x80008000u);
}

// Row R of the lane's four: its 16 subvectors into the lane's stage row.
template <int R, bool BF16, bool LUT>
__device__ __forceinline__ void dq_row(const uint32_t (&w)[kWords], float sc, float of, const uint16_t* lut_row,
                                       int b_d, uint32_t imask, const uint4* cb, uint4* stg_row, int swz) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t pay = payload_of(w, 4 * j + R);
    const uint32_t cd = pay >> b_d;
    float rad;
    if constexpr (LUT) rad = lut_row ? __half2float(__ushort_as_half(__ldg(lut_row + cd))) : 0.f;
    else rad = __fmaf_rn(sc, (float)cd, of);
    const float2 rad2 = make_float2(rad, rad);
    const uint4 cw = cb[pay & imask];
    const uint32_t S = w[j];
    uint4 o;
    o.x = dq_pair<BF16>(rad2, cw.x, S, 4 * R + 0);
    o.y = dq_pair<BF16>(rad2, cw.y, S, 4 * R + 1);
    o.z = dq_pair<BF16>(rad2, cw.z, S, 4 * R + 2);
    o.w = dq_pair<BF16>(rad2, cw.w, S, 4 * R + 3);
    stg_row[j ^ swz] = o;
  }
}

template <bool BF16, bool LUT>
__global__ void __launch_bounds__(kDqWarps * 32, 2)
dequant_kernel(const uint8_t* __restrict__ packed, int N, int K, int b_d, const uint16_t* __restrict__ codebook,
               const uint16_t* __restrict__ scale, const uint16_t* __restrict__ offset,
               const uint16_t* __restrict__ lut, uint16_t* __restrict__ out) {
  extern __shared__ uint4 dq_smem[];
  // In the GEMM's pre-decoded plan this grid follows the activation permute as
  // a programmatic dependent launch and runs beside it (it reads only weights);
  // the GEMM after it may likewise start its prologue early.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int ncw = 1 << b_d;
  uint4* cb = dq_smem;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint4* stg = dq_smem + ncw + warp * kDqStageU4;
  for (int i = threadIdx.x; i < ncw; i += blockDim.x) cb[i] = __ldg(reinterpret_cast<const uint4*>(codebook) + i);
  __syncthreads();
  const int Np = pad_rows(N), Kp = pad_cols(K), G = K / 8, B = Kp / kBlockCols;
  const long long items = (long long)num_tiles(Np) * B * 4;
  const uint32_t imask = (1u << b_d) - 1u;
  const int lut_shift = 10 - b_d;
  for (long long it = blockIdx.x + (long long)warp * gridDim.x; it < items; it += (long long)gridDim.x * kDqWarps) {
    const int r = (int)(it & 3);
    const long long tb = it >> 2;
    const int t = (int)(tb / B), b = (int)(tb % B);
    const int L = tile_lanes(Np, t);
    uint32_t w[kWords];
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (lane < L) v = __ldg(reinterpret_cast<const uint4*>(packed + chunk_offset(Np, Kp, t, b, c, lane)));
      w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
    }
    const int n = t * kTileRows + 4 * lane + r;
    const bool row_ok = lane < L && n < N;
    float sc = 0.f, of = 0.f;
    if (!LUT && row_ok) {
      sc = __half2float(__ushort_as_half(__ldg(scale + n)));
      of = __half2float(__ushort_as_half(__ldg(offset + n)));
    }
    // rows past N (padding, never stored) read no table: a zero radius
    const uint16_t* lut_row = LUT && row_ok ? lut + ((size_t)n << lut_shift) : nullptr;
    uint4* srow = stg + lane * 16;
    const int swz = lane & 15;
    switch (r) {
      case 0: dq_row<0, BF16, LUT>(w, sc, of, lut_row, b_d, imask, cb, srow, swz); break;
      case 1: dq_row<1, BF16, LUT>(w, sc, of, lut_row, b_d, imask, cb, srow, swz); break;
      case 2: dq_row<2, BF16, LUT>(w, sc, of, lut_row, b_d, imask, cb, srow, swz); break;
      default: dq_row<3, BF16, LUT>(w, sc, of, lut_row, b_d, imask, cb, srow, swz); break;
    }
    __syncwarp();
    // rows of lanes 2i and 2i + 1 (output rows 4 lane + r), 16 subvectors each
#pragma unroll 4
    for (int i = 0; i < 16; ++i) {
      const int rl = 2 * i + (lane >> 4), col = lane & 15;
      const int nrow = t * kTileRows + 4 * rl + r;
      const int g = b * 16 + col;
      if (rl < L && nrow < N && g < G)
        *reinterpret_cast<uint4*>(out + (size_t)nrow * K + (size_t)g * 8) = stg[rl * 16 + (col ^ (rl & 15))];
    }
    __syncwarp();
  }
  // Complete only after the grid this one overlapped (the permute): a kernel
  // that waits for this grid then sees both outputs.  No-op in a plain launch.
  asm volatile("griddepcontrol.wait;" ::: "memory");
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

namespace {

template <bool BF16, bool LUT>
cudaError_t launch_dequant_t(const void* packed, int N, int K, int b_d, const uint16_t* codebook,
                             const uint16_t* scale, const uint16_t* offset, const uint16_t* lut, uint16_t* out,
                             bool pdl, cudaStream_t st) {
  const size_t smem = ((size_t)(1 << b_d) + (size_t)kDqWarps * kDqStageU4) * 16;
  static std::atomic<bool> attr_set{false};
  if (!attr_set.load(std::memory_order_acquire)) {
    // the largest codebook (b_d = 10) sets the bound for every launch
    const cudaError_t e = cudaFuncSetAttribute(dequant_kernel<BF16, LUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)(((size_t)1024 + (size_t)kDqWarps * kDqStageU4) * 16));
    if (e != cudaSuccess) return e;
    attr_set.store(true, std::memory_order_release);
  }
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long items = (long long)num_tiles(pad_rows(N)) * (pad_cols(K) / kBlockCols) * 4;
  const long long ctas = std::min<long long>((items + kDqWarps - 1) / kDqWarps, 2LL * sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::max<long long>(1, ctas));
  cfg.blockDim = dim3(kDqWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, dequant_kernel<BF16, LUT>, (const uint8_t*)packed, N, K, b_d,
                                           codebook, scale, offset, lut, out);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

namespace {

cudaError_t dequant_dispatch(const void* packed, int N, int K, int b_d, const uint16_t* codebook,
                             const uint16_t* scale, const uint16_t* offset, const uint16_t* lut, int out_bf16,
                             uint16_t* out, cudaStream_t st, bool pdl) {
  if (out_bf16)
    return lut ? launch_dequant_t<true, true>(packed, N, K, b_d, codebook, scale, offset, lut, out, pdl, st)
               : launch_dequant_t<true, false>(packed, N, K, b_d, codebook, scale, offset, lut, out, pdl, st);
  return lut ? launch_dequant_t<false, true>(packed, N, K, b_d, codebook, scale, offset, lut, out, pdl, st)
             : launch_dequant_t<false, false>(packed, N, K, b_d, codebook, scale, offset, lut, out, pdl, st);
}

}  // namespace

cudaError_t launch_dequant(const void* packed, int N, int K, int b_d, const uint16_t* codebook,
                           const uint16_t* scale, const uint16_t* offset, const uint16_t* lut, int out_bf16,
                           uint16_t* out, cudaStream_t st) {
  return dequant_dispatch(packed, N, K, b_d, codebook, scale, offset, lut, out_bf16, out, st, false);
}

cudaError_t launch_dequant_chained(const void* packed, int N, int K, int b_d, const uint16_t* codebook,
                                   const uint16_t* scale, const uint16_t* offset, const uint16_t* lut, int out_bf16,
                                   uint16_t* out, cudaStream_t st) {
  return dequant_dispatch(packed, N, K, b_d, codebook, scale, offset, lut, out_bf16, out, st, true);
}

}  // namespace svq
