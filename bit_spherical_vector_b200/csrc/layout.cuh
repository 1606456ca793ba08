// layout.cuh -- the device layout of packed SVQ codes (written by svq_repack).
//
// The canonical interchange stream stores, per row, one 18-bit code word per
// subvector of eight weights (8 sign bits, a b_d-bit direction index and a
// b_r = 10 - b_d bit radius code; "SAGE", arXiv 2610.14745, Figure 2 caption).
// The device layout keeps exactly those bits (N*K*9/32 bytes) but regroups them
// so that a warp streams them with 16-byte coalesced loads and a thread can
// pull every field out with one shift and one mask:
//
//   tile      = 128 consecutive rows (the last tile may hold fewer; rows % 4 == 0)
//   block     = 16 consecutive subvectors of every row of a tile (128 columns)
//   Shapes whose N is not a multiple of 4 or whose K is not a multiple of 128
//   are stored padded to Np = 4 ceil(N / 4) rows and Kp = 128 ceil(K / 128)
//   columns with zero codes; the kernels read activation columns >= K as zero
//   and write no output row >= N, so the padding never contributes.
//   lane-block= 4 rows x 16 subvectors = 64 codes = 1152 bits = 144 bytes
//               = 9 x 16-byte chunks, owned by one lane of a warp
//   A tile with L lanes (L = rows/4) stores its blocks in order; inside a block
//   chunk c of lane l sits at byte (c * L + l) * 16, so each chunk index is one
//   contiguous, fully coalesced warp load.
//
// The 36 32-bit words of a lane-block (chunk c holds words 4c .. 4c+3):
//   words 0..15   sign word of subvector j (j = 0..15) for the lane's 4 rows:
//                 for row r and element pair q (elements 2q, 2q+1), t = 4r + q:
//                 bit (15 - t) = sign of element 2q, bit (31 - t) = sign of 2q+1.
//                 Shifting the word left by t puts the pair's two signs on the
//                 sign bits of an fp16x2 pair.
//   words 16..35  payload words P[0..19]; payload = idx | code << b_d (10 bits)
//                 of subvector v = 4j + r:
//                   v < 60 : bits [10*(v%3), 10*(v%3)+10) of P[v/3]
//                   v >= 60: a = v - 60; bits 30..31 of P[5a+i] hold payload
//                            bits (8-2i), (9-2i), i = 0..4.
#pragma once
#include <cstddef>
#include <cstdint>

namespace svq {

constexpr int kTileRows = 128;
constexpr int kRowsPerLane = 4;
constexpr int kGroupsPerBlock = 16;
constexpr int kBlockCols = kGroupsPerBlock * 8;   // 128 input columns per block
constexpr int kLaneBlockBytes = 144;
constexpr int kChunks = 9;
constexpr int kWords = 36;

__host__ __device__ inline int num_tiles(int N) { return (N + kTileRows - 1) / kTileRows; }

__host__ __device__ inline int tile_lanes(int N, int t) {
  const int rows = N - t * kTileRows;
  return (rows >= kTileRows ? kTileRows : rows) / kRowsPerLane;
}

// Byte offset of tile t: every full tile holds 128 * K * 9/32 = 36 K bytes.
__host__ __device__ inline size_t tile_offset(int K, int t) { return (size_t)t * 36 * (size_t)K; }

// Byte offset of chunk c of lane l of block b in tile t.
__host__ __device__ inline size_t chunk_offset(int N, int K, int t, int b, int c, int l) {
  const int L = tile_lanes(N, t);
  return tile_offset(K, t) + (size_t)b * L * kLaneBlockBytes + ((size_t)c * L + l) * 16;
}

// Padded layout dimensions (equal to N and K for the aligned shapes).
__host__ __device__ inline int pad_rows(int N) { return (N + kRowsPerLane - 1) / kRowsPerLane * kRowsPerLane; }
__host__ __device__ inline int pad_cols(int K) { return (K + kBlockCols - 1) / kBlockCols * kBlockCols; }

__host__ __device__ inline bool layout_supported(int N, int K) {
  return N > 0 && K > 0 && K % 8 == 0;
}

// Bytes of the device layout: exactly N * K * 9 / 32 for aligned shapes, the
// padded Np * Kp * 9 / 32 otherwise.
__host__ __device__ inline size_t packed_bytes(int N, int K) {
  return (size_t)pad_rows(N) * (size_t)pad_cols(K) * 9 / 32;
}

}  // namespace svq
