// layout.cuh -- the device layout of packed SVQ codes (written by svq_repack).
//
// The canonical interchange stream stores, per row, one 18-bit code word per
// subvector of eight weights (8 sign bits, a b_d-bit direction index and a
// b_r = 10 - b_d bit radius code; "SAGE", arXiv 2610.14745, Figure 2 caption).
// The device layout keeps exactly those bits (N*K*9/32 bytes) but regroups them
// so that a warp streams them with 16-byte coalesced loads:
//
//   tile      = 128 consecutive rows (the last tile may hold fewer; rows % 4 == 0)
//   block     = 16 consecutive subvectors of every row of a tile (128 columns)
//   lane-block= 144 bytes = 9 x 16-byte chunks (36 32-bit words) per lane
//   A tile with L lanes (L = rows/4) stores its blocks in order; inside a block
//   chunk c of lane l sits at byte (c * L + l) * 16, so each chunk index is one
//   contiguous, fully coalesced warp load.
//
// Two arrangements of the bits inside a block:
//
// * FULL tiles (128 rows, 32 lanes): the "fragment" arrangement, built for the
//   GEMV's tensor-core dot products (mma.m16n8k16, see gemv_device.cuh).  Lane
//   T owns rows 4T..4T+3 for accumulation.  A block is processed in 16 rounds
//   u = 2*gp + rp (group pair gp = 0..7, row pair rp = 0..1); round u covers
//   groups 2gp, 2gp+1 and, for every lane T, rows 4T+2rp, 4T+2rp+1.  Inside a
//   round the subvector (row 4T + 2rp + e, group 2gp + h) is
//     - accumulated by lane T                          ("owner", e, h in 0..1),
//     - fetched from the codebook with the address given by lane
//         8*(2h + e) + T/4                             ("address lane"),
//     - signed by lanes 4*(T/4) + q, q = 0..3, which hold its elements 2q, 2q+1
//       in tensor-core fragment order                  ("sign holders").
//   Each lane's 36 words hold exactly the bits its three roles need.  A block
//   is also split into four quarters A = 0..3 (rounds 4A..4A+3, groups
//   4A..4A+3, all 128 rows), and the words are ordered so that every quarter
//   has the same shape: chunk 2A holds its four sign words, chunk 2A+1 four of
//   its five payload words and word A of chunk 8 the fifth.
//     sign word S_u of round u (word 8*(u/4) + u%4): for w = 4i + j
//                  (i, j = 0..3), bit 15 - w and bit 31 - w are the signs of
//                  elements 2q and 2q + 1 (q = lane % 4) of the subvector (row
//                  16*(lane/4) + 4i + 2rp + (j & 1), group 2gp + (j >> 1)).
//                  Shifting S_u left by w puts that pair on the sign bits of
//                  an fp16x2 word.
//     payload word P_i (i = 0..19; quarter A = i/5, j = i%5: word 8A + 4 + j
//                  for j < 4, word 32 + A for j = 4): the payload words form a
//                  640-bit stream (bit b = bit b%32 of P_{b/32}); slot k (0..3)
//                  of round u is the 10-bit field at bit
//                  160*(u/4) + 10*(4*(u%4) + k), i.e. bit 40*(u%4) + 10k of the
//                  quarter's own 160 bits P_{5A..5A+4}:
//                    bits 0..b_d-1 : direction index of the subvector whose
//                                    codebook address this lane gives for
//                                    tensor-core product k: row
//                                    16*(l%8) + 4k + 2rp + ((l/8) & 1), group
//                                    2gp + (l/16), l = this lane;
//                    bits b_d..9   : radius code of this lane's own subvector
//                                    (row 4*l + 2rp + (k >> 1), group 2gp + (k & 1)).
// * PARTIAL tiles (fewer than 128 rows): the "owner" arrangement; lane l holds
//   its own 4 rows x 16 subvectors:
//     words 0..15  sign word of subvector j for the lane's 4 rows: for row r
//                  and element pair q, t = 4r + q: bit (15 - t) = sign of
//                  element 2q, bit (31 - t) = sign of 2q+1.
//     words 16..35 payload words P[0..19]; payload = idx | code << b_d (10 bits)
//                  of subvector v = 4j + r:
//                    v < 60 : bits [10*(v%3), 10*(v%3)+10) of P[v/3]
//                    v >= 60: a = v - 60; bits 30..31 of P[5a+i] hold payload
//                             bits (8-2i), (9-2i), i = 0..4.
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

// Byte offset of 32-bit word wi (0..35) of lane l inside a block of a tile with L lanes.
__host__ __device__ inline size_t word_offset_in_block(int L, int l, int wi) {
  return ((size_t)(wi >> 2) * L + l) * 16 + (size_t)(wi & 3) * 4;
}

__host__ __device__ inline bool layout_supported(int N, int K) {
  return N > 0 && K > 0 && N % kRowsPerLane == 0 && K % kBlockCols == 0;
}

__host__ __device__ inline size_t packed_bytes(int N, int K) {
  return (size_t)N * (size_t)K * 9 / 32;
}

// ---------------------------------------------------------------- fragment arrangement (full tiles)
// Round of the subvector (row 4T + r, group j) of a block.
__host__ __device__ constexpr int frag_round(int r, int j) { return 2 * (j >> 1) + (r >> 1); }
// Bit position of slot k of round u in the lane's 640-bit payload stream.
__host__ __device__ constexpr int frag_slot_bit(int u, int k) { return 160 * (u >> 2) + 10 * (4 * (u & 3) + k); }
// Where the fields of the subvector (row 4T + r, group j) of a full-tile block live.
__host__ __device__ inline int frag_code_slot(int r, int j) { return 2 * (r & 1) + (j & 1); }     // in lane T
__host__ __device__ inline int frag_addr_lane(int T, int r, int j) { return 8 * (2 * (j & 1) + (r & 1)) + (T >> 2); }
__host__ __device__ inline int frag_addr_slot(int T) { return T & 3; }
__host__ __device__ inline int frag_sign_lane(int T, int q) { return 4 * (T >> 2) + q; }   // elements 2q, 2q+1
__host__ __device__ inline int frag_sign_pos(int T, int r, int j) { return 4 * (T & 3) + 2 * (j & 1) + (r & 1); }
// Inverse: the subvector (row in tile, group in block) behind a lane's roles in round u.
__host__ __device__ inline int frag_sign_row(int l, int u, int w) {
  return 16 * (l >> 2) + 4 * (w >> 2) + 2 * (u & 1) + (w & 1);
}
__host__ __device__ inline int frag_sign_group(int u, int w) { return 2 * (u >> 1) + ((w >> 1) & 1); }
__host__ __device__ inline int frag_addr_row(int l, int u, int k) { return 16 * (l & 7) + 4 * k + 2 * (u & 1) + ((l >> 3) & 1); }
__host__ __device__ inline int frag_addr_group(int l, int u) { return 2 * (u >> 1) + (l >> 4); }
__host__ __device__ inline int frag_code_row(int l, int u, int k) { return 4 * l + 2 * (u & 1) + (k >> 1); }
__host__ __device__ inline int frag_code_group(int u, int k) { return 2 * (u >> 1) + (k & 1); }

// Word index (0..35) of sign word S_u and of payload word P_i in a full-tile lane-block.
__host__ __device__ constexpr int frag_sign_word(int u) { return 8 * (u >> 2) + (u & 3); }
__host__ __device__ constexpr int frag_payload_word(int i) { return (i % 5) < 4 ? 8 * (i / 5) + 4 + (i % 5) : 32 + i / 5; }

// 10-bit field at bit p of a 640-bit payload stream held in 20 words.
__host__ __device__ inline uint32_t payload_field(const uint32_t* P, int p) {
  const int wi = p >> 5, sh = p & 31;
  uint32_t v = P[wi] >> sh;
  if (sh > 22) v |= P[wi + 1] << (32 - sh);
  return v & 0x3FFu;
}

}  // namespace svq
