// sq_layout.h -- index maps of the two packed-weight layouts (host and device).
//
// SQ_LAYOUT_ROWS: row-major arrays (any group size), read by the CUDA-core
// decode kernel.
//
// SQ_LAYOUT_TILES (group size 128): the order in which the tensor-core decode
// kernel streams the weight.  Rows are padded to N16 = roundup(N, 16) and
// channels to K128 = roundup(K, 128) with zeros; tile t = rb * tpr + g covers
// rows [16 rb, 16 rb + 16) and channels [128 g, 128 g + 128), tpr = K128/128.
// Lane L = 4 * gid + q of a warp owns rows r0 = 16 rb + gid and r1 = r0 + 8
// and the 32 channels c = 128 g + 32 q + j, j = 0..31; word w = j / 4 holds
// channels 4w .. 4w + 3.
//   res_q:     tile t is 2048 bytes at 2048 t; lane L's 64 bytes at 64 L are
//              four int8 MMA A fragments (m = 0..3), each four words
//              {r0 word 2m, r1 word 2m, r0 word 2m+1, r1 word 2m+1}.
//   sign/mask: tile t is 64 words at 64 t; lane L's words 2L (row r0) and
//              2L + 1 (row r1).  Channel j of the lane's 32 sits at bit
//              8 * (j % 4) + j / 4, so that the four bits of word w are the
//              top bits of the four bytes of (word << (7 - w)).
//   res_scale: tile t is 16 floats at 16 t, one per row of the row block.
//   alpha:     N16 floats.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define SQ_HD __host__ __device__ __forceinline__
#else
#define SQ_HD inline
#endif

namespace sq {

constexpr int kTileRows = 16;
constexpr int kTileK = 128;

SQ_HD int64_t tiles_rows(int64_t N) { return (N + 15) / 16 * 16; }
SQ_HD int64_t tiles_cols(int64_t K) { return (K + 127) / 128 * 128; }

// Byte offset of code (row, col) in res_q.
SQ_HD int64_t tiled_code_offset(int64_t row, int64_t col, int64_t tpr) {
  const int64_t t = (row >> 4) * tpr + (col >> 7);
  const int rr = (int)(row & 15), cc = (int)(col & 127);
  const int lane = (rr & 7) * 4 + (cc >> 5), j = cc & 31, w = j >> 2;
  return (t * 32 + lane) * 64 + (w >> 1) * 16 + ((w & 1) * 2 + (rr >> 3)) * 4 + (j & 3);
}

// Word index in sign_bits / mask_bits of the 32 channels [32 word, 32 word + 32) of a row.
SQ_HD int64_t tiled_bits_word(int64_t row, int64_t word, int64_t tpr) {
  const int64_t t = (row >> 4) * tpr + (word >> 2);
  const int rr = (int)(row & 15);
  return (t * 32 + (rr & 7) * 4 + (int)(word & 3)) * 2 + (rr >> 3);
}

// Bit position of channel j (0..31) inside a tiled sign / mask word.
SQ_HD int tiled_bit_of(int j) { return 8 * (j & 3) + (j >> 2); }

// Row-order bits (bit j = channel j) -> tiled bit order.
SQ_HD uint32_t tiled_bits_from_row_order(uint32_t b) {
  uint32_t o = 0;
  for (int j = 0; j < 32; ++j) o |= ((b >> j) & 1u) << tiled_bit_of(j);
  return o;
}

// Float index in res_scale of (row, group).
SQ_HD int64_t tiled_scale_index(int64_t row, int64_t g, int64_t tpr) {
  return ((row >> 4) * tpr + g) * 16 + (row & 15);
}

}  // namespace sq
