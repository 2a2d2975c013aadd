// Block fixed-point form of GEMV inputs, laid out as the B operand of the
// integer tensor-core MMA.
//
// A projection input x (a normalised hidden state, a mixer output or the
// SwiGLU product) is consumed block by block, 32 columns at a time, against
// 4-bit or 8-bit integer weights.  Its producer stores each 32-value block as
//     x_j ~= s * X_j,   s = 2^(E - 21),   X_j = rint(x_j / s),  |X_j| <= 2^22
// where 2^E <= max_j |x_j| < 2^(E+1).  s is a power of two, so x_j / s is exact
// and only the rounding to an integer loses anything: at most s/2, i.e. 2^-22
// of the block's largest value.  X_j is split into balanced base-256 digits,
//     X = 65536 * hi + 256 * mid + lo,   hi, mid, lo signed bytes,
// (lo = X mod 256 in [-128, 127], then mid likewise, |hi| <= 65), so one MMA
// with the three digit planes as three B rows forms, per weight row, the exact
// int32 sums H = sum q hi, M = sum q mid, L = sum q lo, and
//     sum_j q_j X_j = 65536 H + 256 M + L
// follows by a fixed sequence of f32 operations.  The integer sums are exact,
// so their grouping never changes a bit and every token count gives the same
// result.  For the Q4_0 offset (q - 8) the block also stores
// Sh = sum_j hi_j and Sml = sum_j (256 mid_j + lo_j).
//
// Layout, per token, per chunk of 256 columns (8 blocks), 2048 bytes: block b
// is a 256-byte record at b * 256, one 8-row x 32-byte B tile in the canonical
// K-major layout (rows 16 bytes apart, the second 16 bytes of K 128 bytes on):
//   [0, 16)    hi  of elements 0..15     [128, 144)  hi  of elements 16..31
//   [16, 32)   mid of elements 0..15     [144, 160)  mid of elements 16..31
//   [32, 48)   lo  of elements 0..15     [160, 176)  lo  of elements 16..31
//   [48, 60)   s (f32), Sh (int32), Sml (int32)
// Rows 3..7 of the tile (bytes 48..127 and 176..255) are multiplied too; the
// MMA columns they produce are never read.  A token row of K columns is
// K/256 * 2048 bytes; token t's chunks follow token t-1's, so the tiles of
// consecutive tokens are `qx_stride` bytes apart (the MMA's 8-row-group stride).
#pragma once

#include "common.cuh"

namespace qhl {

constexpr int kQChunkBytes = 2048;
constexpr int kQBlockBytes = 256;
constexpr int kQMetaOff = 48;

__host__ __device__ inline size_t qact_row_bytes(int cols) { return (size_t)(cols / 256) * kQChunkBytes; }

// Quantise one 32-value block held one value per lane (lane j = element j)
// and store it as block `blk` (global block index) of the token row at `row`.
// Called by a whole warp.
QHL_DEV void qact_store_block(float v, uint8_t* row, int blk, int lane) {
  const float m = warp_max(fabsf(v));
  int E = (int)((__float_as_uint(m) >> 23) & 0xFFu) - 127;     // exponent of the block max (0 / subnormal -> -127)
  E = max(E, -100);
  const float up = __uint_as_float((uint32_t)(127 + 21 - E) << 23);   // 2^(21 - E), exact scaling
  int X = __float2int_rn(__fmul_rn(v, up));
  X = max(-4194304, min(4194304, X));
  const int lo = (int)(int8_t)(X & 0xFF);
  const int X1 = (X - lo) >> 8;            // exact: X - lo is a multiple of 256
  const int mid = (int)(int8_t)(X1 & 0xFF);
  const int hi = (X1 - mid) >> 8;
  uint8_t* base = row + (size_t)(blk >> 3) * kQChunkBytes + (blk & 7) * kQBlockBytes + (lane >> 4) * 128 + (lane & 15);
  base[0] = (uint8_t)hi;
  base[16] = (uint8_t)mid;
  base[32] = (uint8_t)lo;
  const int s_hi = __reduce_add_sync(0xffffffffu, hi);
  const int s_ml = __reduce_add_sync(0xffffffffu, X - 65536 * hi);
  if (lane == 0) {
    uint8_t* meta = row + (size_t)(blk >> 3) * kQChunkBytes + (blk & 7) * kQBlockBytes + kQMetaOff;
    reinterpret_cast<float*>(meta)[0] = __uint_as_float((uint32_t)(127 + E - 21) << 23);   // s = 2^(E - 21)
    reinterpret_cast<int*>(meta)[1] = s_hi;
    reinterpret_cast<int*>(meta)[2] = s_ml;
  }
}

}  // namespace qhl
