// Block fixed-point form of GEMV inputs ("q24 blocks").
//
// A projection input x (a normalised hidden state, a mixer output or the
// SwiGLU product) is consumed block by block, 32 columns at a time, against
// 4-bit or 8-bit integer weights.  Its producer stores each 32-value block as
//     x_j ~= s * X_j,   s = 2^(E - 22),   X_j = rint(x_j / s) in [-(2^23-1), 2^23-1]
// where 2^E <= max_j |x_j| < 2^(E+1).  s is a power of two, so x_j / s is
// exact and only the rounding to an integer loses anything: at most s/2, i.e.
// 2^-23 of the block's largest value, the same relative step as f32 rounding.
// X_j is split into three bytes, X = 65536 * hi + 256 * mid + lo (hi signed,
// mid and lo unsigned), so the GEMV forms
//     sum_j q_j X_j = 65536 * sum q hi + 256 * sum q mid + sum q lo
// from byte dot products (dp4a) in exact int32 arithmetic, followed by a fixed
// sequence of f32 operations.  The integer partial sums are exact, so their
// grouping never changes a bit and every token count gives the same result.
// For the Q4_0 offset (q - 8) the block also stores sum_j hi_j and
// sum_j (256 * mid_j + lo_j).
//
// Layout, per token, per chunk of 256 columns (8 blocks), 864 bytes:
//   [0, 256)    hi bytes,  block b at b*32 + j
//   [256, 512)  mid bytes, block b at 256 + b*32 + j
//   [512, 768)  lo bytes,  block b at 512 + b*32 + j
//   [768, 800)  s per block (f32)
//   [800, 832)  sum_j hi_j per block (int32)
//   [832, 864)  sum_j (256 mid_j + lo_j) per block (int32)
// A token row of K columns is K/256 * 864 bytes.
#pragma once

#include "common.cuh"

namespace qhl {

constexpr int kQChunkBytes = 864;

__host__ __device__ inline size_t qact_row_bytes(int cols) { return (size_t)(cols / 256) * kQChunkBytes; }

// Quantise one 32-value block held one value per lane (lane j = element j)
// and store it as block `blk` (global block index) of the token row at `row`.
QHL_DEV void qact_store_block(float v, uint8_t* row, int blk, int lane) {
  const float m = warp_max(fabsf(v));
  int E = (int)((__float_as_uint(m) >> 23) & 0xFFu) - 127;     // exponent of the block max (0 / subnormal -> -127)
  E = max(E, -100);
  const float up = __uint_as_float((uint32_t)(127 + 22 - E) << 23);   // 2^(22 - E)
  int X = __float2int_rn(__fmul_rn(v, up));
  X = max(-8388607, min(8388607, X));
  const int hi = X >> 16;                  // arithmetic shift: -128 .. 127
  const int ml = X & 0xFFFF;               // 256 * mid + lo, 0 .. 65535
  uint8_t* base = row + (size_t)(blk >> 3) * kQChunkBytes;
  const int b = blk & 7;
  base[b * 32 + lane] = (uint8_t)(hi & 0xFF);
  base[256 + b * 32 + lane] = (uint8_t)(ml >> 8);
  base[512 + b * 32 + lane] = (uint8_t)(ml & 0xFF);
  const int s_hi = __reduce_add_sync(0xffffffffu, hi);
  const int s_ml = __reduce_add_sync(0xffffffffu, ml);
  if (lane == 0) {
    reinterpret_cast<float*>(base + 768)[b] = __uint_as_float((uint32_t)(127 + E - 22) << 23);   // s = 2^(E - 22)
    reinterpret_cast<int*>(base + 800)[b] = s_hi;
    reinterpret_cast<int*>(base + 832)[b] = s_ml;
  }
}

// dp4a flavours: signed x signed, unsigned x unsigned, signed x unsigned.
QHL_DEV int dp4a_ss(uint32_t a, uint32_t b, int c) { return __dp4a((int)a, (int)b, c); }
QHL_DEV int dp4a_uu(uint32_t a, uint32_t b, int c) { return (int)__dp4a(a, b, (unsigned)c); }
QHL_DEV int dp4a_su(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

}  // namespace qhl
