// Packed weight layout for the dequant-GEMV and its exact dequantisation.
//
// GGUF blocks arrive as 18-byte (Q4_0) or 34-byte (Q8_0) array-of-structs
// records, which are not 16-byte aligned.  At load they are repacked, once,
// into "items": one item holds 64 output rows x 8 blocks (256 input columns)
// and is one contiguous, 16-byte aligned record that a single bulk copy moves
// into shared memory.  Items are stored tile-major: item (tile t, chunk c) sits
// at index t * chunks + c.  Inside an item, tile row r = h * 32 + lane
// (h = 0, 1) is the row a GEMV lane owns, so every lane's 16-byte reads are
// contiguous across the warp (conflict-free).
//
//  Q4_0 item (9216 B):  nibbles  [block 8][h 2][lane 32][16 B]   (GGUF byte order kept)
//                       scales   [block 8][lane 32][h 2] binary16
//  Q8_0 item (17408 B): quants   [block 8][half 2][h 2][lane 32][16 B]  signed bytes
//                                16*half .. 16*half+15 of the block
//                       scales   [block 8][lane 32][h 2] binary16
//
// A Q4_0 block keeps its GGUF meaning: element j (j < 16) is the low nibble of
// byte j, element j + 16 the high nibble, weight = (nibble - 8) * d.  Q8_0:
// weight = q * d.  (SwarmLLM README: 4-bit values with an f16 scale per block; model
// table "GGUF Q4_0", "GGUF Q8_0 / Q4_0".)
#pragma once

#include "common.cuh"

namespace qhl {

constexpr int kQ4_0 = 2;
constexpr int kQ8_0 = 8;
constexpr int kTileRows = 64;
constexpr int kChunkBlocks = 8;
constexpr int kChunkCols = kChunkBlocks * 32;

template <int QT> struct QLayout;
template <> struct QLayout<kQ4_0> {
  static constexpr int kQuantBytes = 8192;   // per item
  static constexpr int kItemBytes = 9216;
  static constexpr int kGgufBlock = 18;
};
template <> struct QLayout<kQ8_0> {
  static constexpr int kQuantBytes = 16384;
  static constexpr int kItemBytes = 17408;
  static constexpr int kGgufBlock = 34;
};

inline __host__ __device__ int item_bytes(int qt) { return qt == kQ4_0 ? 9216 : 17408; }
inline __host__ __device__ int gguf_block_bytes(int qt) { return qt == kQ4_0 ? 18 : 34; }

// Exact nibble/byte -> float conversion.  A masked field OR'ed into the bit
// pattern of 2^23 is the float 2^23 + field * 2^s; one packed FMA scales it by
// 2^-s and subtracts 2^(23-s) + offset, which is exact (the result is a small
// integer), so the dequantised quant is bit-exact before the f16 scale is
// applied.
constexpr uint32_t kMagic = 0x4B000000u;   // bit pattern of 2^23

// (a & MASK) | magic in one LOP3 (the mask is an immediate, the magic a
// register), reinterpreted as a float.
template <uint32_t MASK>
QHL_DEV float magic_field(uint32_t a, uint32_t magic) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "n"(MASK), "r"(magic));
  return __uint_as_float(d);
}

// Q4_0: the 32-bit word i (bytes 4i .. 4i+3) of a block holds elements
// 4i, 4i+16, 4i+1, 4i+17, 4i+2, 4i+18, 4i+3, 4i+19 in its eight nibbles.
// Returns them as (q-8) pairs: p[0] = (e4i, e4i+1), p[1] = (e4i+2, e4i+3),
// p[2] = (e4i+16, e4i+17), p[3] = (e4i+18, e4i+19).
QHL_DEV void q4_word(uint32_t w, float2 p[4]) {
  const float2 s_lo = make_float2(1.0f, 0.00390625f);          // 1, 2^-8
  const float2 c_lo = make_float2(-8388616.0f, -32776.0f);     // -(2^23+8), -(2^15+8)
  const float2 s_hi = make_float2(0.0625f, 0.000244140625f);   // 2^-4, 2^-12
  const float2 c_hi = make_float2(-524296.0f, -2056.0f);       // -(2^19+8), -(2^11+8)
  const uint32_t m = kMagic;
  const uint32_t w2 = w >> 16;
  p[0] = ffma2(make_float2(magic_field<0x000Fu>(w, m), magic_field<0x0F00u>(w, m)), s_lo, c_lo);
  p[1] = ffma2(make_float2(magic_field<0x000Fu>(w2, m), magic_field<0x0F00u>(w2, m)), s_lo, c_lo);
  p[2] = ffma2(make_float2(magic_field<0x00F0u>(w, m), magic_field<0xF000u>(w, m)), s_hi, c_hi);
  p[3] = ffma2(make_float2(magic_field<0x00F0u>(w2, m), magic_field<0xF000u>(w2, m)), s_hi, c_hi);
}

// Q8_0: word i holds signed elements 4i .. 4i+3.
// p[0] = (e4i, e4i+1), p[1] = (e4i+2, e4i+3) as signed integers (the sign
// bits are flipped to offset binary, q + 128, before the mask-or).
QHL_DEV void q8_word(uint32_t w_signed, float2 p[2]) {
  const float2 s = make_float2(1.0f, 0.00390625f);
  const float2 c = make_float2(-8388736.0f, -32896.0f);        // -(2^23+128), -(2^15+128)
  const uint32_t m = kMagic;
  const uint32_t w = w_signed ^ 0x80808080u;
  const uint32_t w2 = w >> 16;
  p[0] = ffma2(make_float2(magic_field<0x00FFu>(w, m), magic_field<0xFF00u>(w, m)), s, c);
  p[1] = ffma2(make_float2(magic_field<0x00FFu>(w2, m), magic_field<0xFF00u>(w2, m)), s, c);
}

}  // namespace qhl
