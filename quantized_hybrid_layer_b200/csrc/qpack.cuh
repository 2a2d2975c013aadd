// Packed weight layout for the dequant-GEMV and its exact dequantisation.
//
// GGUF blocks arrive as 18-byte (Q4_0) or 34-byte (Q8_0) array-of-structs
// records, which are not 16-byte aligned.  At load they are repacked, once,
// into "items": one item holds 128 output rows x 8 blocks (256 input columns)
// and is one contiguous, 16-byte aligned record that two bulk copies move into
// shared memory (the quants, then the scales).  Items are stored tile-major:
// item (tile t, chunk c) sits at index t * chunks + c.  Inside an item the
// thread that owns row r (one thread per row, the row's tensor-memory lane)
// reads 16 contiguous bytes per block, and a warp's 32 rows are 512 contiguous
// bytes (conflict-free shared-memory reads):
//
//  Q4_0 item (18432 B):  quants  [block 8][row 128][16 B]          GGUF byte order
//                        scales  [row 128][block 8] binary16        at 16384
//  Q8_0 item (34816 B):  quants  [block 8][half 2][row 128][16 B]  signed bytes,
//                                half h holds elements 16h .. 16h+15
//                        scales  [row 128][block 8] binary16        at 32768
//
// A Q4_0 block keeps its GGUF meaning: element j (j < 16) is the low nibble of
// byte j, element j + 16 the high nibble, weight = (nibble - 8) * d.  Q8_0:
// weight = q * d.  (SwarmLLM README: 4-bit values with an f16 scale per block;
// model table "GGUF Q4_0", "GGUF Q8_0 / Q4_0".)  Gate and up projections are
// packed as pairs: rows 0..63 of a tile are gate features 64t .. 64t+63, rows
// 64..127 the up rows of the same features, for the SwiGLU epilogue.
#pragma once

#include "common.cuh"

namespace qhl {

constexpr int kQ4_0 = 2;
constexpr int kQ8_0 = 8;
constexpr int kTileRows = 128;
constexpr int kChunkBlocks = 8;
constexpr int kChunkCols = kChunkBlocks * 32;

template <int QT> struct QLayout;
template <> struct QLayout<kQ4_0> {
  static constexpr int kQuantBytes = 16384;   // per item
  static constexpr int kScaleBytes = 2048;
  static constexpr int kItemBytes = 18432;
  static constexpr int kGgufBlock = 18;
};
template <> struct QLayout<kQ8_0> {
  static constexpr int kQuantBytes = 32768;
  static constexpr int kScaleBytes = 2048;
  static constexpr int kItemBytes = 34816;
  static constexpr int kGgufBlock = 34;
};

inline __host__ __device__ int item_bytes(int qt) { return qt == kQ4_0 ? 18432 : 34816; }
inline __host__ __device__ int item_quant_bytes(int qt) { return qt == kQ4_0 ? 16384 : 32768; }
inline __host__ __device__ int gguf_block_bytes(int qt) { return qt == kQ4_0 ? 18 : 34; }

// Offset of row r's 16 quant bytes of block b (half h: Q8_0 only) in an item.
inline __host__ __device__ int q4_off(int b, int r) { return (b * kTileRows + r) * 16; }
inline __host__ __device__ int q8_off(int b, int h, int r) { return ((b * 2 + h) * kTileRows + r) * 16; }
inline __host__ __device__ int scale_off(int qt, int b, int r) { return item_quant_bytes(qt) + r * 16 + b * 2; }

// One Q4_0 block of one row (16 bytes, GGUF order) as the 32 unsigned bytes
// 0..15 the integer MMA takes for elements 0..31: word i of the result holds
// elements 4i .. 4i+3 (byte j of word i = element 4i + j).  The low nibbles of
// the 16 bytes are elements 0..15, the high nibbles elements 16..31.
QHL_DEV void q4_unpack(const uint4 w, uint32_t (&a)[8]) {
  a[0] = w.x & 0x0F0F0F0Fu;
  a[1] = w.y & 0x0F0F0F0Fu;
  a[2] = w.z & 0x0F0F0F0Fu;
  a[3] = w.w & 0x0F0F0F0Fu;
  a[4] = (w.x >> 4) & 0x0F0F0F0Fu;
  a[5] = (w.y >> 4) & 0x0F0F0F0Fu;
  a[6] = (w.z >> 4) & 0x0F0F0F0Fu;
  a[7] = (w.w >> 4) & 0x0F0F0F0Fu;
}

}  // namespace qhl
