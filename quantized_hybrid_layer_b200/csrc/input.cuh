// The stage input: z = h * gamma (the first layer's RMSNorm weight) in block
// fixed point and per-tile sums of squares of h, exactly as the residual
// epilogue of the GEMV writes them (same 128-row tiles, same tile_sumsq), so a
// stage that starts at layer L gives the same bits as the same layers inside a
// longer stage.
#pragma once

#include "qgemv.cuh"

namespace qhl {

// One 128-row tile of h for all NT tokens, by 128 threads (four warps, thread
// = row); red = shared [4] floats; `bar_id` names a barrier over the 128 threads.
template <int NT>
QHL_DEV void input_unit(const float* h, int H, const float* gamma, uint8_t* qz, int qz_stride, float* ss,
                        int ss_stride, int tile, float* red, int bar_id) {
  const int quarter = (threadIdx.x >> 5) & 3, lane = threadIdx.x & 31;
  const int gr = tile * kTileRows + quarter * 32 + lane;   // H is a multiple of 256: every row is valid
  const float g = gamma[gr];
#pragma unroll 1
  for (int t = 0; t < NT; ++t) {
    const float v = h[(size_t)t * H + gr];
    qact_store_block(__fmul_rn(v, g), qz + (size_t)t * qz_stride, tile * 4 + quarter, lane);
    const float s = tile_sumsq(v, red, quarter, lane, bar_id);
    if (quarter == 0 && lane == 0) ss[(size_t)t * ss_stride + tile] = s;
  }
}

}  // namespace qhl
