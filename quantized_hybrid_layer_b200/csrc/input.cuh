// The stage input: z = h * gamma (the first layer's RMSNorm weight) in block
// fixed point and per-tile sums of squares of h, exactly as the residual
// epilogue of the GEMV writes them, so a stage that starts at layer L gives the
// same bits as the same layers inside a longer stage.
#pragma once

#include "qact.cuh"

namespace qhl {

// One 64-row tile of h for all NT tokens; sm = shared [NT * 64] f32.
// Called by 256 threads (8 warps).
template <int NT>
QHL_DEV void input_unit(const float* h, int H, const float* gamma, uint8_t* qz, int qz_stride, float* ss,
                        int ss_stride, int tile, float* sm) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int idx = threadIdx.x; idx < NT * 64; idx += 256) {
    const int t = idx >> 6, gr = tile * 64 + (idx & 63);
    sm[idx] = h[(size_t)t * H + gr];
  }
  named_sync(1, 256);
  for (int p = warp; p < NT * 2; p += 8) {
    const int t = p >> 1, b = p & 1, gr = tile * 64 + b * 32 + lane;
    qact_store_block(__fmul_rn(sm[t * 64 + b * 32 + lane], gamma[gr]), qz + (size_t)t * qz_stride, tile * 2 + b, lane);
  }
  if (threadIdx.x < NT) ss[(size_t)threadIdx.x * ss_stride + tile] = sumsq64(sm + threadIdx.x * 64);
  named_sync(1, 256);   // sm reusable by the caller
}

}  // namespace qhl
