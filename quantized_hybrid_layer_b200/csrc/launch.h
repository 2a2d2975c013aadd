// Host-side launch wrappers for the stage kernels (one translation unit per
// kernel family; the runtime only sees these declarations).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "attention.cuh"
#include "deltanet.cuh"
#include "input.cuh"
#include "pass.cuh"
#include "qgemv.cuh"

namespace qhl {

// cudaLaunchKernelEx with an optional programmatic-dependent-launch attribute:
// the kernel may start while the previous kernel on the stream is still
// running; it must call griddepcontrol.wait before reading that kernel's output.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// GEMV: qt in {2, 8}, nt in 1..16, epi in {EPI_STORE, EPI_SWIGLU, EPI_RESID}.
cudaError_t gemv_prepare(int qt);   // sets the dynamic shared-memory limit of every instantiation
cudaError_t launch_gemv(int qt, int nt, int epi, const GemvArgs& a, int grid, cudaStream_t s, bool pdl);
int gemv_smem(int qt, int nt);

cudaError_t mixers_prepare(int rep);   // rep = query heads per KV head
cudaError_t launch_dn_step(int nt, const DnArgs& a, int grid, cudaStream_t s, bool pdl);
cudaError_t launch_attn_partial(int nt, const AttnArgs& a, int nchunk, int hkv, cudaStream_t s, bool pdl);
cudaError_t launch_attn_combine(int nt, const AttnArgs& a, cudaStream_t s, bool pdl);
cudaError_t launch_stage_input(int nt, const float* h, int H, const float* gamma, uint8_t* qz, int qz_stride,
                               float* ss, int ss_stride, cudaStream_t s);
cudaError_t launch_quantize_rows(const float* x, int n, int cols, uint8_t* qx, cudaStream_t s);
cudaError_t launch_hidden_from_f16(const void* in, float* out, int n, cudaStream_t s);   // binary16 -> f32
cudaError_t launch_hidden_to_f16(const float* in, void* out, int n, cudaStream_t s);     // f32 -> binary16 (RNE)

cudaError_t launch_repack(int qt, const uint8_t* a, const uint8_t* b, int rows, int cols, uint8_t* out,
                          cudaStream_t s);
cudaError_t launch_dequant(int qt, const uint8_t* packed, int rows, int cols, int paired, int row0, int nrows,
                           float* out, cudaStream_t s);
cudaError_t launch_rope_table(float2* tab, int max_ctx, int rope_dims, double theta, cudaStream_t s);
cudaError_t launch_commit(int* ctrl, int n_accepted, int n_dn, int ring, cudaStream_t s);
cudaError_t launch_set_int(int* p, int v, cudaStream_t s);

// Persistent pass (pass.cuh, instantiated in pass.cu for n_tok 1..kPassMaxTok).
cudaError_t pass_prepare(int qt);
cudaError_t pass_occupancy(int qt, int nt, int* blocks);   // co-resident CTAs per SM (0: not instantiated)
cudaError_t launch_pass(int qt, int nt, const PassArgs& p, cudaStream_t s);

// CTAs that own items of a tiles x chunks GEMV on `cap` CTAs (one per SM).
// When the CTAs can own whole tiles -- a divisor of `tiles` no smaller than
// 85% of `cap` -- no tile is split and no stream-K fix-up runs (the gate/up
// projection of the 27B shape: 272 tiles on 136 of 148 CTAs); otherwise a
// balanced stream-K split over min(cap, items) CTAs.  Depends on the shape
// and `cap` only, never on the token count.
inline int gemv_workers(int tiles, int chunks, int cap) {
  if (tiles >= cap)
    for (int w = cap; w * 100 >= cap * 85; --w)
      if (tiles % w == 0) return w;
  const long long items = (long long)tiles * chunks;
  return (int)(items < cap ? items : cap);
}

// packed-layout geometry
inline int packed_tiles(int rows, bool paired) { return paired ? (rows + 63) / 64 : (rows + kTileRows - 1) / kTileRows; }
inline size_t packed_bytes(int qt, int rows, int cols, bool paired) {
  if (rows <= 0 || cols <= 0 || cols % kChunkCols || (qt != kQ4_0 && qt != kQ8_0)) return 0;
  return (size_t)packed_tiles(rows, paired) * (cols / kChunkCols) * item_bytes(qt);
}

}  // namespace qhl
