// Mixer kernels' launch wrappers (DeltaNet step, attention), the stage input
// kernel, weight repacking, dequantisation check, RoPE table and the tiny
// control kernels used by commit / rollback.
#include <algorithm>

#include "launch.h"

namespace qhl {

cudaError_t gemv_prepare_4();
cudaError_t gemv_prepare_8();
cudaError_t launch_gemv_4(int nt, int epi, const GemvArgs& a, int grid, cudaStream_t s, bool pdl);
cudaError_t launch_gemv_8(int nt, int epi, const GemvArgs& a, int grid, cudaStream_t s, bool pdl);
int gemv_smem_4(int nt);
int gemv_smem_8(int nt);

cudaError_t gemv_prepare(int qt) { return qt == kQ4_0 ? gemv_prepare_4() : gemv_prepare_8(); }
cudaError_t launch_gemv(int qt, int nt, int epi, const GemvArgs& a, int grid, cudaStream_t s, bool pdl) {
  if (qt == kQ4_0) return launch_gemv_4(nt, epi, a, grid, s, pdl);
  if (qt == kQ8_0) return launch_gemv_8(nt, epi, a, grid, s, pdl);
  return cudaErrorInvalidValue;
}
int gemv_smem(int qt, int nt) { return qt == kQ4_0 ? gemv_smem_4(nt) : gemv_smem_8(nt); }

#define QHL_NT_CASES(X) X(1) X(2) X(3) X(4) X(5) X(6) X(7) X(8) X(9) X(10) X(11) X(12) X(13) X(14) X(15) X(16)

// ---------------------------------------------------------------------------
// stage input: z = h * gamma (the first layer's RMSNorm weight) in block fixed
// point and per-tile sums of squares of h, exactly as the residual epilogue of
// the GEMV writes them, so a stage that starts at layer L gives the same bits
// as the same layers inside a longer stage.
template <int NT>
__global__ void __launch_bounds__(256) stage_input_kernel(const float* h, int H, const float* gamma, uint8_t* qz,
                                                          int qz_stride, float* ss, int ss_stride) {
  __shared__ float sm[NT * 64];
  if (threadIdx.x == 0) pdl_launch();
  input_unit<NT>(h, H, gamma, qz, qz_stride, ss, ss_stride, blockIdx.x, sm);
}

// f32 rows -> block fixed point, one warp per (token, 32-column block).  The
// GEMV that follows is launched as a programmatic dependent: it may start
// streaming weights at once and waits (griddepcontrol.wait) before reading qx.
__global__ void quantize_rows_kernel(const float* x, int n, int cols, uint8_t* qx) {
  if (threadIdx.x == 0) pdl_launch();
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31, nb = cols / 32;
  if (gw >= (long long)n * nb) return;
  const int t = (int)(gw / nb), b = (int)(gw % nb);
  qact_store_block(x[(size_t)t * cols + b * 32 + lane], qx + (size_t)t * qact_row_bytes(cols), b, lane);
}

cudaError_t launch_quantize_rows(const float* x, int n, int cols, uint8_t* qx, cudaStream_t s) {
  const long long warps = (long long)n * (cols / 32);
  quantize_rows_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, s>>>(x, n, cols, qx);
  return cudaGetLastError();
}

// Hidden state at the stage boundary in binary16 (the peers' wire format):
// widened to f32 exactly on the way in, rounded to nearest even on the way out.
__global__ void hidden_from_f16_kernel(const __half* in, float* out, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    out[i] = __half2float(in[i]);
}

__global__ void hidden_to_f16_kernel(const float* in, __half* out, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    out[i] = __float2half_rn(in[i]);
}

static unsigned elementwise_blocks(int n) { return (unsigned)std::min((n + 255) / 256, 148 * 8); }

cudaError_t launch_hidden_from_f16(const void* in, float* out, int n, cudaStream_t s) {
  hidden_from_f16_kernel<<<elementwise_blocks(n), 256, 0, s>>>(static_cast<const __half*>(in), out, n);
  return cudaGetLastError();
}

cudaError_t launch_hidden_to_f16(const float* in, void* out, int n, cudaStream_t s) {
  hidden_to_f16_kernel<<<elementwise_blocks(n), 256, 0, s>>>(in, static_cast<__half*>(out), n);
  return cudaGetLastError();
}

__global__ void commit_kernel(int* ctrl, int n_accepted, int n_dn, int ring);

// Full shared-memory carveout for every stage kernel (see gemv_q4.cu), and the
// attention kernel's dynamic shared-memory limit.
template <typename K>
static cudaError_t max_carveout(K k) {
  return cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
}

cudaError_t mixers_prepare(int rep) {
  cudaError_t e = cudaSuccess;
#define P(N)                                                                                            \
  if (e == cudaSuccess)                                                                                 \
    e = cudaFuncSetAttribute(attn_partial_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize,        \
                             attn_smem_bytes<N>(rep));                                                  \
  if (e == cudaSuccess) e = max_carveout(attn_partial_kernel<N>);                                       \
  if (e == cudaSuccess) e = max_carveout(attn_combine_kernel<N>);                                       \
  if (e == cudaSuccess) e = max_carveout(dn_step_kernel<N>);                                            \
  if (e == cudaSuccess) e = max_carveout(stage_input_kernel<N>);
  QHL_NT_CASES(P)
#undef P
  if (e == cudaSuccess) e = max_carveout(commit_kernel);
  return e;
}

cudaError_t launch_dn_step(int nt, const DnArgs& a, int grid, cudaStream_t s, bool pdl) {
  switch (nt) {
#define C(N) case N: return launch_ex(dn_step_kernel<N>, dim3(grid), dim3(256), 0, s, pdl, a);
    QHL_NT_CASES(C)
#undef C
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attn_partial(int nt, const AttnArgs& a, int nchunk, int hkv, cudaStream_t s, bool pdl) {
  const int rep = a.Hq / a.Hkv;
  switch (nt) {
#define C(N)                                                                                               \
  case N:                                                                                                  \
    return launch_ex(attn_partial_kernel<N>, dim3(nchunk, hkv, (N + kAttGroup - 1) / kAttGroup), dim3(256),    \
                     (size_t)attn_smem_bytes<N>(rep), s, pdl, a);
    QHL_NT_CASES(C)
#undef C
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attn_combine(int nt, const AttnArgs& a, cudaStream_t s, bool pdl) {
  switch (nt) {
#define C(N) case N: return launch_ex(attn_combine_kernel<N>, dim3(N * a.Hq), dim3(256), (size_t)3 * a.nchunk * 4, s, pdl, a);
    QHL_NT_CASES(C)
#undef C
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_stage_input(int nt, const float* h, int H, const float* gamma, uint8_t* qz, int qz_stride,
                               float* ss, int ss_stride, cudaStream_t s) {
  switch (nt) {
#define C(N) case N: return launch_ex(stage_input_kernel<N>, dim3(H / 64), dim3(256), 0, s, false, h, H, gamma, qz, qz_stride, ss, ss_stride);
    QHL_NT_CASES(C)
#undef C
    default: return cudaErrorInvalidValue;
  }
}

// ---------------------------------------------------------------------------
// GGUF array-of-structs blocks -> packed items (layout in qpack.cuh).
// One thread per (item, block, tile row).  Rows past the matrix are filled
// with zero weights.  paired: tile rows 0..31 come from a (features t*32..),
// rows 32..63 from b (the same features), for the SwiGLU epilogue.
__global__ void repack_kernel(int qt, const uint8_t* a, const uint8_t* b, int rows, int paired, int tiles,
                              int chunks, uint8_t* out) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)tiles * chunks * 512) return;
  const long long item = idx / 512;
  const int rem = (int)(idx % 512), blk = rem / 64, r = rem % 64;
  const int t = (int)(item / chunks), c = (int)(item % chunks);
  const int h = r / 32, lane = r % 32;
  const uint8_t* src = a;
  int srow;
  if (paired) {
    srow = t * 32 + lane;
    src = h ? b : a;
  } else {
    srow = t * 64 + r;
  }
  const bool valid = srow < rows;
  const int bb = gguf_block_bytes(qt);
  const long long nb = (long long)chunks * kChunkBlocks;
  const uint8_t* sp = src + (valid ? ((long long)srow * nb + (long long)c * kChunkBlocks + blk) * bb : 0);
  uint8_t* base = out + item * item_bytes(qt);
  if (qt == kQ4_0) {
    uint8_t* q = base + ((blk * 2 + h) * 32 + lane) * 16;
    for (int i = 0; i < 16; ++i) q[i] = valid ? sp[2 + i] : 0x88;
    uint8_t* s = base + 8192 + (blk * 32 + lane) * 4 + h * 2;
    s[0] = valid ? sp[0] : 0;
    s[1] = valid ? sp[1] : 0;
  } else {
    for (int half = 0; half < 2; ++half) {
      uint8_t* q = base + (((blk * 2 + half) * 2 + h) * 32 + lane) * 16;
      for (int i = 0; i < 16; ++i) q[i] = valid ? sp[2 + 16 * half + i] : 0;
    }
    uint8_t* s = base + 16384 + (blk * 32 + lane) * 4 + h * 2;
    s[0] = valid ? sp[0] : 0;
    s[1] = valid ? sp[1] : 0;
  }
}

cudaError_t launch_repack(int qt, const uint8_t* a, const uint8_t* b, int rows, int cols, uint8_t* out,
                          cudaStream_t s) {
  const bool paired = b != nullptr;
  const int tiles = packed_tiles(rows, paired), chunks = cols / kChunkCols;
  const long long n = (long long)tiles * chunks * 512;
  repack_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(qt, a, b, rows, paired ? 1 : 0, tiles, chunks, out);
  return cudaGetLastError();
}

// Dequantise rows of a packed matrix with the GEMV's conversion (q4_word /
// q8_word) times the f16 scale: one thread per (row, block).
__global__ void dequant_kernel(int qt, const uint8_t* P, int rows, int cols, int paired, int row0, int nrows,
                               float* out) {
  const int nb = cols / 32;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)nrows * nb) return;
  const int r = row0 + (int)(idx / nb), kb = (int)(idx % nb);
  int tile, h, lane;
  if (paired) {
    const int f = r % rows;
    h = r / rows;
    tile = f / 32;
    lane = f % 32;
  } else {
    tile = r / 64;
    h = (r % 64) / 32;
    lane = r % 32;
  }
  const int chunks = cols / kChunkCols, c = kb / kChunkBlocks, blk = kb % kChunkBlocks;
  const uint8_t* base = P + ((size_t)tile * chunks + c) * item_bytes(qt);
  const int qb = qt == kQ4_0 ? 8192 : 16384;
  const uint16_t sbits = *reinterpret_cast<const uint16_t*>(base + qb + (blk * 32 + lane) * 4 + h * 2);
  const float d = __half2float(__ushort_as_half(sbits));
  float w[32];
  if (qt == kQ4_0) {
    const uint4 wv = *reinterpret_cast<const uint4*>(base + ((blk * 2 + h) * 32 + lane) * 16);
    const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
    for (int i = 0; i < 4; ++i) {
      float2 p[4];
      q4_word(ws[i], p);
      w[4 * i] = p[0].x;
      w[4 * i + 1] = p[0].y;
      w[4 * i + 2] = p[1].x;
      w[4 * i + 3] = p[1].y;
      w[16 + 4 * i] = p[2].x;
      w[17 + 4 * i] = p[2].y;
      w[18 + 4 * i] = p[3].x;
      w[19 + 4 * i] = p[3].y;
    }
  } else {
    for (int half = 0; half < 2; ++half) {
      const uint4 wv = *reinterpret_cast<const uint4*>(base + (((blk * 2 + half) * 2 + h) * 32 + lane) * 16);
      const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
      for (int i = 0; i < 4; ++i) {
        float2 p[2];
        q8_word(ws[i], p);
        w[16 * half + 4 * i] = p[0].x;
        w[16 * half + 4 * i + 1] = p[0].y;
        w[16 * half + 4 * i + 2] = p[1].x;
        w[16 * half + 4 * i + 3] = p[1].y;
      }
    }
  }
  float* o = out + (size_t)(r - row0) * cols + kb * 32;
  for (int e = 0; e < 32; ++e) o[e] = __fmul_rn(w[e], d);
}

cudaError_t launch_dequant(int qt, const uint8_t* packed, int rows, int cols, int paired, int row0, int nrows,
                           float* out, cudaStream_t s) {
  const long long n = (long long)nrows * (cols / 32);
  if (n <= 0) return cudaSuccess;
  dequant_kernel<<<(unsigned)((n + 127) / 128), 128, 0, s>>>(qt, packed, rows, cols, paired, row0, nrows, out);
  return cudaGetLastError();
}

// cos / sin of p * theta^(-2i/rope_dims) for every position, in double, rounded to f32.
__global__ void rope_table_kernel(float2* tab, int max_ctx, int half, int rope_dims, double theta) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)max_ctx * half) return;
  const int p = (int)(idx / half), i = (int)(idx % half);
  const double ang = (double)p * pow(theta, -2.0 * i / rope_dims);
  double sn, cs;
  sincos(ang, &sn, &cs);
  tab[idx] = make_float2((float)cs, (float)sn);
}

cudaError_t launch_rope_table(float2* tab, int max_ctx, int rope_dims, double theta, cudaStream_t s) {
  const int half = rope_dims / 2;
  const long long n = (long long)max_ctx * half;
  rope_table_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(tab, max_ctx, half, rope_dims, theta);
  return cudaGetLastError();
}

// ctrl[0] = committed length, ctrl[1 + i] = ring index of DeltaNet layer i.
__global__ void commit_kernel(int* ctrl, int n_accepted, int n_dn, int ring) {
  if (threadIdx.x == 0) ctrl[0] += n_accepted;
  for (int i = threadIdx.x; i < n_dn; i += blockDim.x) ctrl[1 + i] = (ctrl[1 + i] + n_accepted) % ring;
}

cudaError_t launch_commit(int* ctrl, int n_accepted, int n_dn, int ring, cudaStream_t s) {
  commit_kernel<<<1, 128, 0, s>>>(ctrl, n_accepted, n_dn, ring);
  return cudaGetLastError();
}

__global__ void set_int_kernel(int* p, int v) { *p = v; }

cudaError_t launch_set_int(int* p, int v, cudaStream_t s) {
  set_int_kernel<<<1, 1, 0, s>>>(p, v);
  return cudaGetLastError();
}

}  // namespace qhl
