// Mixer kernels' launch wrappers (DeltaNet step, attention), the stage input
// kernel, weight repacking, dequantisation check, RoPE table and the tiny
// control kernels used by commit / rollback.
#include <algorithm>

#include "launch.h"

namespace qhl {

#define QHL_NT_CASES(X) X(1) X(2) X(3) X(4) X(5) X(6) X(7) X(8) X(9) X(10) X(11) X(12) X(13) X(14) X(15) X(16)

// ---------------------------------------------------------------------------
// stage input: z = h * gamma (the first layer's RMSNorm weight) in block fixed
// point and per-tile sums of squares of h, exactly as the residual epilogue of
// the GEMV writes them (input.cuh), one 128-row tile per CTA of 128 threads.
template <int NT>
__global__ void __launch_bounds__(128) stage_input_kernel(const float* h, int H, const float* gamma, uint8_t* qz,
                                                          int qz_stride, float* ss, int ss_stride) {
  __shared__ float red[4];
  if (threadIdx.x == 0) pdl_launch();
  input_unit<NT>(h, H, gamma, qz, qz_stride, ss, ss_stride, blockIdx.x, red, kBarMix);
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
  if (e == cudaSuccess)                                                                                 \
    e = cudaFuncSetAttribute(attn_combine_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize,        \
                             combine_smem_bytes(kAttMaxCtx / kAttChunk));                                \
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
#define C(N)                                                                                                \
  case N:                                                                                                   \
    return launch_ex(attn_combine_kernel<N>, dim3(N * a.Hq * kCombineParts), dim3(256),                     \
                     (size_t)combine_smem_bytes(a.nchunk), s, pdl, a);
    QHL_NT_CASES(C)
#undef C
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_stage_input(int nt, const float* h, int H, const float* gamma, uint8_t* qz, int qz_stride,
                               float* ss, int ss_stride, cudaStream_t s) {
  switch (nt) {
#define C(N) case N: return launch_ex(stage_input_kernel<N>, dim3(H / kTileRows), dim3(128), 0, s, false, h, H, gamma, qz, qz_stride, ss, ss_stride);
    QHL_NT_CASES(C)
#undef C
    default: return cudaErrorInvalidValue;
  }
}

// ---------------------------------------------------------------------------
// GGUF array-of-structs blocks -> packed items (layout in qpack.cuh).
// One thread per (item, block, tile row).  Rows past the matrix get zero
// weights (Q4_0 nibbles 8, Q8_0 bytes 0, scale 0).  paired: tile rows 0..63
// come from a (features 64 t ..), rows 64..127 from b (the same features), for
// the SwiGLU epilogue.
__global__ void repack_kernel(int qt, const uint8_t* a, const uint8_t* b, int rows, int paired, int tiles,
                              int chunks, uint8_t* out) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)tiles * chunks * (kChunkBlocks * kTileRows)) return;
  const long long item = idx / (kChunkBlocks * kTileRows);
  const int rem = (int)(idx % (kChunkBlocks * kTileRows)), blk = rem / kTileRows, r = rem % kTileRows;
  const int t = (int)(item / chunks), c = (int)(item % chunks);
  const uint8_t* src = a;
  int srow;
  if (paired) {
    srow = t * 64 + (r & 63);
    src = r >= 64 ? b : a;
  } else {
    srow = t * kTileRows + r;
  }
  const bool valid = srow < rows;
  const int bb = gguf_block_bytes(qt);
  const long long nb = (long long)chunks * kChunkBlocks;
  const uint8_t* sp = src + (valid ? ((long long)srow * nb + (long long)c * kChunkBlocks + blk) * bb : 0);
  uint8_t* base = out + item * item_bytes(qt);
  if (qt == kQ4_0) {
    uint8_t* q = base + q4_off(blk, r);
    for (int i = 0; i < 16; ++i) q[i] = valid ? sp[2 + i] : 0x88;
  } else {
    for (int h = 0; h < 2; ++h) {
      uint8_t* q = base + q8_off(blk, h, r);
      for (int i = 0; i < 16; ++i) q[i] = valid ? sp[2 + 16 * h + i] : 0;
    }
  }
  uint8_t* sc = base + scale_off(qt, blk, r);
  sc[0] = valid ? sp[0] : 0;
  sc[1] = valid ? sp[1] : 0;
}

cudaError_t launch_repack(int qt, const uint8_t* a, const uint8_t* b, int rows, int cols, uint8_t* out,
                          cudaStream_t s) {
  const bool paired = b != nullptr;
  const int tiles = packed_tiles(rows, paired), chunks = cols / kChunkCols;
  const long long n = (long long)tiles * chunks * (kChunkBlocks * kTileRows);
  repack_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(qt, a, b, rows, paired ? 1 : 0, tiles, chunks, out);
  return cudaGetLastError();
}

// Dequantise rows of a packed matrix: the GEMV's own operand preparation (the
// 8-bit A bytes q4_unpack / the Q8_0 bytes give the MMA) times the f16 scale,
// one thread per (row, block).
__global__ void dequant_kernel(int qt, const uint8_t* P, int rows, int cols, int paired, int row0, int nrows,
                               float* out) {
  const int nb = cols / 32;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)nrows * nb) return;
  const int r = row0 + (int)(idx / nb), kb = (int)(idx % nb);
  int tile, tr;
  if (paired) {
    const int f = r % rows;
    tile = f / 64;
    tr = (r / rows) * 64 + f % 64;
  } else {
    tile = r / kTileRows;
    tr = r % kTileRows;
  }
  const int chunks = cols / kChunkCols, c = kb / kChunkBlocks, blk = kb % kChunkBlocks;
  const uint8_t* base = P + ((size_t)tile * chunks + c) * item_bytes(qt);
  const uint16_t sbits = *reinterpret_cast<const uint16_t*>(base + scale_off(qt, blk, tr));
  const float d = __half2float(__ushort_as_half(sbits));
  uint32_t av[8];
  if (qt == kQ4_0) {
    q4_unpack(*reinterpret_cast<const uint4*>(base + q4_off(blk, tr)), av);
  } else {
    const uint4 w0 = *reinterpret_cast<const uint4*>(base + q8_off(blk, 0, tr));
    const uint4 w1 = *reinterpret_cast<const uint4*>(base + q8_off(blk, 1, tr));
    av[0] = w0.x; av[1] = w0.y; av[2] = w0.z; av[3] = w0.w;
    av[4] = w1.x; av[5] = w1.y; av[6] = w1.z; av[7] = w1.w;
  }
  float* o = out + (size_t)(r - row0) * cols + kb * 32;
  for (int e = 0; e < 32; ++e) {
    const uint32_t byte = (av[e >> 2] >> (8 * (e & 3))) & 0xFFu;
    const int q = qt == kQ4_0 ? (int)byte - 8 : (int)(int8_t)byte;
    o[e] = __fmul_rn((float)q, d);
  }
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
