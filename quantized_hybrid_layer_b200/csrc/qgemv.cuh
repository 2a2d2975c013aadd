// Fused dequant-GEMV / skinny GEMM over packed Q4_0 / Q8_0 weights.
//
// y[t][r] = sum_c x[t][c] * W[r][c] for n_tok = NT tokens (1..16), the
// projection every layer of the stage streams: "every token reads all of the
// weights once" (SwarmLLM README, paragraph after the peer diagram).  Decode is
// memory-bound, so the kernel is built to keep HBM busy:
//
//  * Persistent stream-K grid, one CTA per SM.  The (tile, chunk) items of the
//    packed matrix are split into contiguous equal ranges, one per CTA, so every
//    SM streams the same number of bytes whatever the matrix shape.
//  * One producer warp per CTA moves items (64 rows x 256 columns, one
//    contiguous record) into a ring of shared-memory stages with bulk async
//    copies (cp.async.bulk + mbarrier, L2 evict-first).  The weights never
//    depend on the previous kernel, so the producer starts before
//    griddepcontrol.wait: under programmatic dependent launch the next
//    projection's weights are in flight while the previous kernel drains.
//  * Eight consumer warps; warp w dequantises block w of each item.  Lane l
//    owns tile rows l and l + 32, so the x values are warp-uniform broadcast
//    loads and no cross-lane reduction is needed.  Nibbles/bytes become floats
//    exactly (mask-or into 2^23, one packed FMA), products are accumulated with
//    packed f32x2 FMAs, and the per-block f16 scale is applied once per block.
//  * Reduction order is fixed and independent of NT: per row, blocks in item
//    order inside a warp, then warps 0..7, then CTAs in grid order (stream-K
//    partials, combined by whichever CTA finishes a tile last).  Each token's
//    sum is computed by exactly the same operations whatever NT is, so a
//    16-token pass is bit-identical to 16 single-token passes.
//  * Fused epilogues: input RMS scale (RMSNorm folded as rstd * sum(z W) with
//    z = h * gamma written by the producer of h), SwiGLU on paired gate/up
//    rows, residual add with the next RMSNorm's z and per-tile sum of squares.
#pragma once

#include "qpack.cuh"

namespace qhl {

enum Epi : int { EPI_STORE = 0, EPI_SWIGLU = 1, EPI_RESID = 2 };

struct GemvArgs {
  const uint8_t* W;        // packed items, tile-major
  int tiles, chunks;       // item grid: tiles x chunks
  const float* x;          // [NT][x_stride] input (z for normed inputs)
  int x_stride;
  float* y;                // STORE / SWIGLU output; RESID: residual stream (in/out)
  int y_stride;
  int out_valid;           // STORE/RESID: valid rows; SWIGLU: valid features
  const float* ss_in;      // optional per-tile sums of squares of the pre-norm input: [NT][ss_stride]
  int ss_tiles, ss_stride;
  float inv_dim, eps;      // rstd = 1 / sqrt(sum(ss) * inv_dim + eps)
  const float* gamma_next; // RESID: next RMSNorm weight (z_out = h_new * gamma_next)
  float* z_out;
  int z_stride;
  float* ss_out;           // RESID: per-tile sum of squares of h_new, [NT][ss_out_stride]
  int ss_out_stride;
  float* partials;         // stream-K scratch: [2 * workers][NT][64]
  int* counters;           // stream-K tile counters, zero between launches
  int workers;             // CTAs that own items (<= items, == grid size)
  unsigned* err;           // device error word
};

constexpr int kConsumerWarps = 8;
constexpr int kGemvThreads = (kConsumerWarps + 1) * 32;
// Stream-K workers per SM: the grid is kCtasPerSm * SMs for every token count
// (the split, and hence the summation order, must not depend on NT).
constexpr int kCtasPerSm = 2;

// A stage holds one item's packed weights followed by the item's x columns for
// every token ([NT][256] f32).  Up to 2 tokens the ring is small enough for two
// CTAs of this kernel plus one of the next (under programmatic dependent
// launch) to share an SM; up to 4 tokens two CTAs fit; beyond that one CTA per
// SM runs at a time.
template <int QT, int NT>
struct GemvCfg {
  static constexpr int kStageBytes = QLayout<QT>::kItemBytes + NT * kChunkCols * 4;
  static constexpr int kBudget = NT <= 2 ? 72 * 1024 : (NT <= 4 ? 104 * 1024 : 196 * 1024);
  static constexpr int kRaw = (kBudget - kConsumerWarps * NT * 64 * 4 - 512) / kStageBytes;
  static constexpr int kStages = kRaw < 3 ? 3 : (kRaw > 12 ? 12 : kRaw);
  static constexpr int kMinBlocks = NT <= 2 ? 3 : (NT <= 4 ? 2 : 1);
};

template <int QT, int NT>
constexpr int gemv_smem_bytes() {
  return GemvCfg<QT, NT>::kStages * GemvCfg<QT, NT>::kStageBytes   // stage ring
         + kConsumerWarps * NT * 64 * 4                           // per-warp tile partials
         + 16 * 4                                                 // rstd
         + 2 * GemvCfg<QT, NT>::kStages * 8                       // full/empty mbarriers
         + 16;                                                    // flags
}

// First item of CTA `w` in a balanced contiguous split of `n` items over `p` CTAs.
__host__ __device__ inline long long sk_begin(long long w, long long n, long long p) { return (w * n) / p; }
// CTA owning item i (the largest w with sk_begin(w) <= i).
__host__ __device__ inline long long sk_owner(long long i, long long n, long long p) {
  return ((i + 1) * p - 1) / n;
}

// The quants and scales one lane reads from a stage: its two rows of block `warp`.
template <int QT> struct ItemRegs;
template <> struct ItemRegs<kQ4_0> { uint32_t a[4], b[4]; uint32_t sc; };
template <> struct ItemRegs<kQ8_0> { uint32_t a[8], b[8]; uint32_t sc; };

template <int QT>
QHL_DEV void load_item(const uint8_t* st, int warp, int lane, ItemRegs<QT>& r) {
  if constexpr (QT == kQ4_0) {
    const uint4 wa = *reinterpret_cast<const uint4*>(st + ((warp * 2 + 0) * 32 + lane) * 16);
    const uint4 wb = *reinterpret_cast<const uint4*>(st + ((warp * 2 + 1) * 32 + lane) * 16);
    r.a[0] = wa.x; r.a[1] = wa.y; r.a[2] = wa.z; r.a[3] = wa.w;
    r.b[0] = wb.x; r.b[1] = wb.y; r.b[2] = wb.z; r.b[3] = wb.w;
  } else {
    const uint8_t* base = st + (warp * 4) * 32 * 16;   // [half][h][lane][16]
    const uint4 wa0 = *reinterpret_cast<const uint4*>(base + ((0 * 2 + 0) * 32 + lane) * 16);
    const uint4 wa1 = *reinterpret_cast<const uint4*>(base + ((1 * 2 + 0) * 32 + lane) * 16);
    const uint4 wb0 = *reinterpret_cast<const uint4*>(base + ((0 * 2 + 1) * 32 + lane) * 16);
    const uint4 wb1 = *reinterpret_cast<const uint4*>(base + ((1 * 2 + 1) * 32 + lane) * 16);
    r.a[0] = wa0.x; r.a[1] = wa0.y; r.a[2] = wa0.z; r.a[3] = wa0.w;
    r.a[4] = wa1.x; r.a[5] = wa1.y; r.a[6] = wa1.z; r.a[7] = wa1.w;
    r.b[0] = wb0.x; r.b[1] = wb0.y; r.b[2] = wb0.z; r.b[3] = wb0.w;
    r.b[4] = wb1.x; r.b[5] = wb1.y; r.b[6] = wb1.z; r.b[7] = wb1.w;
  }
  r.sc = *reinterpret_cast<const uint32_t*>(st + QLayout<QT>::kQuantBytes + (warp * 32 + lane) * 4);
}

// Accumulate one block for both rows and all NT tokens.  Per token and row the
// operation sequence is fixed: packed FMAs over the block's element pairs in
// word order, the two lanes added, then one FMA with the block scale.
template <int QT, int NT>
QHL_DEV void compute_item(const ItemRegs<QT>& r, const float* xcol, float (&r0)[NT], float (&r1)[NT]) {
  constexpr int x_stride = kChunkCols;   // x chunk in shared memory: [NT][256]
  float2 a0[NT], a1[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) { a0[t] = make_float2(0.f, 0.f); a1[t] = make_float2(0.f, 0.f); }
  if constexpr (QT == kQ4_0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 p[4], q[4];
      q4_word(r.a[i], p);
      q4_word(r.b[i], q);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float4* xv = reinterpret_cast<const float4*>(xcol + t * x_stride);
        const float4 xa = xv[i];
        const float4 xb = xv[4 + i];
        const float2 x0 = make_float2(xa.x, xa.y), x1 = make_float2(xa.z, xa.w);
        const float2 x2 = make_float2(xb.x, xb.y), x3 = make_float2(xb.z, xb.w);
        a0[t] = ffma2(p[0], x0, a0[t]);
        a0[t] = ffma2(p[1], x1, a0[t]);
        a0[t] = ffma2(p[2], x2, a0[t]);
        a0[t] = ffma2(p[3], x3, a0[t]);
        a1[t] = ffma2(q[0], x0, a1[t]);
        a1[t] = ffma2(q[1], x1, a1[t]);
        a1[t] = ffma2(q[2], x2, a1[t]);
        a1[t] = ffma2(q[3], x3, a1[t]);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float2 p[2], q[2];
      q8_word(r.a[i], p);
      q8_word(r.b[i], q);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float4 xa = reinterpret_cast<const float4*>(xcol + t * x_stride)[i];
        const float2 x0 = make_float2(xa.x, xa.y), x1 = make_float2(xa.z, xa.w);
        a0[t] = ffma2(p[0], x0, a0[t]);
        a0[t] = ffma2(p[1], x1, a0[t]);
        a1[t] = ffma2(q[0], x0, a1[t]);
        a1[t] = ffma2(q[1], x1, a1[t]);
      }
    }
  }
  const float d0 = __half2float(__ushort_as_half(static_cast<unsigned short>(r.sc & 0xFFFFu)));
  const float d1 = __half2float(__ushort_as_half(static_cast<unsigned short>(r.sc >> 16)));
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    r0[t] = __fmaf_rn(d0, __fadd_rn(a0[t].x, a0[t].y), r0[t]);
    r1[t] = __fmaf_rn(d1, __fadd_rn(a1[t].x, a1[t].y), r1[t]);
  }
}

// Epilogue for one finished tile; vals = [NT][64] final sums in shared memory.
template <int EPI, int NT>
QHL_DEV void gemv_epilogue(const GemvArgs& a, int tile, float* vals, const float* rstd, int tid) {
  if constexpr (EPI == EPI_STORE) {
    for (int idx = tid; idx < NT * 64; idx += 256) {
      const int t = idx >> 6, row = idx & 63, gr = tile * 64 + row;
      if (gr < a.out_valid) a.y[(size_t)t * a.y_stride + gr] = __fmul_rn(vals[idx], rstd[t]);
    }
  } else if constexpr (EPI == EPI_SWIGLU) {
    for (int idx = tid; idx < NT * 32; idx += 256) {
      const int t = idx >> 5, r = idx & 31, f = tile * 32 + r;
      if (f < a.out_valid) {
        const float g = __fmul_rn(vals[t * 64 + r], rstd[t]);
        const float u = __fmul_rn(vals[t * 64 + 32 + r], rstd[t]);
        const float s = __fdiv_rn(g, __fadd_rn(1.f, expf(-g)));   // silu(g) = g * sigmoid(g)
        a.y[(size_t)t * a.y_stride + f] = __fmul_rn(s, u);
      }
    }
  } else {
    for (int idx = tid; idx < NT * 64; idx += 256) {
      const int t = idx >> 6, row = idx & 63, gr = tile * 64 + row;
      float hn = 0.f;
      if (gr < a.out_valid) {
        float* hp = a.y + (size_t)t * a.y_stride + gr;
        hn = __fadd_rn(*hp, vals[idx]);
        *hp = hn;
        if (a.z_out) a.z_out[(size_t)t * a.z_stride + gr] = __fmul_rn(hn, a.gamma_next[gr]);
      }
      vals[idx] = hn;
    }
    if (a.ss_out) {
      named_sync(1, 256);
      if (tid < NT) a.ss_out[(size_t)tid * a.ss_out_stride + tile] = sumsq64(vals + tid * 64);
    }
  }
}

template <int QT, int NT, int EPI>
__global__ void __launch_bounds__(kGemvThreads, GemvCfg<QT, NT>::kMinBlocks) qgemv_kernel(const GemvArgs a) {
  constexpr int S = GemvCfg<QT, NT>::kStages;
  constexpr int IB = QLayout<QT>::kItemBytes;
  constexpr int SB = GemvCfg<QT, NT>::kStageBytes;
  constexpr int XB = kChunkCols * 4;      // bytes of one token's x chunk
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* stages = smem;
  float* red = reinterpret_cast<float*>(smem + S * SB);                 // [8][NT][64]
  float* rstd = red + kConsumerWarps * NT * 64;                          // [16]
  uint64_t* bars = reinterpret_cast<uint64_t*>(rstd + 16);              // full[S], empty[S]
  int* flag = reinterpret_cast<int*>(bars + 2 * S);

  const int cta = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) pdl_launch();
  if (cta >= a.workers) return;
  const long long n_items = (long long)a.tiles * a.chunks;
  const long long i0 = sk_begin(cta, n_items, a.workers);
  const long long i1 = sk_begin(cta + 1, n_items, a.workers);

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&bars[s]), 1);
      mbar_init(smem_u32(&bars[S + s]), kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------- producer: stream this CTA's items into the ring ----------
    // Weights never depend on earlier kernels: the first S items' weights are
    // requested before griddepcontrol.wait.  Their x chunks (written by the
    // previous kernel) follow once the dependency is resolved.
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const int n_local = (int)(i1 - i0);
      const int pre = n_local < S ? n_local : S;
      const int c0 = (int)(i0 % a.chunks);
      auto issue_x = [&](int k, int s) {
        // chunk of local item k: (c0 + k) mod chunks, without 64-bit division
        int c = c0 + k;
        while (c >= a.chunks) c -= a.chunks;
        const uint32_t full = smem_u32(&bars[s]);
        for (int t = 0; t < NT; ++t)
          bulk_g2s_plain(smem_u32(stages + s * SB + IB + t * XB), a.x + (size_t)t * a.x_stride + (size_t)c * kChunkCols,
                         XB, full);
      };
      for (int k = 0; k < pre; ++k) {
        const uint32_t full = smem_u32(&bars[k]);
        mbar_arrive_expect_tx(full, SB);
        bulk_g2s(smem_u32(stages + k * SB), a.W + (i0 + k) * IB, IB, full, pol);
      }
      pdl_wait();
      for (int k = 0; k < pre; ++k) issue_x(k, k);
      for (int k = pre; k < n_local; ++k) {
        const int s = k % S, round = k / S;
        mbar_wait(smem_u32(&bars[S + s]), (round - 1) & 1, a.err);
        const uint32_t full = smem_u32(&bars[s]);
        mbar_arrive_expect_tx(full, SB);
        bulk_g2s(smem_u32(stages + s * SB), a.W + (i0 + k) * IB, IB, full, pol);
        issue_x(k, s);
      }
    }
    return;
  }

  // ---------------- consumers ------------------------------------------------
  pdl_wait();   // x, ss_in, the residual stream and the scratch come from earlier kernels
  if (tid < NT)
    rstd[tid] = a.ss_in ? rstd_from_partials(a.ss_in + (size_t)tid * a.ss_stride, a.ss_tiles, a.inv_dim, a.eps) : 1.f;

  float r0[NT], r1[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) { r0[t] = 0.f; r1[t] = 0.f; }
  bool timed_out = false;
  int tile = (int)(i0 / a.chunks);
  const int first_tile = tile;

  auto flush = [&](int tl) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      red[(warp * NT + t) * 64 + lane] = r0[t];
      red[(warp * NT + t) * 64 + 32 + lane] = r1[t];
      r0[t] = 0.f;
      r1[t] = 0.f;
    }
    named_sync(1, 256);
    for (int idx = tid; idx < NT * 64; idx += 256) {
      float v = red[idx];
#pragma unroll
      for (int w = 1; w < kConsumerWarps; ++w) v = __fadd_rn(v, red[w * NT * 64 + idx]);
      red[idx] = v;
    }
    named_sync(1, 256);
    const long long t_lo = (long long)tl * a.chunks, t_hi = t_lo + a.chunks;
    if (t_lo >= i0 && t_hi <= i1) {
      gemv_epilogue<EPI, NT>(a, tl, red, rstd, tid);
    } else {
      // stream-K: publish this CTA's partial; the last contributor finishes the tile
      float* mine = a.partials + (size_t)(2 * cta + (tl == first_tile ? 0 : 1)) * NT * 64;
      for (int idx = tid; idx < NT * 64; idx += 256) mine[idx] = red[idx];
      __threadfence();
      named_sync(1, 256);
      const long long cf = sk_owner(t_lo, n_items, a.workers);
      const long long cl = sk_owner(t_hi - 1, n_items, a.workers);
      if (tid == 0) {
        const int old = atomicAdd(&a.counters[tl], 1);
        *flag = (old == (int)(cl - cf)) ? 1 : 0;
      }
      named_sync(1, 256);
      if (*flag) {
        __threadfence();
        for (int idx = tid; idx < NT * 64; idx += 256) {
          float v = 0.f;
          for (long long c = cf; c <= cl; ++c) {
            const int ft = (int)(sk_begin(c, n_items, a.workers) / a.chunks);
            const float* pc = a.partials + (size_t)(2 * c + (tl == ft ? 0 : 1)) * NT * 64;
            const float pv = __ldcg(pc + idx);
            v = (c == cf) ? pv : __fadd_rn(v, pv);
          }
          red[idx] = v;
        }
        named_sync(1, 256);
        gemv_epilogue<EPI, NT>(a, tl, red, rstd, tid);
        if (tid == 0) a.counters[tl] = 0;
      }
    }
    named_sync(1, 256);
  };

  named_sync(1, 256);   // rstd visible
  const int n_local = (int)(i1 - i0);
  int chunk = (int)(i0 - (long long)tile * a.chunks);
  int s = 0;
  uint32_t phase = 0;
  for (int k = 0; k < n_local; ++k) {
    if (chunk == a.chunks) {
      flush(tile);
      ++tile;
      chunk = 0;
    }
    if (!mbar_wait(smem_u32(&bars[s]), phase, a.err)) timed_out = true;
    ItemRegs<QT> regs;
    const uint8_t* st = stages + s * SB;
    load_item<QT>(st, warp, lane, regs);
    compute_item<QT, NT>(regs, reinterpret_cast<const float*>(st + IB) + warp * 32, r0, r1);
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars[S + s]));   // stage free for the producer
    ++chunk;
    if (++s == S) {
      s = 0;
      phase ^= 1u;
    }
  }
  if (i1 > i0) flush(tile);
  if (timed_out && lane == 0) {
    // error path: let any copy still in flight land before the CTA exits
    for (int s = 0; s < S; ++s) mbar_wait(smem_u32(&bars[s]), 0, nullptr);
  }
}

}  // namespace qhl
