// Fused dequant-GEMV / skinny GEMM over packed Q4_0 / Q8_0 weights.
//
// y[t][r] = sum_c x[t][c] * W[r][c] for n_tok = NT tokens (1..16), the
// projection every layer of the stage streams: "every token reads all of the
// weights once" (SwarmLLM README, paragraph after the peer diagram).  Decode is
// memory-bound, so the kernel is built to keep HBM busy and the SM's integer
// and FP pipes well below their limits:
//
//  * Persistent stream-K grid, two CTAs per SM.  The (tile, chunk) items of the
//    packed matrix are split into contiguous equal ranges, one per CTA, so every
//    SM streams the same number of bytes whatever the matrix shape.
//  * One producer warp per CTA moves items (64 rows x 256 columns, one
//    contiguous record) and the matching x columns into a ring of shared-memory
//    stages with bulk async copies (cp.async.bulk + mbarrier, L2 evict-first for
//    weights).  The weights never depend on the previous kernel, so the first
//    stages are requested before griddepcontrol.wait: under programmatic
//    dependent launch a projection's weights stream in while the previous
//    kernel drains.
//  * Eight consumer warps; warp w handles block w of each item.  Lane l owns
//    tile rows l and l + 32, so x is read as warp-uniform broadcasts and no
//    cross-lane reduction is needed.  x arrives in block fixed-point form
//    (qact.cuh): each block's sum_j q_j X_j is formed exactly in int32 with
//    byte dot products (dp4a) against the 4-bit (or 8-bit) quants, and one FMA
//    per block adds d * s * sum to the row's f32 accumulator.
//  * Reduction order is fixed and independent of NT: per row, exact integer
//    block sums, blocks in item order inside a warp, then warps 0..7, then CTAs
//    in grid order (stream-K partials, combined by whichever CTA finishes a tile
//    last).  Each token's result is produced by the same operations whatever NT
//    is, so a 16-token pass is bit-identical to 16 single-token passes.
//  * Fused epilogues: input RMS scale (RMSNorm folded as rstd * sum(z W) with
//    z = h * gamma written by the producer of h), SwiGLU on paired gate/up rows
//    writing the down projection's input in block fixed-point form, and the
//    residual add writing h, the next RMSNorm's z (block fixed point) and its
//    per-tile sums of squares.
#pragma once

#include "qact.cuh"
#include "qpack.cuh"

namespace qhl {

enum Epi : int { EPI_STORE = 0, EPI_SWIGLU = 1, EPI_RESID = 2 };

struct GemvArgs {
  const uint8_t* W;        // packed items, tile-major
  int tiles, chunks;       // item grid: tiles x chunks
  const uint8_t* qx;       // input in block fixed point: [NT][qx_stride bytes]
  int qx_stride;
  float* y;                // STORE: f32 output [NT][y_stride]; RESID: residual stream h (in/out)
  int y_stride;
  int out_valid;           // STORE/RESID: valid rows; SWIGLU: valid features
  uint8_t* qout;           // SWIGLU: silu(g)*u; RESID: h_new * gamma_next (block fixed point), or null
  int qout_stride;
  const float* ss_in;      // optional per-tile sums of squares of the pre-norm input: [NT][ss_stride]
  int ss_tiles, ss_stride;
  float inv_dim, eps;      // rstd = 1 / sqrt(sum(ss) * inv_dim + eps)
  const float* gamma_next; // RESID: next RMSNorm weight
  float* ss_out;           // RESID: per-tile sum of squares of h_new, [NT][ss_out_stride], or null
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

// A stage holds one item's packed weights followed by the item's x chunk for
// every token ([NT][864] bytes).  Up to 2 tokens the ring is small enough for
// two CTAs of this kernel plus one of the next (under programmatic dependent
// launch) to share an SM; up to 4 tokens two CTAs fit; beyond that one CTA per
// SM runs at a time.
template <int QT, int NT>
struct GemvCfg {
  static constexpr int kStageBytes = QLayout<QT>::kItemBytes + NT * kQChunkBytes;
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

// x words of one block: 8 words per byte plane (word k = elements 4k..4k+3).
struct XBlock { uint32_t hi[8], mid[8], lo[8]; float s; int s_hi, s_ml; };

QHL_DEV void load_xblock(const uint8_t* xt, int warp, XBlock& x) {
  const uint4* ph = reinterpret_cast<const uint4*>(xt + warp * 32);
  const uint4* pm = reinterpret_cast<const uint4*>(xt + 256 + warp * 32);
  const uint4* pl = reinterpret_cast<const uint4*>(xt + 512 + warp * 32);
  const uint4 h0 = ph[0], h1 = ph[1], m0 = pm[0], m1 = pm[1], l0 = pl[0], l1 = pl[1];
  x.hi[0] = h0.x; x.hi[1] = h0.y; x.hi[2] = h0.z; x.hi[3] = h0.w;
  x.hi[4] = h1.x; x.hi[5] = h1.y; x.hi[6] = h1.z; x.hi[7] = h1.w;
  x.mid[0] = m0.x; x.mid[1] = m0.y; x.mid[2] = m0.z; x.mid[3] = m0.w;
  x.mid[4] = m1.x; x.mid[5] = m1.y; x.mid[6] = m1.z; x.mid[7] = m1.w;
  x.lo[0] = l0.x; x.lo[1] = l0.y; x.lo[2] = l0.z; x.lo[3] = l0.w;
  x.lo[4] = l1.x; x.lo[5] = l1.y; x.lo[6] = l1.z; x.lo[7] = l1.w;
  x.s = reinterpret_cast<const float*>(xt + 768)[warp];
  x.s_hi = reinterpret_cast<const int*>(xt + 800)[warp];
  x.s_ml = reinterpret_cast<const int*>(xt + 832)[warp];
}

// acc = fma(d * s, 65536 * H + ML, acc): the block's exact integer partial sums
// turned into one f32 update by a fixed sequence of operations.
QHL_DEV float block_update(float d, float s, int H, int ML, float acc) {
  const float v = __fmaf_rn(__int2float_rn(H), 65536.f, __int2float_rn(ML));
  return __fmaf_rn(__fmul_rn(d, s), v, acc);
}

// One block for both rows and all NT tokens.
template <int QT, int NT>
QHL_DEV void compute_item(const ItemRegs<QT>& r, const uint8_t* xs, int warp, float (&r0)[NT], float (&r1)[NT]) {
  const float d0 = __half2float(__ushort_as_half(static_cast<unsigned short>(r.sc & 0xFFFFu)));
  const float d1 = __half2float(__ushort_as_half(static_cast<unsigned short>(r.sc >> 16)));
  if constexpr (QT == kQ4_0) {
    // low nibbles of word i are elements 4i..4i+3, high nibbles 16+4i..16+4i+3
    uint32_t qa[8], qb[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      qa[i] = r.a[i] & 0x0F0F0F0Fu;
      qa[4 + i] = (r.a[i] >> 4) & 0x0F0F0F0Fu;
      qb[i] = r.b[i] & 0x0F0F0F0Fu;
      qb[4 + i] = (r.b[i] >> 4) & 0x0F0F0F0Fu;
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      XBlock x;
      load_xblock(xs + t * kQChunkBytes, warp, x);
      int H0 = 0, M0 = 0, L0 = 0, H1 = 0, M1 = 0, L1 = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {        // q in 0..15: signed x signed is exact for hi
        H0 = dp4a_ss(qa[k], x.hi[k], H0);
        M0 = dp4a_uu(qa[k], x.mid[k], M0);
        L0 = dp4a_uu(qa[k], x.lo[k], L0);
        H1 = dp4a_ss(qb[k], x.hi[k], H1);
        M1 = dp4a_uu(qb[k], x.mid[k], M1);
        L1 = dp4a_uu(qb[k], x.lo[k], L1);
      }
      // sum_j (q_j - 8) X_j = 65536 (H - 8 sum hi) + (256 M + L - 8 sum ml)
      r0[t] = block_update(d0, x.s, H0 - 8 * x.s_hi, M0 * 256 + L0 - 8 * x.s_ml, r0[t]);
      r1[t] = block_update(d1, x.s, H1 - 8 * x.s_hi, M1 * 256 + L1 - 8 * x.s_ml, r1[t]);
    }
  } else {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      XBlock x;
      load_xblock(xs + t * kQChunkBytes, warp, x);
      int H0 = 0, M0 = 0, L0 = 0, H1 = 0, M1 = 0, L1 = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {        // word k holds signed quants 4k..4k+3
        H0 = dp4a_ss(r.a[k], x.hi[k], H0);
        M0 = dp4a_su(r.a[k], x.mid[k], M0);
        L0 = dp4a_su(r.a[k], x.lo[k], L0);
        H1 = dp4a_ss(r.b[k], x.hi[k], H1);
        M1 = dp4a_su(r.b[k], x.mid[k], M1);
        L1 = dp4a_su(r.b[k], x.lo[k], L1);
      }
      r0[t] = block_update(d0, x.s, H0, M0 * 256 + L0, r0[t]);
      r1[t] = block_update(d1, x.s, H1, M1 * 256 + L1, r1[t]);
    }
  }
}

// Epilogue for one finished tile; vals = [NT][64] final sums in shared memory.
// Called by all 256 consumer threads.
template <int EPI, int NT>
QHL_DEV void gemv_epilogue(const GemvArgs& a, int tile, float* vals, const float* rstd, int tid) {
  const int warp = tid >> 5, lane = tid & 31;
  if constexpr (EPI == EPI_STORE) {
    for (int idx = tid; idx < NT * 64; idx += 256) {
      const int t = idx >> 6, row = idx & 63, gr = tile * 64 + row;
      if (gr < a.out_valid) a.y[(size_t)t * a.y_stride + gr] = __fmul_rn(vals[idx], rstd[t]);
    }
  } else if constexpr (EPI == EPI_SWIGLU) {
    // tile rows 0..31 are gate rows of features tile*32.., rows 32..63 the matching up rows
    for (int t = warp; t < NT; t += kConsumerWarps) {
      const int f = tile * 32 + lane;
      float u = 0.f;
      if (f < a.out_valid) {
        const float g = __fmul_rn(vals[t * 64 + lane], rstd[t]);
        const float up = __fmul_rn(vals[t * 64 + 32 + lane], rstd[t]);
        u = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.f, expf(-g))), up);   // silu(g) * up
      }
      qact_store_block(u, a.qout + (size_t)t * a.qout_stride, tile, lane);
    }
  } else {
    for (int idx = tid; idx < NT * 64; idx += 256) {
      const int t = idx >> 6, row = idx & 63, gr = tile * 64 + row;
      float hn = 0.f;
      if (gr < a.out_valid) {
        float* hp = a.y + (size_t)t * a.y_stride + gr;
        hn = __fadd_rn(__ldcg(hp), vals[idx]);   // through L2: h may come from another CTA of the same kernel
        *hp = hn;
      }
      vals[idx] = hn;
    }
    named_sync(1, 256);
    if (a.qout) {
      for (int p = warp; p < NT * 2; p += kConsumerWarps) {
        const int t = p >> 1, b = p & 1, gr = tile * 64 + b * 32 + lane;
        const float z = gr < a.out_valid ? __fmul_rn(vals[t * 64 + b * 32 + lane], a.gamma_next[gr]) : 0.f;
        qact_store_block(z, a.qout + (size_t)t * a.qout_stride, tile * 2 + b, lane);
      }
    }
    if (a.ss_out && tid < NT) a.ss_out[(size_t)tid * a.ss_out_stride + tile] = sumsq64(vals + tid * 64);
  }
}

// Consumer side of one GEMV for CTA `cta` (the 256 threads of warps 0..7):
// takes this CTA's stream-K items, in order, from the shared-memory ring
// (`slot` / `phase` carry the ring position across calls), accumulates,
// and finishes every tile it touches (directly or through the stream-K
// partials).  `red` = [8][NT][64] f32, `rstd` = [16] f32, `flag` = one int.
template <int QT, int NT, int EPI, int S>
QHL_DEV void gemv_consume(const GemvArgs& a, int cta, uint8_t* stages, uint64_t* bars, float* red, float* rstd,
                          int* flag, int& slot, uint32_t& phase, bool& timed_out) {
  constexpr int IB = QLayout<QT>::kItemBytes;
  constexpr int SB = IB + NT * kQChunkBytes;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long n_items = (long long)a.tiles * a.chunks;
  const long long i0 = sk_begin(cta, n_items, a.workers);
  const long long i1 = sk_begin(cta + 1, n_items, a.workers);
  const int n_local = cta < a.workers ? (int)(i1 - i0) : 0;

  if (n_local == 0) return;
  // the input's RMS scale, one warp per token; only the epilogue reads it,
  // after the first flush's barriers
  for (int t = warp; t < NT; t += kConsumerWarps) {
    const float r = a.ss_in ? rstd_warp(a.ss_in + (size_t)t * a.ss_stride, a.ss_tiles, a.inv_dim, a.eps, lane) : 1.f;
    if (lane == 0) rstd[t] = r;
  }

  float r0[NT], r1[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) { r0[t] = 0.f; r1[t] = 0.f; }
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
      // (release: the barrier orders every thread's stores before thread 0's
      // fence and counter increment; acquire: the last arriver's fence after
      // its increment, then the barrier, orders the partial loads after it)
      float* mine = a.partials + (size_t)(2 * cta + (tl == first_tile ? 0 : 1)) * NT * 64;
      for (int idx = tid; idx < NT * 64; idx += 256) mine[idx] = red[idx];
      named_sync(1, 256);
      const long long cf = sk_owner(t_lo, n_items, a.workers);
      const long long cl = sk_owner(t_hi - 1, n_items, a.workers);
      if (tid == 0) {
        __threadfence();
        const int old = atomicAdd(&a.counters[tl], 1);
        const int last = (old == (int)(cl - cf)) ? 1 : 0;
        if (last) __threadfence();
        *flag = last;
      }
      named_sync(1, 256);
      if (*flag) {
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

  int chunk = (int)(i0 - (long long)tile * a.chunks);
  for (int k = 0; k < n_local; ++k) {
    if (chunk == a.chunks) {
      flush(tile);
      ++tile;
      chunk = 0;
    }
    // after one timed-out wait the rest of the call runs without waiting (the
    // error is recorded; results are garbage, but the kernel ends promptly)
    if (!timed_out && !mbar_wait(smem_u32(&bars[slot]), phase, a.err)) timed_out = true;
    ItemRegs<QT> regs;
    const uint8_t* st = stages + slot * SB;
    load_item<QT>(st, warp, lane, regs);
    compute_item<QT, NT>(regs, st + IB, warp, r0, r1);
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars[S + slot]));   // stage free for the producer
    ++chunk;
    if (++slot == S) {
      slot = 0;
      phase ^= 1u;
    }
  }
  flush(tile);
}

template <int QT, int NT, int EPI>
__global__ void __launch_bounds__(kGemvThreads, GemvCfg<QT, NT>::kMinBlocks) qgemv_kernel(const GemvArgs a) {
  constexpr int S = GemvCfg<QT, NT>::kStages;
  constexpr int IB = QLayout<QT>::kItemBytes;
  constexpr int SB = GemvCfg<QT, NT>::kStageBytes;
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
  const int n_local = (int)(i1 - i0);

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
      const int pre = n_local < S ? n_local : S;
      const int c0 = (int)(i0 % a.chunks);
      auto issue_x = [&](int k, int s) {
        int c = c0 + k;                    // chunk of local item k, without 64-bit division
        while (c >= a.chunks) c -= a.chunks;
        const uint32_t full = smem_u32(&bars[s]);
        for (int t = 0; t < NT; ++t)
          bulk_g2s_plain(smem_u32(stages + s * SB + IB + t * kQChunkBytes),
                         a.qx + (size_t)t * a.qx_stride + (size_t)c * kQChunkBytes, kQChunkBytes, full);
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
  pdl_wait();   // ss_in, the residual stream and the scratch come from earlier kernels
  int slot = 0;
  uint32_t phase = 0;
  bool timed_out = false;
  gemv_consume<QT, NT, EPI, S>(a, cta, stages, bars, red, rstd, flag, slot, phase, timed_out);
  if (timed_out && tid == 0) drain_inflight_copies();   // error path
}

}  // namespace qhl
