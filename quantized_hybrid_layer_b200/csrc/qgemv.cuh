// Fused dequant-GEMV / skinny GEMM over packed Q4_0 / Q8_0 weights on the
// fifth-generation tensor cores.
//
// y[t][r] = sum_c x[t][c] * W[r][c] for n_tok = NT tokens (1..16), the
// projection every layer of the stage streams: one decoded token streams the
// whole weight set a single time (SwarmLLM README, paragraph after the peer
// diagram).  Decode is memory-bound, so the kernel is built to keep HBM busy
// with as little SM work per weight byte as possible:
//
//  * Persistent stream-K grid of one CTA per SM.  The (tile, chunk) items of
//    the packed matrix (128 rows x 256 columns, qpack.cuh) are split into
//    contiguous equal ranges, one per CTA.  A CTA needs under half an SM's
//    shared and tensor memory at one or two tokens, so the next projection's
//    CTA (a programmatic dependent launch) is resident beside it and streams
//    its own weights while this one drains.
//  * Warp roles.  Warp 0 (one thread) streams items into two shared-memory
//    rings with bulk async copies: the quants into the weight ring, the block
//    scales and the item's x columns (qact.cuh) into the x ring.  Warps 2..5
//    ("unpack", thread = row) turn a row's quants into the MMA's 8-bit A
//    operand and store it in tensor memory.  Warp 1 (one thread) issues, per
//    block of 32 columns, one tcgen05.mma kind::i8 of M = 128 rows,
//    N = 8 rows per token (the hi / mid / lo digit planes of x and five
//    unused rows), K = 32: exact int32 sums H, M, L per (row, token) in
//    tensor memory.  Warps 6..9 ("update", thread = row) read them back and
//    add d * s * (65536 H + 256 M + L) to the row's f32 accumulator, then
//    finish tiles (stream-K fix-up and the fused epilogue).
//  * Reduction order is fixed and independent of NT: per row, exact integer
//    block sums, one f32 update per block in item order, then CTAs in grid
//    order (stream-K partials, combined by whichever CTA finishes a tile
//    last).  Each token's result is produced by the same operations whatever
//    NT is, so a 16-token pass is bit-identical to 16 single-token passes.
//  * Fused epilogues: input RMS scale (RMSNorm folded as rstd * sum(z W) with
//    z = h * gamma written by the producer of h), SwiGLU on paired gate/up rows
//    writing the down projection's input in block fixed-point form, and the
//    residual add writing h, the next RMSNorm's z (block fixed point) and its
//    per-tile sums of squares.
//  * Every wait is bounded (common.cuh); after a timeout each role stops, the
//    MMA thread waits for its issued MMAs, and the CTA frees its tensor memory.
#pragma once

#include "qact.cuh"
#include "qpack.cuh"
#include "tc5.cuh"

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
  float* partials;         // stream-K scratch: [2 * workers][NT][128]
  int* counters;           // stream-K tile counters, zero between launches
  int workers;             // CTAs that own items (<= items, == grid size)
  unsigned* err;           // device error word
  // The pass's next projection (null if none): this kernel's producer warms L2
  // with the first items the next kernel's CTA of the same index will stream.
  const uint8_t* next_W;
  int next_items, next_workers;
  // Failure injection for tests of the bounded waits (0 / -1 in normal use):
  // iteration cap of every wait (0 = kWaitLimit), and a local item index whose
  // quants CTA 0's producer never requests, so that its unpack warps' wait on
  // them runs out.
  uint32_t wait_limit;
  int fault_item;
};

// Balanced contiguous split of n items (n < 2^31) over p CTAs: CTA w owns
// items [begin(w), begin(w + 1)) with begin(w) = floor(w n / p), evaluated in
// 32-bit arithmetic as w q + floor(w r / p) (q = n / p, r = n % p).
struct StreamK {
  int n, p, q, r;
  __host__ __device__ StreamK(int n_, int p_) : n(n_), p(p_), q(n_ / p_), r(n_ % p_) {}
  __host__ __device__ int begin(int w) const { return w * q + (w * r) / p; }
  // The CTA owning item i: the largest w with begin(w) <= i (a float estimate,
  // then exact integer steps).
  __host__ __device__ int owner(int i) const {
    int w = (int)(((float)i + 0.5f) * (float)p / (float)n);
    w = w < 0 ? 0 : (w >= p ? p - 1 : w);
    while (w + 1 < p && begin(w + 1) <= i) ++w;
    while (w > 0 && begin(w) > i) --w;
    return w;
  }
};

// Warp roles: weight producer, MMA issuer, C::kUnpackWarps unpack warps
// (eight, two per tensor-memory lane quarter and half an item each, where
// registers allow it; else four), the four update warps, the x producer and
// the second MMA issuer.
constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kUnpackWarp0 = 2;
// Named barriers: 1 = the (first) four update warps, 2 = every warp that
// touches tensor memory, 3 = the second four update warps, 4 = all eight.
constexpr int kBarUpdate = 1;
constexpr int kBarTmem = 2;
constexpr int kBarUpdate2 = 3;
constexpr int kBarUpdateAll = 4;
constexpr int kBarSetup = 7;
constexpr int kBarInit = 8;

// Geometry and shared-memory layout of one GEMV configuration: weight type,
// token count, shared-memory budget, x-ring depth SX, tensor-memory A and D
// buffers NA and ND, the deepest weight ring to use, and `EXTRA` bytes of
// shared memory left for the caller after the GEMV's own regions.
template <int QT_, int NT_, int BUDGET, int SX_, int NA_, int ND_, int SWMAX, int EXTRA>
struct GemvGeom {
  static constexpr int kQT = QT_, kNT = NT_;
  static constexpr int kN = NT_ == 1 ? 8 : 16 * ((NT_ + 1) / 2);   // MMA N: 8 rows per token, padded
  static constexpr int kNTP = kN / 8;                               // token regions in an x slot
  static constexpr int kGB = (64 / kN) >= 8 ? 8 : ((64 / kN) >= 1 ? 64 / kN : 1);   // blocks per D group
  static constexpr int kNG = 8 / kGB;                               // D groups per item
  static constexpr int kDCols = kGB * kN;                           // tensor-memory columns of a D buffer
  static constexpr int kACols = 64;                                 // 8 blocks x 32 bytes / 4
  static constexpr int kNA = NA_, kND = ND_;
  // One D group per item and as many A as D buffers: a single commit per item
  // (on dfull) also tells the unpack warps that the item's A buffer is free.
  static constexpr bool kOneCommit = kNG == 1 && NA_ == ND_;
  static constexpr int kDOff = kNA * kACols;
  static constexpr int kTmemNeed = kDOff + kND * kDCols;
  static constexpr int kTmemCols = kTmemNeed <= 256 ? 256 : 512;
  static constexpr int kQB = QLayout<QT_>::kQuantBytes;
  static constexpr int kXS = QLayout<QT_>::kScaleBytes + kNTP * kQChunkBytes;   // x slot: scales, then tokens
  static constexpr int kSX = SX_;
  static constexpr int kEpi = NT_ * kTileRows * 4;                  // epilogue exchange [NT][128] f32
  static constexpr int kNumBars = 2 * 16 + 3 * SX_ + 2 * NA_ + 2 * ND_ + 1;   // upper bound (SW <= 16)
  static constexpr int kFixed = kEpi + 16 * 4 + 16 + kNumBars * 8 + EXTRA;
  static constexpr int kSW0 = (BUDGET - kFixed - SX_ * kXS) / kQB;
  static constexpr int kSW = kSW0 > SWMAX ? SWMAX : kSW0;
  // shared-memory layout (the rings first; every slot 16-byte aligned)
  static constexpr int kXOff = kSW * kQB;
  static constexpr int kEpiOff = kXOff + kSX * kXS;
  static constexpr int kExtraOff = kEpiOff + kEpi;
  static constexpr int kRstdOff = kExtraOff + (EXTRA + 15) / 16 * 16;
  static constexpr int kSlotOff = kRstdOff + 16 * 4;
  static constexpr int kBarOff = kSlotOff + 16;
  // barriers: wfull[SW], wempty[SW], xfull[SX], sfull[SX], xempty[SX], afull[NA], afree[NA], dfull[ND],
  // dfree[ND], drain
  static constexpr int kSmem = kBarOff + (2 * kSW + 3 * kSX + 2 * kNA + 2 * kND + 1) * 8;
  static_assert(kSW >= 2 && kSW <= 16, "weight ring depth");
  static_assert(kTmemNeed <= 512, "tensor memory");
  static_assert(kSmem <= BUDGET, "shared-memory budget");
};

// The stand-alone projection kernel's configuration: one CTA per SM with a
// deep weight ring (the bytes in flight per SM decide the streaming rate) and
// four A and four D buffers in tensor memory, so the unpack warps, the MMA
// thread and the update warps each run up to four items apart instead of
// waiting on one another's latencies.
// x-ring depth: up to 140 KB of x slots, leaving at least three weight slots
// (two of Q8_0's 32 KB beyond eight tokens), an even count from 2 to 16 (a
// slot holds the block scales and 2 KB per 8-row MMA group).  With many
// tokens an item's x columns outweigh its quants, and they are requested only
// when the update warps release a slot, so the ring must cover their latency.
constexpr int gemv_sx(int qt, int nt) {
  const int xs = 2048 + (nt == 1 ? 1 : 2 * ((nt + 1) / 2)) * 2048;
  const int keep = qt == kQ4_0 ? 3 * 16384 : (nt > 8 ? 2 : 3) * 32768;
  const int room = 213 * 1024 - keep;
  const int sx = ((room < 140 * 1024 ? room : 140 * 1024) / xs) & ~1;
  return sx < 2 ? 2 : (sx > 16 ? 16 : sx);
}
// Tensor-memory buffers: four A and four D buffers up to eight tokens; beyond,
// where one D group is 128 columns, two A and three D buffers.
// Weight ring: four items for one token, twelve beyond.  When every CTA of a
// launch starts at once, a shallow ring lands each CTA's first item sooner
// (fewer requests queue ahead of it); four items on 148 SMs still hold about
// 10 MB in flight, enough to keep HBM busy.  With more tokens the ring depth
// makes no measurable difference.
template <int QT, int NT>
struct GemvCfg : GemvGeom<QT, NT, 225 * 1024, gemv_sx(QT, NT), NT <= 8 ? 4 : 2, NT <= 8 ? 4 : 3,
                          NT == 1 ? 4 : 12, 0> {
  static constexpr int kMinBlocks = 1;
  // Sixteen warps, 128 registers a thread (four warps per SM sub-partition).
  // Up to eight tokens: eight unpack warps (half an item each) and four update
  // warps; beyond, where the f32 updates dominate, four unpack warps and two
  // sets of four update warps, each set owning half of the tokens.
  static constexpr int kUnpackWarps = NT <= 8 ? 8 : 4;
  static constexpr int kUpdateWarps = NT <= 8 ? 4 : 8;
  static constexpr int kNTA = kUpdateWarps == 8 ? (NT + 1) / 2 : NT;   // tokens of the first set
  static constexpr int kUpdateWarp0 = kUnpackWarp0 + kUnpackWarps;
  static constexpr int kXWarp = kUpdateWarp0 + kUpdateWarps;
  static constexpr int kMma2Warp = kXWarp + 1;
  // Two MMA threads where an item is one or two D groups (their barrier
  // checks and bookkeeping then cost as much as the MMAs); beyond, one thread
  // that keeps every D buffer in play (the second MMA warp idles).
  static constexpr int kMmaThreads = NT <= 2 ? 2 : 1;
  static constexpr int kThreads = (kMma2Warp + 1) * 32;
  // each MMA thread waits on its own half of the A, D and x slots (item K
  // uses A slot K % NA and x slot K % SX, both even counts)
  static_assert(kMmaThreads == 1 || (GemvCfg::kNA % 2 == 0 && GemvCfg::kND % 2 == 0 && GemvCfg::kSX % 2 == 0),
                "slots per MMA thread");
};

template <int QT, int NT>
constexpr int gemv_smem_bytes() {
  return GemvCfg<QT, NT>::kSmem;
}

// Non-blocking test of an mbarrier phase.
QHL_DEV bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of two / three mbarrier phases at once: the tests go out
// back to back, so a check of barriers that have already completed (the
// common case in a full pipeline) costs one shared-memory round trip, not one
// per barrier.  A parity of ((K / depth) - 1) & 1 with K < depth names the
// phase before a fresh barrier's first, which counts as complete.
QHL_DEV bool mbar_test2(uint32_t b0, uint32_t p0, uint32_t b1, uint32_t p1) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred q0, q1;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q0, [%1], %2;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q1, [%3], %4;\n\t"
      "and.pred q0, q0, q1;\n\t"
      "selp.u32 %0, 1, 0, q0;\n\t}"
      : "=r"(ok)
      : "r"(b0), "r"(p0), "r"(b1), "r"(p1)
      : "memory");
  return ok != 0;
}
// The two phases' states as bits 0 and 1, in one round trip.
QHL_DEV uint32_t mbar_test2m(uint32_t b0, uint32_t p0, uint32_t b1, uint32_t p1) {
  uint32_t m;
  asm volatile(
      "{\n\t.reg .pred q0, q1;\n\t.reg .b32 r0, r1;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q0, [%1], %2;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q1, [%3], %4;\n\t"
      "selp.u32 r0, 1, 0, q0;\n\t"
      "selp.u32 r1, 2, 0, q1;\n\t"
      "or.b32 %0, r0, r1;\n\t}"
      : "=r"(m)
      : "r"(b0), "r"(p0), "r"(b1), "r"(p1)
      : "memory");
  return m;
}
QHL_DEV bool mbar_test3(uint32_t b0, uint32_t p0, uint32_t b1, uint32_t p1, uint32_t b2, uint32_t p2) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred q0, q1, q2;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q0, [%1], %2;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q1, [%3], %4;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q2, [%5], %6;\n\t"
      "and.pred q0, q0, q1;\n\t"
      "and.pred q0, q0, q2;\n\t"
      "selp.u32 %0, 1, 0, q0;\n\t}"
      : "=r"(ok)
      : "r"(b0), "r"(p0), "r"(b1), "r"(p1), "r"(b2), "r"(p2)
      : "memory");
  return ok != 0;
}

// Stream-K tile counter: add 1 with release (this CTA's partial, published by
// every update thread before the named barrier, becomes visible with it) and
// acquire (the last contributor then sees every other partial).
QHL_DEV int counter_add_acq_rel(int* p) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
  return old;
}

// f32 update of one (row, block, token): acc + d * s * sum_j q_j X_j, with the
// exact integer sums H, M, L of the three digit planes.
template <int QT>
QHL_DEV float block_update(float acc, float d, float s, int H, int M, int L, int Sh, int Sml) {
  int Hx = H, MLx = M * 256 + L;
  if constexpr (QT == kQ4_0) {   // weights are nibble - 8
    Hx -= 8 * Sh;
    MLx -= 8 * Sml;
  }
  const float v = __fmaf_rn(__int2float_rn(Hx), 65536.f, __int2float_rn(MLx));
  return __fmaf_rn(__fmul_rn(d, s), v, acc);
}

// The same update for two tokens at once on packed f32 pairs: each lane is
// rounded exactly as block_update rounds it, so the results are the same bits.
template <int QT>
QHL_DEV float2 block_update2(float2 acc, float d, float2 s, int H0, int M0, int L0, int H1, int M1, int L1, int2 Sh,
                             int2 Sml) {
  int Hx0 = H0, MLx0 = M0 * 256 + L0, Hx1 = H1, MLx1 = M1 * 256 + L1;
  if constexpr (QT == kQ4_0) {   // weights are nibble - 8
    Hx0 -= 8 * Sh.x;
    MLx0 -= 8 * Sml.x;
    Hx1 -= 8 * Sh.y;
    MLx1 -= 8 * Sml.y;
  }
  const float2 v = __ffma2_rn(make_float2(__int2float_rn(Hx0), __int2float_rn(Hx1)), make_float2(65536.f, 65536.f),
                              make_float2(__int2float_rn(MLx0), __int2float_rn(MLx1)));
  return __ffma2_rn(__fmul2_rn(make_float2(d, d), s), v, acc);
}

// Sum of squares of a 128-row tile held one row per thread by four warps
// (quarter q = rows 32q .. 32q + 31): xor-butterfly per warp, then the four
// warps in order.  The one definition used for the per-tile RMSNorm partials
// everywhere, so a stage's result never depends on which kernel produced its
// input.  `red` = shared [4] per token; `bar_id` names a barrier over the four
// warps (128 threads).  Returns the sum in every thread.
QHL_DEV float tile_sumsq(float v, float* red, int quarter, int lane, int bar_id) {
  const float w = warp_sum(__fmul_rn(v, v));
  if (lane == 0) red[quarter] = w;
  named_sync(bar_id, 128);
  const float s = __fadd_rn(__fadd_rn(__fadd_rn(red[0], red[1]), red[2]), red[3]);
  named_sync(bar_id, 128);
  return s;
}

// The tokens one set of four update warps owns: [T0, T0 + NTL) of the
// pass's tokens, with its own named barrier `barq` (128 threads) and the
// barrier `barall` over every update warp (`nall` threads; the same barrier
// when one set owns every token).
struct UpdSlice {
  int barq, barall, nall;
};

// Epilogue of one finished tile by a set of four update warps, thread = tile
// row r (quarter q = r / 32); v[t] = the tile's final sums for row r and
// token T0 + t.
template <int EPI, int T0, int NTL>
QHL_DEV void gemv_epilogue(const GemvArgs& a, int tile, const float (&v)[NTL], const float* rstd, float* ex,
                           int quarter, int lane, const UpdSlice& us, const float (&yres)[NTL]) {
  const int r = quarter * 32 + lane;
  if constexpr (EPI == EPI_STORE) {
    const int gr = tile * kTileRows + r;
    if (gr < a.out_valid)
#pragma unroll
      for (int t = 0; t < NTL; ++t) a.y[(size_t)(T0 + t) * a.y_stride + gr] = __fmul_rn(v[t], rstd[T0 + t]);
  } else if constexpr (EPI == EPI_SWIGLU) {
    // rows 0..63: gate rows of features 64 tile + r; rows 64..127 the matching up rows
    if (r >= 64)
#pragma unroll
      for (int t = 0; t < NTL; ++t) ex[(T0 + t) * kTileRows + r - 64] = __fmul_rn(v[t], rstd[T0 + t]);
    named_sync(us.barq, 128);
    if (r < 64) {
      const int f = tile * 64 + r;
#pragma unroll
      for (int t = 0; t < NTL; ++t) {
        float u = 0.f;
        if (f < a.out_valid) {
          const float g = __fmul_rn(v[t], rstd[T0 + t]);
          const float up = ex[(T0 + t) * kTileRows + r];
          u = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.f, expf(-g))), up);   // silu(g) * up
        }
        qact_store_block(u, a.qout + (size_t)(T0 + t) * a.qout_stride, tile * 2 + quarter, lane);
      }
    }
    named_sync(us.barq, 128);
  } else {
    const int gr = tile * kTileRows + r;
    const bool valid = gr < a.out_valid;
    const float gam = a.qout && valid ? __ldg(a.gamma_next + gr) : 0.f;
#pragma unroll
    for (int t = 0; t < NTL; ++t) {
      const int tg = T0 + t;
      float hn = 0.f;
      if (valid) {
        hn = __fadd_rn(yres[t], v[t]);
        a.y[(size_t)tg * a.y_stride + gr] = hn;
      }
      if (a.qout) qact_store_block(__fmul_rn(hn, gam), a.qout + (size_t)tg * a.qout_stride, tile * 4 + quarter, lane);
      if (a.ss_out) {
        const float s = tile_sumsq(hn, ex + 4 * tg, quarter, lane, us.barq);
        if (r == 0) a.ss_out[(size_t)tg * a.ss_out_stride + tile] = s;
      }
    }
  }
}

// bar.red.or over the `nthreads` threads of named barrier `id`.
QHL_DEV bool bar_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// The residual stream of tile `tile`'s rows for tokens [T0, T0 + NTL), read
// when the CTA starts on the tile so that the epilogue does not wait for it
// (residual epilogue only; the rows are written only by the tile's epilogue).
template <int EPI, int T0, int NTL>
QHL_DEV void load_residual(const GemvArgs& a, int tile, int r, float (&yres)[NTL]) {
#pragma unroll
  for (int t = 0; t < NTL; ++t) yres[t] = 0.f;
  if constexpr (EPI == EPI_RESID) {
    const int gr = tile * kTileRows + r;
    if (gr < a.out_valid)
#pragma unroll
      for (int t = 0; t < NTL; ++t) yres[t] = __ldcg(a.y + (size_t)(T0 + t) * a.y_stride + gr);
  }
}

// A shared tile whose partial this CTA has published: its counter's old value
// (held by the thread that added to it) and the count that makes this CTA the
// tile's last contributor.
template <int NTL>
struct TilePend {
  int tile = -1, old = 0, need = 0;
  float yres[NTL];   // the tile's residual rows, read at its start
};

// Update warps, stream-K: finish tile `tl` given this CTA's partial v for
// tokens [T0, T0 + NTL).  A tile the CTA owns whole goes straight to the
// epilogue.  Otherwise the partial is published (slot 0: the CTA's first
// tile, slot 1: its last) and counted, and the count's answer is left
// pending, to be read by tile_resolve at the end of the CTA's range, so that
// the memory round trip never stalls the update warps mid-stream.  Every
// update warp of the CTA takes part.
template <int EPI, int NT, int T0, int NTL>
QHL_DEV void gemv_finish_tile(const GemvArgs& a, int cta, const StreamK& sk, int i0, int i1, int tl, float (&v)[NTL],
                              const float (&yres)[NTL], const float* rstd, float* ex, TilePend<NTL>& pend,
                              int quarter, int lane, const UpdSlice& us) {
  const int r = quarter * 32 + lane;
  const int t_lo = tl * a.chunks, t_hi = t_lo + a.chunks;
  if (t_lo >= i0 && t_hi <= i1) {
    gemv_epilogue<EPI, T0, NTL>(a, tl, v, rstd, ex, quarter, lane, us, yres);
    return;
  }
#pragma unroll
  for (int t = 0; t < NTL; ++t) pend.yres[t] = yres[t];
  const int first_tile = i0 / a.chunks;
  float* mine = a.partials + (size_t)(2 * cta + (tl == first_tile ? 0 : 1)) * NT * kTileRows;
#pragma unroll
  for (int t = 0; t < NTL; ++t) mine[(T0 + t) * kTileRows + r] = v[t];
  named_sync(us.barall, us.nall);   // every update thread's partial stores come before the release below
  pend.tile = tl;
  pend.need = sk.owner(t_hi - 1) - sk.owner(t_lo);
  if (T0 == 0 && r == 0) {
    __threadfence();
    pend.old = atomicAdd(&a.counters[tl], 1);   // read in tile_resolve
  }
}

// Read a pending tile's count: if this CTA was the tile's last contributor,
// sum every contributor's partial in CTA order (tile tl is the first tile of
// every contributor after cf, and of cf exactly when cf's range starts at the
// tile's first item) and run the epilogue.
template <int EPI, int NT, int T0, int NTL>
QHL_DEV void tile_resolve(const GemvArgs& a, const StreamK& sk, TilePend<NTL>& pend, const float* rstd, float* ex,
                          int quarter, int lane, const UpdSlice& us) {
  const int r = quarter * 32 + lane;
  const int tl = pend.tile;
  const bool last = bar_or(us.barall, us.nall, T0 == 0 && r == 0 && pend.old == pend.need);
  pend.tile = -1;
  if (!last) return;
  __threadfence();   // every thread orders its partial loads after the count
  const int t_lo = tl * a.chunks, t_hi = t_lo + a.chunks;
  const int cf = sk.owner(t_lo), cl = sk.owner(t_hi - 1);
  const int cf_slot = sk.begin(cf) == t_lo ? 0 : 1;
  float acc[NTL];
  constexpr int CB = 4;
  for (int c0 = cf; c0 <= cl; c0 += CB) {
    float pv[CB][NTL];
#pragma unroll
    for (int k = 0; k < CB; ++k) {
      const int c = c0 + k;
      if (c <= cl) {
        const float* pc = a.partials + (size_t)(2 * c + (c == cf ? cf_slot : 0)) * NT * kTileRows;
#pragma unroll
        for (int t = 0; t < NTL; ++t) pv[k][t] = ld_cg_once(pc + (T0 + t) * kTileRows + r);
      }
    }
#pragma unroll
    for (int k = 0; k < CB; ++k)
      if (c0 + k <= cl) {
#pragma unroll
        for (int t = 0; t < NTL; ++t) acc[t] = (c0 + k == cf) ? pv[k][t] : __fadd_rn(acc[t], pv[k][t]);
      }
  }
  gemv_epilogue<EPI, T0, NTL>(a, tl, acc, rstd, ex, quarter, lane, us, pend.yres);
  if (T0 == 0 && r == 0) a.counters[tl] = 0;
}

// Pointers of one CTA's GEMV machinery in shared memory (layout of config C).
template <class C>
struct GemvSmem {
  uint8_t* wring;
  uint8_t* xring;
  float* ex;
  uint8_t* extra;
  float* rstd;
  uint32_t* tslot;
  int* flag;
  uint64_t *wfull, *wempty, *xfull, *sfull, *xempty, *afull, *afree, *dfull, *dfree, *drain;
  QHL_DEV explicit GemvSmem(uint8_t* base) {
    wring = base;
    xring = base + C::kXOff;
    ex = reinterpret_cast<float*>(base + C::kEpiOff);
    extra = base + C::kExtraOff;
    rstd = reinterpret_cast<float*>(base + C::kRstdOff);
    tslot = reinterpret_cast<uint32_t*>(base + C::kSlotOff);
    flag = reinterpret_cast<int*>(base + C::kSlotOff + 4);
    wfull = reinterpret_cast<uint64_t*>(base + C::kBarOff);
    wempty = wfull + C::kSW;
    xfull = wfull + 2 * C::kSW;
    sfull = xfull + C::kSX;
    xempty = sfull + C::kSX;
    afull = xempty + C::kSX;
    afree = afull + C::kNA;
    dfull = afree + C::kNA;
    dfree = dfull + C::kND;
    drain = dfree + C::kND;
  }
  // barrier set-up by the 32 lanes of one warp
  QHL_DEV void init(int lane) const {
    for (int s = lane; s < C::kSW; s += 32) {
      mbar_init(smem_u32(&wfull[s]), 1);
      mbar_init(smem_u32(&wempty[s]), C::kUnpackWarps);
    }
    for (int s = lane; s < C::kSX; s += 32) {
      mbar_init(smem_u32(&xfull[s]), 1);
      mbar_init(smem_u32(&sfull[s]), 1);
      mbar_init(smem_u32(&xempty[s]), C::kUpdateWarps);
    }
    for (int b = lane; b < C::kNA; b += 32) {
      mbar_init(smem_u32(&afull[b]), C::kUnpackWarps);
      mbar_init(smem_u32(&afree[b]), 1);
    }
    for (int b = lane; b < C::kND; b += 32) {
      mbar_init(smem_u32(&dfull[b]), 1);
      mbar_init(smem_u32(&dfree[b]), C::kUpdateWarps);
    }
    if (lane == 0) mbar_init(smem_u32(drain), C::kMmaThreads);
    fence_mbar_init();
  }
};

// D buffer of group g of item K and the index of that use among the
// buffer's uses (its barrier phase).  With two MMA threads each owns half of
// the buffers (thread K & 1 takes item K), so that every barrier is waited on
// by one thread, one phase at a time: a parity wait cannot tell a phase from
// the one two before it.
template <class C>
QHL_DEV void d_slot(uint32_t K, int g, int& db, uint32_t& use) {
  if constexpr (C::kMmaThreads == 1) {
    const uint32_t gc = K * C::kNG + g;
    db = gc % C::kND;
    use = gc / C::kND;
  } else {
    constexpr int kOwn = C::kND / 2;
    const uint32_t lg = (K >> 1) * C::kNG + g;   // the group's index among its thread's groups
    db = (int)(K & 1u) + 2 * (int)(lg % kOwn);
    use = lg / kOwn;
  }
}

// The roles below process this CTA's items [i0, i0 + n) of one projection.  K0
// is the running count of items the CTA has taken through its rings before
// this projection: ring slots, buffer indices and barrier phases follow from
// the running count K0 + k, so consecutive projections can share one CTA's
// rings and buffers.

// Copies of one item's parts into the rings (producer thread).
template <class C>
QHL_DEV void issue_weights(const GemvArgs& a, const GemvSmem<C>& S, int item, uint32_t K, uint64_t pol) {
  constexpr int QT = C::kQT;
  const int s = K % C::kSW;
  mbar_arrive_expect_tx(smem_u32(&S.wfull[s]), C::kQB);
  bulk_g2s(smem_u32(S.wring + s * C::kQB), a.W + (size_t)item * QLayout<QT>::kItemBytes, C::kQB,
           smem_u32(&S.wfull[s]), pol);
}
template <class C>
QHL_DEV void issue_scales(const GemvArgs& a, const GemvSmem<C>& S, int item, uint32_t K, uint64_t pol) {
  constexpr int QT = C::kQT;
  const int s = K % C::kSX;
  mbar_arrive_expect_tx(smem_u32(&S.sfull[s]), QLayout<QT>::kScaleBytes);
  bulk_g2s(smem_u32(S.xring + s * C::kXS), a.W + (size_t)item * QLayout<QT>::kItemBytes + C::kQB,
           QLayout<QT>::kScaleBytes, smem_u32(&S.sfull[s]), pol);
}
template <class C>
QHL_DEV void issue_x(const GemvArgs& a, const GemvSmem<C>& S, int chunk, uint32_t K) {
  constexpr int QT = C::kQT, NT = C::kNT;
  const int s = K % C::kSX;
  mbar_arrive_expect_tx(smem_u32(&S.xfull[s]), NT * kQChunkBytes);
  for (int t = 0; t < NT; ++t)
    bulk_g2s_plain(smem_u32(S.xring + s * C::kXS + QLayout<QT>::kScaleBytes + t * kQChunkBytes),
                   a.qx + (size_t)t * a.qx_stride + (size_t)chunk * kQChunkBytes, kQChunkBytes,
                   smem_u32(&S.xfull[s]));
}

// Producers of one stand-alone projection (K0 = 0), two threads in two warps
// so that neither ring waits for the other's slots.  The weight thread keeps
// the weight ring full: it requests the first ring (beyond one token, the
// first two items and the rest once item 0 has landed; the weights never
// depend on earlier kernels), and then each item as soon as its slot is
// released, sleeping in the barrier wait in between.  The x thread does the
// same for the x ring (an item's block scales and x columns); the x columns
// are written by the previous kernel, so they are requested only once
// griddepcontrol.wait has returned.  Each returns false on a timeout.
template <class C>
QHL_DEV bool produce_weights(const GemvArgs& a, const GemvSmem<C>& S, int cta, int i0, int n) {
  constexpr int QT = C::kQT;
  constexpr int SW = C::kSW;
  const uint64_t pol = policy_evict_first();
  for (int k = 0; k < n; ++k) {
    if (k >= SW && !mbar_wait(smem_u32(&S.wempty[k % SW]), ((k / SW) - 1) & 1u, a.err, a.wait_limit)) return false;
    // beyond one token (a twelve-item ring) the rest of the first ring only
    // once the first item is in: the copies in flight share the SM's
    // bandwidth, and the pipeline starts on item 0; the four-item ring of one
    // token goes out at once
    if (C::kNT > 1 && k == 2 && n > 2 && !(cta == 0 && a.fault_item == 0) &&
        !mbar_wait(smem_u32(&S.wfull[0]), 0u, a.err, a.wait_limit))
      return false;
    if (cta == 0 && k == a.fault_item) continue;   // injected failure: this slot never fills
    issue_weights<C>(a, S, i0 + k, (uint32_t)k, pol);
  }
  if (a.next_W && cta < a.next_workers) {
    // every own item is on its way: warm L2 with the next projection's first
    // items of this CTA index while the consumers finish
    const StreamK skn(a.next_items, a.next_workers);
    const int j0 = skn.begin(cta), nj = min(SW, skn.begin(cta + 1) - j0);
    for (int k = 0; k < nj; ++k)
      bulk_prefetch_l2(a.next_W + (size_t)(j0 + k) * QLayout<QT>::kItemBytes, QLayout<QT>::kItemBytes);
  }
  return true;
}
// The x producer is a whole warp.  Its lane 0 bulk-copies each item's block
// scales and x columns into the x ring as slots are released.  Bulk copies of
// one SM are served in order, so at the start of a projection the first x
// columns (a few KB from L2) queue behind the weight copies already requested.
// At two tokens, behind a twelve-item weight ring, the whole warp moves the
// first two items' x columns through the load/store path instead (each lane
// loads its 16-byte pieces, stores them and fences them for the tensor core's
// async proxy).  At one token the four-item ring holds few copies ahead of
// them, and the bulk copies alone are faster (0 to 4 head items on the
// 64-layer decode pass: 234.6, 232.9, 232.1, 231.7, 231.0 tok/s).
template <class C>
QHL_DEV bool produce_x(const GemvArgs& a, const GemvSmem<C>& S, int i0, int n, int lane) {
  constexpr int QT = C::kQT, NT = C::kNT, SX = C::kSX;
  constexpr int kPer = kQChunkBytes / 16 / 32;      // 16-byte pieces per lane and token
  constexpr int kHead = NT == 2 ? 2 : 0;            // items through the load/store path (16 pieces a lane)
  static_assert(kHead <= SX, "head items take distinct x slots");
  const uint64_t pol = policy_evict_first();
  if (lane == 0)
    for (int k = 0; k < n && k < SX; ++k) issue_scales<C>(a, S, i0 + k, (uint32_t)k, pol);
  pdl_wait();
  int c = i0 % a.chunks;   // chunk of the next item, stepped without division
  const int nh = min(kHead, n);
  if constexpr (kHead > 0) {
    uint4 v[kHead > 0 ? kHead : 1][NT * kPer];
    int cc = c;
#pragma unroll
    for (int j = 0; j < kHead; ++j) {
      if (j < nh)
#pragma unroll
        for (int i = 0; i < NT * kPer; ++i)
          v[j][i] = ld_cg_once(reinterpret_cast<const uint4*>(a.qx + (size_t)(i / kPer) * a.qx_stride +
                                                              (size_t)cc * kQChunkBytes) +
                               (i % kPer) * 32 + lane);
      if (++cc == a.chunks) cc = 0;
    }
#pragma unroll
    for (int j = 0; j < kHead; ++j)
      if (j < nh) {
        uint8_t* slot = S.xring + j * C::kXS + QLayout<QT>::kScaleBytes;
#pragma unroll
        for (int i = 0; i < NT * kPer; ++i)
          *reinterpret_cast<uint4*>(slot + (i / kPer) * kQChunkBytes + ((i % kPer) * 32 + lane) * 16) = v[j][i];
      }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0)
      for (int j = 0; j < nh; ++j) mbar_arrive(smem_u32(&S.xfull[j]));
    c = cc;
  }
  if (lane != 0) return true;
  for (int k = nh; k < n; ++k) {
    if (k >= SX) {
      if (!mbar_wait(smem_u32(&S.xempty[k % SX]), ((k / SX) - 1) & 1u, a.err, a.wait_limit)) return false;
      issue_scales<C>(a, S, i0 + k, (uint32_t)k, pol);
    }
    issue_x<C>(a, S, c, (uint32_t)k);
    if (++c == a.chunks) c = 0;
  }
  return true;
}

// Unpack warps (thread = row r of quarter `quarter`): each item's quants into
// the A operand in tensor memory.  With C::kUnpackWarps = 8 two warps share a
// lane quarter and `part` 0 / 1 takes blocks 0..3 / 4..7 of every item.
// Returns false on a timeout.
template <class C>
QHL_DEV bool unpack_items(const GemvArgs& a, const GemvSmem<C>& S, uint32_t tmem, int n, uint32_t K0, int quarter,
                          int part, int lane) {
  constexpr int QT = C::kQT;
  constexpr int kHalves = 8 / C::kUnpackWarps;   // groups of four blocks per warp and item
  static_assert(C::kUnpackWarps == 4 || C::kUnpackWarps == 8, "unpack warps");
  const int r = quarter * 32 + lane;
  const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
  for (int k = 0; k < n; ++k) {
    const uint32_t K = K0 + k;
    const int ab = K % C::kNA, sw = K % C::kSW;
    // the A buffer is free once the MMAs of item K - NA have completed: its
    // afree barrier, or with one commit per item the dfull barrier of its D
    // buffer; for K < NA the weight barrier stands in (nothing to wait for)
    uint32_t b_free = smem_u32(&S.wfull[sw]), p_free = (K / C::kSW) & 1u;
    if (K >= (uint32_t)C::kNA) {
      if constexpr (C::kOneCommit) {
        int db;
        uint32_t use;
        d_slot<C>(K - C::kNA, 0, db, use);
        b_free = smem_u32(&S.dfull[db]);
        p_free = use & 1u;
      } else {
        b_free = smem_u32(&S.afree[ab]);
        p_free = ((K / C::kNA) - 1) & 1u;
      }
    }
    if (!mbar_test2(smem_u32(&S.wfull[sw]), (K / C::kSW) & 1u, b_free, p_free) &&
        (!mbar_wait(smem_u32(&S.wfull[sw]), (K / C::kSW) & 1u, a.err, a.wait_limit) ||
         !mbar_wait(b_free, p_free, a.err, a.wait_limit)))
      return false;
    tc_fence_after();
    const uint8_t* q = S.wring + sw * C::kQB;
    const uint32_t ta = tmem + lane_base + ab * C::kACols;
    // the row's loads of four blocks first (one round of shared-memory
    // latency), then one tensor-memory store of the four
#pragma unroll
    for (int hh = 0; hh < kHalves; ++hh) {
      const int h = part * kHalves + hh;
      uint32_t av[32];
      if constexpr (QT == kQ4_0) {
        uint4 w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] = *reinterpret_cast<const uint4*>(q + q4_off(4 * h + j, r));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t blk[8];
          q4_unpack(w[j], blk);
#pragma unroll
          for (int i = 0; i < 8; ++i) av[8 * j + i] = blk[i];
        }
      } else {
        uint4 w[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          w[2 * j] = *reinterpret_cast<const uint4*>(q + q8_off(4 * h + j, 0, r));
          w[2 * j + 1] = *reinterpret_cast<const uint4*>(q + q8_off(4 * h + j, 1, r));
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          av[4 * j] = w[j].x; av[4 * j + 1] = w[j].y; av[4 * j + 2] = w[j].z; av[4 * j + 3] = w[j].w;
        }
      }
      tmem_st32(ta + 32 * h, av);
    }
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(smem_u32(&S.afull[ab]));
      mbar_arrive(smem_u32(&S.wempty[sw]));
    }
  }
  return true;
}

// MMA issuer (one thread): per item and block one M = 128, N = 8 per token,
// K = 32 integer MMA into a D buffer.  With C::kMmaThreads = 2 two threads
// take alternate items (`sel` = 0 / 1: even / odd running count), so that one
// thread's barrier checks and bookkeeping overlap the other's MMAs.  Returns
// false on a timeout.
template <class C>
QHL_DEV bool mma_items(const GemvArgs& a, const GemvSmem<C>& S, uint32_t tmem, int n, uint32_t K0, int sel) {
  constexpr int QT = C::kQT;
  constexpr uint32_t idesc = idesc_i8(QT == kQ8_0, kTileRows, C::kN);
  for (int k = 0; k < n; ++k) {
    const uint32_t K = K0 + k;
    if (C::kMmaThreads == 2 && (int)(K & 1u) != sel) continue;
    const int ab = K % C::kNA, sx = K % C::kSX;
    // fast path: the A buffer, the x slot and the first D buffer all ready
    int db0;
    uint32_t use0;
    d_slot<C>(K, 0, db0, use0);
    // (use0 = 0: parity 1 names the phase before the fresh barrier's first)
    const bool ready = mbar_test3(smem_u32(&S.afull[ab]), (K / C::kNA) & 1u, smem_u32(&S.xfull[sx]),
                                  (K / C::kSX) & 1u, smem_u32(&S.dfree[db0]), (use0 - 1) & 1u);
    if (!ready && (!mbar_wait(smem_u32(&S.afull[ab]), (K / C::kNA) & 1u, a.err, a.wait_limit) ||
                   !mbar_wait(smem_u32(&S.xfull[sx]), (K / C::kSX) & 1u, a.err, a.wait_limit)))
      return false;
    tc_fence_after();
    const uint32_t xs = smem_u32(S.xring + sx * C::kXS + QLayout<QT>::kScaleBytes);
    const uint64_t desc0 = smem_desc_kmajor(xs, 128, kQChunkBytes);   // block b: start address + b * 256 / 16
    for (int g = 0; g < C::kNG; ++g) {
      int db;
      uint32_t use;
      d_slot<C>(K, g, db, use);
      if (!(ready && g == 0) && use >= 1 && !mbar_wait(smem_u32(&S.dfree[db]), (use - 1) & 1u, a.err, a.wait_limit))
        return false;
      tc_fence_after();
#pragma unroll
      for (int j = 0; j < C::kGB; ++j) {
        const int b = g * C::kGB + j;
        const uint64_t desc = desc0 + (uint64_t)(b * (kQBlockBytes >> 4));
        mma_i8_ts(tmem + C::kDOff + db * C::kDCols + j * C::kN, tmem + ab * C::kACols + 8 * b, desc, idesc, false);
      }
      tc_commit(&S.dfull[db]);
    }
    if constexpr (!C::kOneCommit) tc_commit(&S.afree[ab]);
  }
  return true;
}

// Update warps (thread = row r of quarter `quarter`; one set of four warps per
// token slice [T0, T0 + NTL)): f32 block updates of every item in order, then
// the tile finish at each tile boundary.  rstd[] must hold the input's RMS
// scale.  The update warps take every decision together.  Returns false on a
// timeout.
template <class C, int EPI, int T0, int NTL>
QHL_DEV bool update_items(const GemvArgs& a, const GemvSmem<C>& S, uint32_t tmem, int cta, int i0, int n,
                          uint32_t K0, int quarter, int lane, const UpdSlice& us) {
  constexpr int QT = C::kQT, NT = C::kNT;
  const int r = quarter * 32 + lane;
  const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
  const StreamK sk(a.tiles * a.chunks, a.workers);
  const int i1 = i0 + n;
  float acc[NTL];
#pragma unroll
  for (int t = 0; t < NTL; ++t) acc[t] = 0.f;
  int tile = i0 / a.chunks;
  int ci = i0 - tile * a.chunks;   // chunk of item k within its tile
  bool timed_out = false;
  TilePend<NTL> pend[2];           // a CTA shares at most two tiles: its first and its last
  int np = 0;
  float yres[NTL];
  load_residual<EPI, T0, NTL>(a, tile, r, yres);
  for (int k = 0; k < n; ++k, ++ci) {
    const uint32_t K = K0 + k;
    const int sx = K % C::kSX;
    if (ci == a.chunks) {   // item k starts the next tile: finish this one
      if (!bar_and(us.barall, us.nall, !timed_out)) return false;
      gemv_finish_tile<EPI, NT, T0, NTL>(a, cta, sk, i0, i1, tile, acc, yres, S.rstd, S.ex, pend[np], quarter, lane,
                                         us);
      if (pend[np].tile >= 0) ++np;
#pragma unroll
      for (int t = 0; t < NTL; ++t) acc[t] = 0.f;
      ++tile;
      ci = 0;
      load_residual<EPI, T0, NTL>(a, tile, r, yres);
    }
    const uint8_t* xsl = S.xring + sx * C::kXS;
    uint4 sc4 = make_uint4(0, 0, 0, 0);
    uint32_t known = 0;   // groups of this item whose D is known to be complete
    for (int g = 0; g < C::kNG; ++g) {
      int db;
      uint32_t use;
      d_slot<C>(K, g, db, use);
      // (the first group also waits for the x slot itself: its scales and
      // block metadata are read here, not only by the MMA; later groups test
      // the next group's D in the same round trip).  After a timeout this
      // warp waits for nothing more; the update warps agree on stopping at the
      // next tile boundary, before any named barrier they share.
      bool ready = (known >> g) & 1u;
      if (!timed_out && !ready && g > 0) {
        if (g + 1 < C::kNG) {
          int db1;
          uint32_t use1;
          d_slot<C>(K, g + 1, db1, use1);
          const uint32_t m = mbar_test2m(smem_u32(&S.dfull[db]), use & 1u, smem_u32(&S.dfull[db1]), use1 & 1u);
          ready = m & 1u;
          if (m == 3u) known |= 1u << (g + 1);
        } else {
          ready = mbar_test(smem_u32(&S.dfull[db]), use & 1u);
        }
      }
      if (!timed_out && !ready && !(g == 0 && mbar_test3(smem_u32(&S.dfull[db]), use & 1u, smem_u32(&S.xfull[sx]),
                                                         (K / C::kSX) & 1u, smem_u32(&S.sfull[sx]), (K / C::kSX) & 1u)))
        timed_out = !(mbar_wait(smem_u32(&S.dfull[db]), use & 1u, a.err, a.wait_limit) &&
                      (g > 0 || (mbar_wait(smem_u32(&S.xfull[sx]), (K / C::kSX) & 1u, a.err, a.wait_limit) &&
                                 mbar_wait(smem_u32(&S.sfull[sx]), (K / C::kSX) & 1u, a.err, a.wait_limit))));
      if (timed_out) continue;
      tc_fence_after();
      if (g == 0) sc4 = *reinterpret_cast<const uint4*>(xsl + r * 16);   // the row's 8 block scales
      int dv[C::kGB][NTL][4];
#pragma unroll
      for (int j = 0; j < C::kGB; ++j)
#pragma unroll
        for (int t = 0; t < NTL; ++t)
          tmem_ld4(tmem + lane_base + C::kDOff + db * C::kDCols + j * C::kN + (T0 + t) * 8, dv[j][t]);
      tmem_ld_wait();
      const uint32_t scw[4] = {sc4.x, sc4.y, sc4.z, sc4.w};
#pragma unroll
      for (int j = 0; j < C::kGB; ++j) {
        const int b = g * C::kGB + j;
        const uint32_t w = scw[b >> 1];
        const float d = __half2float(__ushort_as_half(static_cast<unsigned short>((b & 1) ? (w >> 16) : (w & 0xFFFFu))));
#pragma unroll
        for (int t = 0; t + 1 < NTL; t += 2) {   // token pairs on packed f32 lanes
          const int4 m0 = *reinterpret_cast<const int4*>(xsl + QLayout<QT>::kScaleBytes + (T0 + t) * kQChunkBytes +
                                                         b * kQBlockBytes + kQMetaOff);
          const int4 m1 = *reinterpret_cast<const int4*>(xsl + QLayout<QT>::kScaleBytes + (T0 + t + 1) * kQChunkBytes +
                                                         b * kQBlockBytes + kQMetaOff);
          const float2 r2 = block_update2<QT>(make_float2(acc[t], acc[t + 1]), d,
                                              make_float2(__int_as_float(m0.x), __int_as_float(m1.x)), dv[j][t][0],
                                              dv[j][t][1], dv[j][t][2], dv[j][t + 1][0], dv[j][t + 1][1],
                                              dv[j][t + 1][2], make_int2(m0.y, m1.y), make_int2(m0.z, m1.z));
          acc[t] = r2.x;
          acc[t + 1] = r2.y;
        }
        if constexpr (NTL % 2 == 1) {
          constexpr int t = NTL - 1;
          const int4 m = *reinterpret_cast<const int4*>(xsl + QLayout<QT>::kScaleBytes + (T0 + t) * kQChunkBytes +
                                                        b * kQBlockBytes + kQMetaOff);
          acc[t] = block_update<QT>(acc[t], d, __int_as_float(m.x), dv[j][t][0], dv[j][t][1], dv[j][t][2], m.y, m.z);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&S.dfree[db]));
    }
    __syncwarp();
    if (!timed_out && lane == 0) mbar_arrive(smem_u32(&S.xempty[sx]));
  }
  if (!bar_and(us.barall, us.nall, !timed_out)) return false;
  gemv_finish_tile<EPI, NT, T0, NTL>(a, cta, sk, i0, i1, tile, acc, yres, S.rstd, S.ex, pend[np], quarter, lane, us);
  if (pend[np].tile >= 0) ++np;
  for (int j = 0; j < np; ++j) tile_resolve<EPI, NT, T0, NTL>(a, sk, pend[j], S.rstd, S.ex, quarter, lane, us);
  return true;
}
// One set of four update warps owning every token.
template <class C, int EPI>
QHL_DEV bool update_items(const GemvArgs& a, const GemvSmem<C>& S, uint32_t tmem, int cta, int i0, int n,
                          uint32_t K0, int quarter, int lane) {
  return update_items<C, EPI, 0, C::kNT>(a, S, tmem, cta, i0, n, K0, quarter, lane,
                                         UpdSlice{kBarUpdate, kBarUpdate, 128});
}

// The input's RMS scale of tokens [t0, t0 + nt) into S.rstd (one set of
// four update warps, barrier `bar`; after the dependency on the kernel that
// wrote ss_in is resolved).
template <class C>
QHL_DEV void load_rstd(const GemvArgs& a, const GemvSmem<C>& S, int quarter, int lane, int t0 = 0, int nt = C::kNT,
                       int bar = kBarUpdate) {
  for (int t = t0 + quarter; t < t0 + nt; t += 4) {
    const float rs = a.ss_in ? rstd_warp(a.ss_in + (size_t)t * a.ss_stride, a.ss_tiles, a.inv_dim, a.eps, lane) : 1.f;
    if (lane == 0) S.rstd[t] = rs;
  }
  named_sync(bar, 128);
}

template <int QT, int NT, int EPI>
__global__ void __launch_bounds__(GemvCfg<QT, NT>::kThreads, GemvCfg<QT, NT>::kMinBlocks) qgemv_kernel(const GemvArgs a) {
  using C = GemvCfg<QT, NT>;
  extern __shared__ __align__(16) uint8_t gsmem[];
  const GemvSmem<C> S(gsmem);
  const int cta = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) pdl_launch();
  if (cta >= a.workers) return;
  const StreamK sk(a.tiles * a.chunks, a.workers);
  const int i0 = sk.begin(cta), n = sk.begin(cta + 1) - i0;
  if (n == 0) return;

  // The weight producer sets up the barriers and starts its ring at once; the
  // x producer waits for the barriers only; the other warps also wait for the
  // tensor-memory address.  (Counts: kBarInit 32 + 32, kBarSetup 32 + 32
  // arriving + the rest waiting.)
  if (warp == kProducerWarp) {
    S.init(lane);
    __syncwarp();
    named_arrive(kBarInit, 64);
    named_arrive(kBarSetup, C::kThreads);
    if (lane == 0 && !produce_weights<C>(a, S, cta, i0, n)) drain_inflight_copies();   // error path
    return;   // the producers take no part in the tensor-memory teardown
  }
  if (warp == C::kXWarp) {
    named_sync(kBarInit, 64);
    named_arrive(kBarSetup, C::kThreads);
    if (!produce_x<C>(a, S, i0, n, lane) && lane == 0) drain_inflight_copies();   // error path
    return;
  }
  if (warp == kMmaWarp) tmem_alloc(S.tslot, C::kTmemCols);
  tc_fence_before();
  named_sync(kBarSetup, C::kThreads);
  tc_fence_after();
  const uint32_t tmem = *S.tslot;

  bool ok = true;
  if (warp == kMmaWarp || warp == C::kMma2Warp) {
    if (lane == 0 && (warp == kMmaWarp || C::kMmaThreads == 2)) {
      ok = mma_items<C>(a, S, tmem, n, 0, warp == kMmaWarp ? 0 : 1);
      // every MMA this thread issued has completed before tensor memory goes
      tc_commit(S.drain);
      if (!mbar_wait(smem_u32(S.drain), 0, a.err, a.wait_limit)) ok = false;
    }
    __syncwarp();
  } else if (warp < C::kUpdateWarp0) {
    ok = unpack_items<C>(a, S, tmem, n, 0, warp & 3, (warp - kUnpackWarp0) >> 2, lane);
  } else {
    pdl_wait();   // ss_in, the residual stream and the scratch come from earlier kernels
    if constexpr (C::kUpdateWarps == 4) {
      load_rstd<C>(a, S, warp & 3, lane);
      ok = update_items<C, EPI>(a, S, tmem, cta, i0, n, 0, warp & 3, lane);
    } else {
      constexpr int NA = C::kNTA;
      if (warp < C::kUpdateWarp0 + 4) {
        load_rstd<C>(a, S, warp & 3, lane, 0, NA, kBarUpdate);
        ok = update_items<C, EPI, 0, NA>(a, S, tmem, cta, i0, n, 0, warp & 3, lane,
                                         UpdSlice{kBarUpdate, kBarUpdateAll, 256});
      } else {
        load_rstd<C>(a, S, warp & 3, lane, NA, NT - NA, kBarUpdate2);
        ok = update_items<C, EPI, NA, NT - NA>(a, S, tmem, cta, i0, n, 0, warp & 3, lane,
                                               UpdSlice{kBarUpdate2, kBarUpdateAll, 256});
      }
    }
  }
  // ---------------- teardown: tensor memory back, after every MMA and load --
  tc_fence_before();
  named_sync(kBarTmem, C::kThreads - 64);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
  if (!ok && lane == 0) drain_inflight_copies();   // error path
}

}  // namespace qhl
