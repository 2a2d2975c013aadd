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

// Warp roles.
constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kUnpackWarp0 = 2;   // warps 2..5
constexpr int kUpdateWarp0 = 6;   // warps 6..9
constexpr int kGemvCtaThreads = 320;
// Named barriers: 1 = the four update warps, 2 = every warp that touches tensor memory.
constexpr int kBarUpdate = 1;
constexpr int kBarTmem = 2;

// Geometry and shared-memory layout of one (weight type, token count).
template <int QT, int NT>
struct GemvCfg {
  static constexpr int kN = NT == 1 ? 8 : 16 * ((NT + 1) / 2);   // MMA N: 8 rows per token, padded
  static constexpr int kNTP = kN / 8;                              // token regions in an x slot
  static constexpr int kGB = (64 / kN) >= 8 ? 8 : ((64 / kN) >= 1 ? 64 / kN : 1);   // blocks per D group
  static constexpr int kNG = 8 / kGB;                              // D groups per item
  static constexpr int kDCols = kGB * kN;                          // tensor-memory columns of a D buffer
  static constexpr int kACols = 64;                                // 8 blocks x 32 bytes / 4
  static constexpr int kDOff = 2 * kACols;
  static constexpr int kTmemCols = kDOff + 2 * kDCols <= 256 ? 256 : 512;
  static constexpr int kQB = QLayout<QT>::kQuantBytes;
  static constexpr int kXS = QLayout<QT>::kScaleBytes + kNTP * kQChunkBytes;   // x slot: scales, then tokens
  // two CTAs per SM (this projection and the next) at one and two tokens (Q4_0)
  static constexpr bool kPair = QT == kQ4_0 && NT <= 2;
  static constexpr int kBudget = kPair ? 110 * 1024 : 200 * 1024;
  static constexpr int kEpi = NT * kTileRows * 4;                  // epilogue exchange [NT][128] f32
  static constexpr int kFixed = kEpi + 16 * 4 + 16 + 320;          // + rstd, tmem slot, barriers
  static constexpr int kSX = kPair ? 6 : 3;
  static constexpr int kSW0 = (kBudget - kFixed - kSX * kXS) / kQB;
  static constexpr int kSW = kSW0 > 8 ? 8 : kSW0;
  static constexpr int kMinBlocks = kPair ? 2 : 1;
  // shared-memory layout (the rings first; every slot 16-byte aligned)
  static constexpr int kXOff = kSW * kQB;
  static constexpr int kEpiOff = kXOff + kSX * kXS;
  static constexpr int kRstdOff = kEpiOff + kEpi;
  static constexpr int kSlotOff = kRstdOff + 16 * 4;
  static constexpr int kBarOff = kSlotOff + 16;
  // barriers: wfull[SW], wempty[SW], xfull[SX], xempty[SX], afull[2], afree[2], dfull[2], dfree[2], drain
  static constexpr int kNumBars = 2 * kSW + 2 * kSX + 9;
  static constexpr int kSmem = kBarOff + kNumBars * 8;
  static_assert(kSW >= 2, "weight ring too shallow");
  static_assert(kNumBars * 8 <= 320, "barrier area");
  static_assert(kSmem <= kBudget, "shared-memory budget");
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

// Epilogue of one finished tile by the four update warps, thread = tile row r
// (quarter q = r / 32); v[t] = the tile's final sums for row r.
template <int EPI, int NT>
QHL_DEV void gemv_epilogue(const GemvArgs& a, int tile, const float (&v)[NT], const float* rstd, float* ex, int quarter,
                           int lane) {
  const int r = quarter * 32 + lane;
  if constexpr (EPI == EPI_STORE) {
    const int gr = tile * kTileRows + r;
    if (gr < a.out_valid)
#pragma unroll
      for (int t = 0; t < NT; ++t) a.y[(size_t)t * a.y_stride + gr] = __fmul_rn(v[t], rstd[t]);
  } else if constexpr (EPI == EPI_SWIGLU) {
    // rows 0..63: gate rows of features 64 tile + r; rows 64..127 the matching up rows
    if (r >= 64)
#pragma unroll
      for (int t = 0; t < NT; ++t) ex[t * kTileRows + r - 64] = __fmul_rn(v[t], rstd[t]);
    named_sync(kBarUpdate, 128);
    if (r < 64) {
      const int f = tile * 64 + r;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float u = 0.f;
        if (f < a.out_valid) {
          const float g = __fmul_rn(v[t], rstd[t]);
          const float up = ex[t * kTileRows + r];
          u = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.f, expf(-g))), up);   // silu(g) * up
        }
        qact_store_block(u, a.qout + (size_t)t * a.qout_stride, tile * 2 + quarter, lane);
      }
    }
    named_sync(kBarUpdate, 128);
  } else {
    const int gr = tile * kTileRows + r;
    const bool valid = gr < a.out_valid;
    const float gam = a.qout && valid ? __ldg(a.gamma_next + gr) : 0.f;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float hn = 0.f;
      if (valid) {
        hn = __fadd_rn(__ldcg(a.y + (size_t)t * a.y_stride + gr), v[t]);
        a.y[(size_t)t * a.y_stride + gr] = hn;
      }
      if (a.qout) qact_store_block(__fmul_rn(hn, gam), a.qout + (size_t)t * a.qout_stride, tile * 4 + quarter, lane);
      if (a.ss_out) {
        const float s = tile_sumsq(hn, ex + 4 * t, quarter, lane, kBarUpdate);
        if (r == 0) a.ss_out[(size_t)t * a.ss_out_stride + tile] = s;
      }
    }
  }
}

// Update warps: finish tile `tl` given this CTA's partial v (stream-K fix-up
// if the tile is shared, then the epilogue).
template <int EPI, int NT>
QHL_DEV void gemv_finish_tile(const GemvArgs& a, int cta, const StreamK& sk, int i0, int i1, int tl, float (&v)[NT],
                              const float* rstd, float* ex, int* flag, int quarter, int lane) {
  const int r = quarter * 32 + lane;
  const int t_lo = tl * a.chunks, t_hi = t_lo + a.chunks;
  if (t_lo >= i0 && t_hi <= i1) {
    gemv_epilogue<EPI, NT>(a, tl, v, rstd, ex, quarter, lane);
    return;
  }
  // publish this CTA's partial (slot 0: its first tile, slot 1: its last)
  const int first_tile = i0 / a.chunks;
  float* mine = a.partials + (size_t)(2 * cta + (tl == first_tile ? 0 : 1)) * NT * kTileRows;
#pragma unroll
  for (int t = 0; t < NT; ++t) mine[t * kTileRows + r] = v[t];
  __threadfence();
  named_sync(kBarUpdate, 128);
  const int cf = sk.owner(t_lo), cl = sk.owner(t_hi - 1);
  if (r == 0) *flag = counter_add_acq_rel(&a.counters[tl]) == cl - cf ? 1 : 0;
  named_sync(kBarUpdate, 128);
  const int last = *flag;
  named_sync(kBarUpdate, 128);
  if (!last) return;
  __threadfence();   // every thread orders its partial loads after the acquire above
  // combine every contributor's partial in CTA order; tile tl is the first
  // tile of every contributor after cf, and of cf exactly when cf's range
  // starts at the tile's first item
  const int cf_slot = sk.begin(cf) == t_lo ? 0 : 1;
  float acc[NT];
  constexpr int CB = 4;
  for (int c0 = cf; c0 <= cl; c0 += CB) {
    float pv[CB][NT];
#pragma unroll
    for (int k = 0; k < CB; ++k) {
      const int c = c0 + k;
      if (c <= cl) {
        const float* pc = a.partials + (size_t)(2 * c + (c == cf ? cf_slot : 0)) * NT * kTileRows;
#pragma unroll
        for (int t = 0; t < NT; ++t) pv[k][t] = c == cta ? v[t] : ld_cg_once(pc + t * kTileRows + r);
      }
    }
#pragma unroll
    for (int k = 0; k < CB; ++k)
      if (c0 + k <= cl) {
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = (c0 + k == cf) ? pv[k][t] : __fadd_rn(acc[t], pv[k][t]);
      }
  }
  gemv_epilogue<EPI, NT>(a, tl, acc, rstd, ex, quarter, lane);
  if (r == 0) a.counters[tl] = 0;
}

template <int QT, int NT, int EPI>
__global__ void __launch_bounds__(kGemvCtaThreads, GemvCfg<QT, NT>::kMinBlocks) qgemv_kernel(const GemvArgs a) {
  using C = GemvCfg<QT, NT>;
  constexpr int SW = C::kSW, SX = C::kSX, QB = C::kQB, XS = C::kXS;
  extern __shared__ __align__(16) uint8_t gsmem[];
  uint8_t* wring = gsmem;
  uint8_t* xring = gsmem + C::kXOff;
  float* ex = reinterpret_cast<float*>(gsmem + C::kEpiOff);
  float* rstd = reinterpret_cast<float*>(gsmem + C::kRstdOff);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(gsmem + C::kSlotOff);
  int* flag = reinterpret_cast<int*>(gsmem + C::kSlotOff + 4);
  uint64_t* bars = reinterpret_cast<uint64_t*>(gsmem + C::kBarOff);
  uint64_t* wfull = bars;
  uint64_t* wempty = bars + SW;
  uint64_t* xfull = bars + 2 * SW;
  uint64_t* xempty = bars + 2 * SW + SX;
  uint64_t* afull = bars + 2 * SW + 2 * SX;
  uint64_t* afree = afull + 2;
  uint64_t* dfull = afull + 4;
  uint64_t* dfree = afull + 6;
  uint64_t* drain = afull + 8;

  const int cta = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) pdl_launch();
  if (cta >= a.workers) return;
  const StreamK sk(a.tiles * a.chunks, a.workers);
  const int i0 = sk.begin(cta), i1 = sk.begin(cta + 1), n = i1 - i0;
  if (n == 0) return;

  if (tid == 0) {
    for (int s = 0; s < SW; ++s) {
      mbar_init(smem_u32(&wfull[s]), 1);
      mbar_init(smem_u32(&wempty[s]), 4);
    }
    for (int s = 0; s < SX; ++s) {
      mbar_init(smem_u32(&xfull[s]), 1);
      mbar_init(smem_u32(&xempty[s]), 4);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&afull[b]), 4);
      mbar_init(smem_u32(&afree[b]), 1);
      mbar_init(smem_u32(&dfull[b]), 1);
      mbar_init(smem_u32(&dfree[b]), 4);
    }
    mbar_init(smem_u32(drain), 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc(tslot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == kProducerWarp) {
    // ---------------- producer: one thread streams this CTA's items ----------
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const int c0 = i0 % a.chunks;
      auto chunk_of = [&](int k) {   // chunk of local item k, without 64-bit division
        int c = c0 + k % a.chunks;
        return c >= a.chunks ? c - a.chunks : c;
      };
      auto issue_w = [&](int k) {
        const int s = k % SW;
        if (cta == 0 && k == a.fault_item) return;   // injected failure: this slot never fills
        mbar_arrive_expect_tx(smem_u32(&wfull[s]), QB);
        bulk_g2s(smem_u32(wring + s * QB), a.W + (size_t)(i0 + k) * QLayout<QT>::kItemBytes, QB,
                 smem_u32(&wfull[s]), pol);
      };
      auto issue_scales = [&](int k) {
        const int s = k % SX;
        mbar_arrive_expect_tx(smem_u32(&xfull[s]), QLayout<QT>::kScaleBytes + NT * kQChunkBytes);
        bulk_g2s(smem_u32(xring + s * XS), a.W + (size_t)(i0 + k) * QLayout<QT>::kItemBytes + QB,
                 QLayout<QT>::kScaleBytes, smem_u32(&xfull[s]), pol);
      };
      auto issue_x = [&](int k) {
        const int s = k % SX, c = chunk_of(k);
        for (int t = 0; t < NT; ++t)
          bulk_g2s_plain(smem_u32(xring + s * XS + QLayout<QT>::kScaleBytes + t * kQChunkBytes),
                         a.qx + (size_t)t * a.qx_stride + (size_t)c * kQChunkBytes, kQChunkBytes,
                         smem_u32(&xfull[s]));
      };
      // weights never depend on earlier kernels: the first rings are requested
      // before griddepcontrol.wait; the x columns (written by the previous
      // kernel) once the dependency is resolved
      int kw = 0, kx = 0;
      for (; kw < n && kw < SW; ++kw) issue_w(kw);
      for (int k = 0; k < n && k < SX; ++k) issue_scales(k);
      pdl_wait();
      for (; kx < n && kx < SX; ++kx) issue_x(kx);
      bool ok = true;
      for (uint32_t spins = 0; ok && (kw < n || kx < n);) {
        bool did = false;
        if (kw < n && mbar_test(smem_u32(&wempty[kw % SW]), ((kw / SW) - 1) & 1u)) {
          issue_w(kw++);
          did = true;
        }
        if (kx < n && mbar_test(smem_u32(&xempty[kx % SX]), ((kx / SX) - 1) & 1u)) {
          issue_scales(kx);
          issue_x(kx++);
          did = true;
        }
        if (did) {
          spins = 0;
        } else if (++spins > wait_limit(a.wait_limit)) {
          atomicOr(a.err, ERR_WAIT_TIMEOUT);
          ok = false;
        } else {
          __nanosleep(32);   // both rings full: poll lightly
        }
      }
      if (ok && a.next_W && cta < a.next_workers) {
        // every own item is on its way: warm L2 with the next projection's
        // first items of this CTA index while the consumers finish
        const StreamK skn(a.next_items, a.next_workers);
        const int j0 = skn.begin(cta), nj = min(SW, skn.begin(cta + 1) - j0);
        for (int k = 0; k < nj; ++k) bulk_prefetch_l2(a.next_W + (size_t)(j0 + k) * QLayout<QT>::kItemBytes,
                                                      QLayout<QT>::kItemBytes);
      }
      if (!ok) drain_inflight_copies();   // error path
    }
    return;   // the producer takes no part in the tensor-memory teardown
  }

  bool timed_out = false;
  if (warp == kMmaWarp) {
    // ---------------- MMA issuer: one thread ---------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(QT == kQ8_0, kTileRows, C::kN);
      uint32_t gc = 0;
      for (int k = 0; k < n && !timed_out; ++k) {
        const int ab = k & 1, sx = k % SX;
        if (!mbar_wait(smem_u32(&afull[ab]), (uint32_t)(k >> 1) & 1u, a.err, a.wait_limit) ||
            !mbar_wait(smem_u32(&xfull[sx]), (uint32_t)(k / SX) & 1u, a.err, a.wait_limit)) {
          timed_out = true;
          break;
        }
        tc_fence_after();
        const uint32_t xs = smem_u32(xring + sx * XS + QLayout<QT>::kScaleBytes);
        for (int g = 0; g < C::kNG; ++g, ++gc) {
          const int db = gc & 1;
          if (gc >= 2 && !mbar_wait(smem_u32(&dfree[db]), ((gc >> 1) - 1) & 1u, a.err, a.wait_limit)) {
            timed_out = true;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int j = 0; j < C::kGB; ++j) {
            const int b = g * C::kGB + j;
            const uint64_t desc = smem_desc_kmajor(xs + b * kQBlockBytes, 128, kQChunkBytes);
            mma_i8_ts(tmem + C::kDOff + db * C::kDCols + j * C::kN, tmem + ab * C::kACols + 8 * b, desc, idesc,
                      false);
          }
          tc_commit(&dfull[db]);
        }
        if (!timed_out) tc_commit(&afree[ab]);
      }
      // every MMA this thread issued has completed before tensor memory goes
      tc_commit(drain);
      if (!mbar_wait(smem_u32(drain), 0, a.err, a.wait_limit)) timed_out = true;
    }
    __syncwarp();
  } else if (warp < kUpdateWarp0) {
    // ---------------- unpack: thread = row, A operand into tensor memory -----
    const int quarter = warp & 3, r = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    for (int k = 0; k < n; ++k) {
      const int ab = k & 1, sw = k % SW;
      if (!mbar_wait(smem_u32(&wfull[sw]), (uint32_t)(k / SW) & 1u, a.err, a.wait_limit) ||
          (k >= 2 && !mbar_wait(smem_u32(&afree[ab]), ((k >> 1) - 1) & 1u, a.err, a.wait_limit))) {
        timed_out = true;
        break;
      }
      tc_fence_after();
      const uint8_t* q = wring + sw * QB;
      const uint32_t ta = tmem + lane_base + ab * C::kACols;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        uint32_t av[8];
        if constexpr (QT == kQ4_0) {
          q4_unpack(*reinterpret_cast<const uint4*>(q + q4_off(b, r)), av);
        } else {
          const uint4 w0 = *reinterpret_cast<const uint4*>(q + q8_off(b, 0, r));
          const uint4 w1 = *reinterpret_cast<const uint4*>(q + q8_off(b, 1, r));
          av[0] = w0.x; av[1] = w0.y; av[2] = w0.z; av[3] = w0.w;
          av[4] = w1.x; av[5] = w1.y; av[6] = w1.z; av[7] = w1.w;
        }
        tmem_st8(ta + 8 * b, av);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&afull[ab]));
        mbar_arrive(smem_u32(&wempty[sw]));
      }
    }
  } else {
    // ---------------- update: thread = row, f32 block updates, tile finish ---
    const int quarter = warp & 3, r = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    pdl_wait();   // ss_in, the residual stream and the scratch come from earlier kernels
    for (int t = quarter; t < NT; t += 4) {
      const float rs = a.ss_in ? rstd_warp(a.ss_in + (size_t)t * a.ss_stride, a.ss_tiles, a.inv_dim, a.eps, lane) : 1.f;
      if (lane == 0) rstd[t] = rs;
    }
    named_sync(kBarUpdate, 128);
    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0.f;
    uint32_t gc = 0;
    int tile = i0 / a.chunks;
    for (int k = 0; k < n; ++k) {
      const int item = i0 + k, sx = k % SX;
      if (item / a.chunks != tile) {
        gemv_finish_tile<EPI, NT>(a, cta, sk, i0, i1, tile, acc, rstd, ex, flag, quarter, lane);
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = 0.f;
        tile = item / a.chunks;
      }
      const uint8_t* xsl = xring + sx * XS;
      uint4 sc4 = make_uint4(0, 0, 0, 0);
      for (int g = 0; g < C::kNG; ++g, ++gc) {
        const int db = gc & 1;
        // the four warps share named barriers in the tile finish, so they
        // decide together: all go on, or all stop
        // (the first group also waits for the x slot itself: its scales and
        // block metadata are read here, not only by the MMA)
        const bool ok = mbar_wait(smem_u32(&dfull[db]), (gc >> 1) & 1u, a.err, a.wait_limit) &&
                        (g > 0 || mbar_wait(smem_u32(&xfull[sx]), (uint32_t)(k / SX) & 1u, a.err, a.wait_limit));
        if (!bar_and(kBarUpdate, 128, ok)) {
          timed_out = true;
          break;
        }
        tc_fence_after();
        if (g == 0) sc4 = *reinterpret_cast<const uint4*>(xsl + r * 16);   // the row's 8 block scales
        int dv[C::kGB][NT][4];
#pragma unroll
        for (int j = 0; j < C::kGB; ++j)
#pragma unroll
          for (int t = 0; t < NT; ++t)
            tmem_ld4(tmem + lane_base + C::kDOff + db * C::kDCols + j * C::kN + t * 8, dv[j][t]);
        tmem_ld_wait();
        const uint32_t scw[4] = {sc4.x, sc4.y, sc4.z, sc4.w};
#pragma unroll
        for (int j = 0; j < C::kGB; ++j) {
          const int b = g * C::kGB + j;
          const uint32_t w = scw[b >> 1];
          const float d = __half2float(__ushort_as_half(static_cast<unsigned short>((b & 1) ? (w >> 16) : (w & 0xFFFFu))));
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const int4 m = *reinterpret_cast<const int4*>(xsl + QLayout<QT>::kScaleBytes + t * kQChunkBytes +
                                                          b * kQBlockBytes + kQMetaOff);
            acc[t] = block_update<QT>(acc[t], d, __int_as_float(m.x), dv[j][t][0], dv[j][t][1], dv[j][t][2], m.y, m.z);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&dfree[db]));
      }
      if (timed_out) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&xempty[sx]));
    }
    if (!timed_out) gemv_finish_tile<EPI, NT>(a, cta, sk, i0, i1, tile, acc, rstd, ex, flag, quarter, lane);
  }
  // ---------------- teardown: tensor memory back, after every MMA and load --
  tc_fence_before();
  named_sync(kBarTmem, kGemvCtaThreads - 32);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
  if (timed_out && lane == 0) drain_inflight_copies();   // error path
}

}  // namespace qhl
