// Fused dequant-GEMV / skinny GEMM over packed Q4_0 / Q8_0 weights.
//
// y[t][r] = sum_c x[t][c] * W[r][c] for n_tok = NT tokens (1..16), the
// projection every layer of the stage streams: one decoded token streams the
// whole weight set a single time (SwarmLLM README, paragraph after the peer
// diagram).  Decode is
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
//    byte dot products (dp4a) against the 4-bit (or 8-bit) quants -- from 4
//    tokens up by integer tensor-core mma instead, with the same exact sums --
//    and one FMA per block adds d * s * sum to the row's f32 accumulator.
//  * A tenth warp finishes tiles (sums the consumer warps' partials, stream-K
//    fix-up, epilogue) while the consumers stream on; once its own items are
//    issued the producer warms L2 with the pass's next projection.
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
  // The pass's next projection (null if none): this kernel's producers warm L2
  // with the first items the next kernel's CTA of the same index will stream.
  const uint8_t* next_W;
  int next_items, next_workers;
};

constexpr int kConsumerWarps = 8;
// Stream-K workers per SM: the grid is kCtasPerSm * SMs for every token count
// (the split, and hence the summation order, must not depend on NT).
constexpr int kCtasPerSm = 2;

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

// ---------------------------------------------------------------------------
// Integer tensor-core path (n_tok >= kMmaTok): the same exact int32 block sums
// as the dp4a path, formed by mma.sync m16n8k32 (8-bit A = weights, B = one
// activation byte plane, columns = tokens), so both paths give bit-identical
// results and a 16-token verify still equals 16 single-token passes.  Warp w
// still owns block w of each item; its 64 rows are 4 m-tiles of 16.  The
// k order inside a block is GGUF's own: byte j of a Q4_0 row holds elements j
// (low nibble) and j + 16 (high nibble), which is exactly the split of the
// A fragment's k range into [4c, 4c + 4) and [16 + 4c, 16 + 4c + 4).
constexpr int kMmaTok = 4;

template <bool AS, bool BS>
QHL_DEV void mma_i8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
#define QHL_MMA_I8(AT, BT)                                                                         \
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32." AT "." BT ".s32 {%0, %1, %2, %3}, "        \
               "{%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"                                 \
               : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])                                    \
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0))
  if constexpr (!AS && BS) QHL_MMA_I8("u8", "s8");
  else if constexpr (!AS && !BS) QHL_MMA_I8("u8", "u8");
  else if constexpr (AS && BS) QHL_MMA_I8("s8", "s8");
  else QHL_MMA_I8("s8", "u8");
#undef QHL_MMA_I8
}

// Tokens per thread in the C fragment (columns 2c, 2c + 1 of every n-tile).
template <int NT>
struct MmaShape {
  static constexpr int kNTiles = (NT + 7) / 8;
  static constexpr int kTok = 2 * kNTiles;
};

// Row of accumulator m (m-tile m / 2, half m % 2) for lane group g.
QHL_DEV int mma_row(int m, int g) { return 16 * (m >> 1) + 8 * (m & 1) + g; }

// One block (warp `warp`) of one item for all NT tokens; acc[m][j]: row
// mma_row(m, g), token 8 * (j / 2) + 2c + (j % 2).
template <int QT, int NT>
QHL_DEV void compute_item_mma(const uint8_t* st, const uint8_t* xs, int warp, int lane,
                              float (&acc)[8][MmaShape<NT>::kTok]) {
  const int g = lane >> 2, c = lane & 3;
  // A fragments of the 4 m-tiles: rows 16mt + g and 16mt + g + 8
  uint32_t a[4][4];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = 16 * mt + 8 * h + g;
      if constexpr (QT == kQ4_0) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(st + ((warp * 2 + (r >> 5)) * 32 + (r & 31)) * 16 + 4 * c);
        a[mt][h] = w & 0x0F0F0F0Fu;                // elements 4c .. 4c + 3
        a[mt][2 + h] = (w >> 4) & 0x0F0F0F0Fu;     // elements 16 + 4c .. 16 + 4c + 3
      } else {
        const uint8_t* base = st + (warp * 4) * 32 * 16;
        a[mt][h] = *reinterpret_cast<const uint32_t*>(base + ((0 * 2 + (r >> 5)) * 32 + (r & 31)) * 16 + 4 * c);
        a[mt][2 + h] = *reinterpret_cast<const uint32_t*>(base + ((1 * 2 + (r >> 5)) * 32 + (r & 31)) * 16 + 4 * c);
      }
    }
  }
  // row scales: word (g + 8q) holds rows g + 8q (low half) and g + 8q + 32 (high half)
  float dsc[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const int r = mma_row(m, g);
    const uint32_t w = *reinterpret_cast<const uint32_t*>(st + QLayout<QT>::kQuantBytes + (warp * 32 + (r & 31)) * 4);
    dsc[m] = __half2float(__ushort_as_half(static_cast<unsigned short>((r >> 5) ? (w >> 16) : (w & 0xFFFFu))));
  }
#pragma unroll
  for (int nt = 0; nt < MmaShape<NT>::kNTiles; ++nt) {
    // B fragments: column g = token 8nt + g, k = 4c .. 4c + 3 and 16 + 4c ..
    const int tb = 8 * nt + g;
    uint32_t b[3][2];
#pragma unroll
    for (int p = 0; p < 3; ++p) {
      if (tb < NT) {
        const uint8_t* xp = xs + tb * kQChunkBytes + p * 256 + warp * 32;
        b[p][0] = *reinterpret_cast<const uint32_t*>(xp + 4 * c);
        b[p][1] = *reinterpret_cast<const uint32_t*>(xp + 16 + 4 * c);
      } else {
        b[p][0] = 0u;
        b[p][1] = 0u;
      }
    }
    // block scales of this thread's two C-fragment tokens
    float s[2];
    int shi[2], sml[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = 8 * nt + 2 * c + e;
      const uint8_t* xt = xs + (t < NT ? t : 0) * kQChunkBytes;
      s[e] = reinterpret_cast<const float*>(xt + 768)[warp];
      shi[e] = reinterpret_cast<const int*>(xt + 800)[warp];
      sml[e] = reinterpret_cast<const int*>(xt + 832)[warp];
    }
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      int dh[4], dm[4], dl[4];
      mma_i8<QT == kQ8_0, true>(dh, a[mt], b[0][0], b[0][1]);    // hi plane: signed
      mma_i8<QT == kQ8_0, false>(dm, a[mt], b[1][0], b[1][1]);   // mid plane: unsigned
      mma_i8<QT == kQ8_0, false>(dl, a[mt], b[2][0], b[2][1]);   // lo plane: unsigned
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int t = 8 * nt + 2 * c + e;
          if (t < NT) {
            const int m = 2 * mt + h, j = 2 * nt + e, q = 2 * h + e;
            if constexpr (QT == kQ4_0)
              acc[m][j] = block_update(dsc[m], s[e], dh[q] - 8 * shi[e], dm[q] * 256 + dl[q] - 8 * sml[e], acc[m][j]);
            else
              acc[m][j] = block_update(dsc[m], s[e], dh[q], dm[q] * 256 + dl[q], acc[m][j]);
          }
        }
    }
  }
}

// ---------------------------------------------------------------------------
// Warp roles of a GEMV CTA: warps 0..7 consume items, warp 8 produces (bulk
// copies into the ring), warp 9 finishes tiles.  The consumers hand each
// finished tile's per-warp sums to the epilogue warp through a small ring of
// reduction buffers (mbarriers "tile full" / "tile free") and go straight on
// with the next item; the epilogue warp sums the eight warps' partials, runs
// the stream-K fix-up and the fused epilogue off the item loop's path.
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kEpilogueWarp = kConsumerWarps + 1;
constexpr int kGemvCtaThreads = (kConsumerWarps + 2) * 32;

// Reduction buffers between consumers and the epilogue warp.
template <int NT>
struct TileRing {
  static constexpr int kBufs = NT <= 4 ? 2 : 1;
  static constexpr int kBufFloats = kConsumerWarps * NT * 64;   // [8][NT][64]
  static constexpr int kBytes = kBufs * kBufFloats * 4;
};

// Hand-off state shared by the consumers and the epilogue warp of one CTA.
struct TileSync {
  float* red;          // [kBufs][8][NT][64]
  uint64_t* full;      // [kBufs], 256 arrivals (every consumer thread)
  uint64_t* free_;     // [kBufs], 32 arrivals (every epilogue lane)
};

// Inputs of a tile's epilogue that do not depend on the tile's sums, loaded
// before the sums are ready: the residual stream h (written by an earlier
// step) and the next RMSNorm weight, for the lanes' elements.
template <int NT>
struct EpiInputs {
  float h[NT * 2];     // element i * 32 + lane of [NT][64]
  float gamma[2];      // rows lane and 32 + lane
};

template <int EPI, int NT>
QHL_DEV void gemv_prefetch(const GemvArgs& a, int tile, int lane, EpiInputs<NT>& in) {
  if constexpr (EPI == EPI_RESID) {
#pragma unroll
    for (int i = 0; i < NT * 2; ++i) {
      const int idx = i * 32 + lane, t = idx >> 6, gr = tile * 64 + (idx & 63);
      in.h[i] = gr < a.out_valid ? ld_cg_once(a.y + (size_t)t * a.y_stride + gr) : 0.f;   // h: written by other CTAs
    }
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int gr = tile * 64 + b * 32 + lane;
      in.gamma[b] = a.qout && gr < a.out_valid ? __ldg(a.gamma_next + gr) : 0.f;
    }
  }
}

// Epilogue of one finished tile by the 32 lanes of the epilogue warp;
// vals = [NT][64] final sums in shared memory, rstd = [NT].
template <int EPI, int NT>
QHL_DEV void gemv_epilogue(const GemvArgs& a, int tile, float* vals, const float* rstd, int lane,
                           const EpiInputs<NT>& in) {
  if constexpr (EPI == EPI_STORE) {
#pragma unroll
    for (int i = 0; i < NT * 2; ++i) {
      const int idx = i * 32 + lane, t = idx >> 6, gr = tile * 64 + (idx & 63);
      if (gr < a.out_valid) a.y[(size_t)t * a.y_stride + gr] = __fmul_rn(vals[idx], rstd[t]);
    }
  } else if constexpr (EPI == EPI_SWIGLU) {
    // tile rows 0..31 are gate rows of features tile*32.., rows 32..63 the matching up rows
#pragma unroll 1
    for (int t = 0; t < NT; ++t) {
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
#pragma unroll
    for (int i = 0; i < NT * 2; ++i) {
      const int idx = i * 32 + lane, t = idx >> 6, gr = tile * 64 + (idx & 63);
      float hn = 0.f;
      if (gr < a.out_valid) {
        hn = __fadd_rn(in.h[i], vals[idx]);
        a.y[(size_t)t * a.y_stride + gr] = hn;
      }
      vals[idx] = hn;
    }
    __syncwarp();
    if (a.qout) {
#pragma unroll 1
      for (int p = 0; p < NT * 2; ++p) {
        const int t = p >> 1, b = p & 1, gr = tile * 64 + b * 32 + lane;
        const float z = gr < a.out_valid ? __fmul_rn(vals[t * 64 + b * 32 + lane], b ? in.gamma[1] : in.gamma[0]) : 0.f;
        qact_store_block(z, a.qout + (size_t)t * a.qout_stride, tile * 2 + b, lane);
      }
    }
    if (a.ss_out && lane < NT) a.ss_out[(size_t)lane * a.ss_out_stride + tile] = sumsq64(vals + lane * 64);
    __syncwarp();
  }
}

// Stream-K tile counter: add 1 with release (this CTA's partial, published
// by every lane before the warp barrier, becomes visible with it) and acquire
// (the last contributor then sees every other partial).
QHL_DEV int counter_add_acq_rel(int* p) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
  return old;
}

// Consumer side of one GEMV for CTA `cta` (the 256 threads of warps 0..7):
// takes this CTA's stream-K items, in order, from the shared-memory ring
// (`slot` / `phase` carry the ring position across calls) and hands every
// tile's per-warp sums to the epilogue warp (`tc` counts hand-offs across
// calls).
template <int QT, int NT, int S>
QHL_DEV void gemv_consume(const GemvArgs& a, int cta, uint8_t* stages, uint64_t* bars, const TileSync& ts, int& slot,
                          uint32_t& phase, uint32_t& tc, bool& timed_out) {
  constexpr int IB = QLayout<QT>::kItemBytes;
  constexpr int SB = IB + NT * kQChunkBytes;
  constexpr int RB = TileRing<NT>::kBufs;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (cta >= a.workers) return;
  const StreamK sk(a.tiles * a.chunks, a.workers);
  const int i0 = sk.begin(cta), n_local = sk.begin(cta + 1) - i0;
  if (n_local == 0) return;

  constexpr bool kMma = NT >= kMmaTok;
  constexpr int kAccA = kMma ? 1 : NT;                        // dp4a: rows lane, lane + 32
  constexpr int kAccT = kMma ? MmaShape<NT>::kTok : 1;        // mma: C-fragment rows and tokens
  float r0[kAccA], r1[kAccA];
  float acc[kMma ? 8 : 1][kAccT];
#pragma unroll
  for (int t = 0; t < kAccA; ++t) { r0[t] = 0.f; r1[t] = 0.f; }
#pragma unroll
  for (int m = 0; m < (kMma ? 8 : 1); ++m)
#pragma unroll
    for (int j = 0; j < kAccT; ++j) acc[m][j] = 0.f;
  auto handoff = [&]() {
    const int buf = (int)(tc % RB);
    const uint32_t use = tc / RB;
    if (use > 0 && !timed_out && !mbar_wait(smem_u32(&ts.free_[buf]), (use - 1) & 1u, a.err)) timed_out = true;
    float* red = ts.red + buf * TileRing<NT>::kBufFloats;
    if constexpr (kMma) {
      const int g = lane >> 2, c = lane & 3;
#pragma unroll
      for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int j = 0; j < kAccT; ++j) {
          const int t = 8 * (j >> 1) + 2 * c + (j & 1);
          if (t < NT) red[(warp * NT + t) * 64 + mma_row(m, g)] = acc[m][j];
          acc[m][j] = 0.f;
        }
    } else {
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        red[(warp * NT + t) * 64 + lane] = r0[t];
        red[(warp * NT + t) * 64 + 32 + lane] = r1[t];
        r0[t] = 0.f;
        r1[t] = 0.f;
      }
    }
    mbar_arrive(smem_u32(&ts.full[buf]));
    ++tc;
  };

  int chunk = i0 % a.chunks;
  for (int k = 0; k < n_local; ++k) {
    if (chunk == a.chunks) {
      handoff();
      chunk = 0;
    }
    // after one timed-out wait the rest of the call runs without waiting (the
    // error is recorded; results are garbage, but the kernel ends promptly)
    if (!timed_out && !mbar_wait(smem_u32(&bars[slot]), phase, a.err)) timed_out = true;
    const uint8_t* st = stages + slot * SB;
    if constexpr (kMma) {
      compute_item_mma<QT, NT>(st, st + IB, warp, lane, acc);
    } else {
      ItemRegs<QT> regs;
      load_item<QT>(st, warp, lane, regs);
      compute_item<QT, NT>(regs, st + IB, warp, r0, r1);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars[S + slot]));   // stage free for the producer
    ++chunk;
    if (++slot == S) {
      slot = 0;
      phase ^= 1u;
    }
  }
  handoff();
}

// Epilogue-warp side of one GEMV: for every tile this CTA touches, in order,
// sum the eight warps' partials (warps 0..7 in order), then either finish the
// tile (all its chunks were this CTA's) or publish the partial and, if this
// CTA is the last contributor to arrive, combine every contributor's partial
// in CTA order and finish it.  `fin` = [NT][64], `rstd` = [NT] (computed
// here, from the previous step's per-tile sums of squares).
template <int EPI, int NT>
QHL_DEV void gemv_finish(const GemvArgs& a, int cta, const TileSync& ts, float* fin, float* rstd, uint32_t& tc,
                         bool& timed_out) {
  constexpr int RB = TileRing<NT>::kBufs;
  const int lane = threadIdx.x & 31;
  if (cta >= a.workers) return;
  const StreamK sk(a.tiles * a.chunks, a.workers);
  const int i0 = sk.begin(cta), i1 = sk.begin(cta + 1);
  if (i1 == i0) return;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const float r = a.ss_in ? rstd_warp(a.ss_in + (size_t)t * a.ss_stride, a.ss_tiles, a.inv_dim, a.eps, lane) : 1.f;
    if (lane == 0) rstd[t] = r;
  }
  __syncwarp();
  const int first_tile = i0 / a.chunks, last_tile = (i1 - 1) / a.chunks;
  for (int tl = first_tile; tl <= last_tile; ++tl) {
    EpiInputs<NT> in;
    gemv_prefetch<EPI, NT>(a, tl, lane, in);
    const int buf = (int)(tc % RB);
    const uint32_t use = tc / RB;
    if (!timed_out && !mbar_wait(smem_u32(&ts.full[buf]), use & 1u, a.err)) timed_out = true;
    const float* red = ts.red + buf * TileRing<NT>::kBufFloats;
#pragma unroll
    for (int i = 0; i < NT * 2; ++i) {
      const int idx = i * 32 + lane;
      float v = red[idx];
#pragma unroll
      for (int w = 1; w < kConsumerWarps; ++w) v = __fadd_rn(v, red[w * NT * 64 + idx]);
      fin[idx] = v;
    }
    __syncwarp();
    mbar_arrive(smem_u32(&ts.free_[buf]));
    ++tc;
    const int t_lo = tl * a.chunks, t_hi = t_lo + a.chunks;
    if (t_lo >= i0 && t_hi <= i1) {
      gemv_epilogue<EPI, NT>(a, tl, fin, rstd, lane, in);
      continue;
    }
    // stream-K: publish this CTA's partial; the last contributor to arrive
    // combines every contributor's partial in CTA order and finishes the tile.
    // Partials move as float2: lane owns elements 2q, 2q + 1, q = j * 32 + lane.
    float2* mine = reinterpret_cast<float2*>(a.partials + (size_t)(2 * cta + (tl == first_tile ? 0 : 1)) * NT * 64);
    const float2* fin2 = reinterpret_cast<const float2*>(fin);
#pragma unroll
    for (int j = 0; j < NT; ++j) mine[j * 32 + lane] = fin2[j * 32 + lane];
    __syncwarp();
    const int cf = sk.owner(t_lo), cl = sk.owner(t_hi - 1);
    int last = 0;
    if (lane == 0) last = counter_add_acq_rel(&a.counters[tl]) == cl - cf ? 1 : 0;
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) continue;
    // Tile tl is the first tile of every contributor after cf, and of cf
    // exactly when cf's range starts at the tile's first item.  Up to 4
    // float2 loads per lane in flight.
    constexpr int CB = NT >= 4 ? 1 : 4 / NT;
    const int cf_slot = sk.begin(cf) == t_lo ? 0 : 1;
    float2 acc[NT];
    for (int c0 = cf; c0 <= cl; c0 += CB) {
      float2 pv[CB][NT];
#pragma unroll
      for (int k = 0; k < CB; ++k) {
        const int c = c0 + k;
        if (c <= cl) {
          const float2* pc =
              reinterpret_cast<const float2*>(a.partials + (size_t)(2 * c + (c == cf ? cf_slot : 0)) * NT * 64);
#pragma unroll
          for (int j = 0; j < NT; ++j) pv[k][j] = ld_cg_once(pc + j * 32 + lane);
        }
      }
#pragma unroll
      for (int k = 0; k < CB; ++k)
        if (c0 + k <= cl) {
#pragma unroll
          for (int j = 0; j < NT; ++j)
            acc[j] = (c0 + k == cf) ? pv[k][j]
                                    : make_float2(__fadd_rn(acc[j].x, pv[k][j].x), __fadd_rn(acc[j].y, pv[k][j].y));
        }
    }
    float2* fout = reinterpret_cast<float2*>(fin);
#pragma unroll
    for (int j = 0; j < NT; ++j) fout[j * 32 + lane] = acc[j];
    __syncwarp();
    gemv_epilogue<EPI, NT>(a, tl, fin, rstd, lane, in);
    if (lane == 0) a.counters[tl] = 0;
  }
}

template <int QT, int NT>
struct GemvCfg {
  static constexpr int kStageBytes = QLayout<QT>::kItemBytes + NT * kQChunkBytes;
  // two CTAs per SM up to 4 tokens, one beyond
  static constexpr int kBudget = NT <= 4 ? 112 * 1024 : 200 * 1024;
  static constexpr int kFixed = TileRing<NT>::kBytes + NT * 64 * 4 + 16 * 4 + 64;
  static constexpr int kRaw = (kBudget - kFixed) / (kStageBytes + 16);
  static constexpr int kStages = kRaw < 3 ? 3 : (kRaw > 16 ? 16 : kRaw);
  static constexpr int kMinBlocks = NT <= 4 ? 2 : 1;
  // shared-memory layout
  static constexpr int kRedOff = kStages * kStageBytes;
  static constexpr int kFinOff = kRedOff + TileRing<NT>::kBytes;
  static constexpr int kRstdOff = kFinOff + NT * 64 * 4;
  static constexpr int kBarOff = kRstdOff + 16 * 4;                        // 8-byte aligned
  static constexpr int kSmem = kBarOff + (2 * kStages + 2 * TileRing<NT>::kBufs) * 8;
};

template <int QT, int NT>
constexpr int gemv_smem_bytes() {
  return GemvCfg<QT, NT>::kSmem;
}

template <int QT, int NT, int EPI>
__global__ void __launch_bounds__(kGemvCtaThreads, GemvCfg<QT, NT>::kMinBlocks) qgemv_kernel(const GemvArgs a) {
  using C = GemvCfg<QT, NT>;
  constexpr int S = C::kStages;
  constexpr int IB = QLayout<QT>::kItemBytes;
  constexpr int SB = C::kStageBytes;
  constexpr int RB = TileRing<NT>::kBufs;
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* stages = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);   // full[S], empty[S], tile full[RB], tile free[RB]
  const TileSync ts{reinterpret_cast<float*>(smem + C::kRedOff), bars + 2 * S, bars + 2 * S + RB};
  float* fin = reinterpret_cast<float*>(smem + C::kFinOff);
  float* rstd = reinterpret_cast<float*>(smem + C::kRstdOff);

  const int cta = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) pdl_launch();
  if (cta >= a.workers) return;
  const StreamK sk(a.tiles * a.chunks, a.workers);
  const int i0 = sk.begin(cta), n_local = sk.begin(cta + 1) - i0;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&bars[s]), 1);
      mbar_init(smem_u32(&bars[S + s]), kConsumerWarps);
    }
    for (int b = 0; b < RB; ++b) {
      mbar_init(smem_u32(&ts.full[b]), kConsumerWarps * 32);
      mbar_init(smem_u32(&ts.free_[b]), 32);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kProducerWarp) {
    // ---------------- producer: stream this CTA's items into the ring ----------
    // Weights never depend on earlier kernels: the first S items' weights are
    // requested before griddepcontrol.wait.  Their x chunks (written by the
    // previous kernel) follow once the dependency is resolved.
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const int pre = n_local < S ? n_local : S;
      const int c0 = i0 % a.chunks;
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
        bulk_g2s(smem_u32(stages + k * SB), a.W + (size_t)(i0 + k) * IB, IB, full, pol);
      }
      pdl_wait();
      for (int k = 0; k < pre; ++k) issue_x(k, k);
      for (int k = pre; k < n_local; ++k) {
        const int s = k % S, round = k / S;
        if (!mbar_wait(smem_u32(&bars[S + s]), (round - 1) & 1, a.err)) {
          drain_inflight_copies();   // error path
          return;
        }
        const uint32_t full = smem_u32(&bars[s]);
        mbar_arrive_expect_tx(full, SB);
        bulk_g2s(smem_u32(stages + s * SB), a.W + (size_t)(i0 + k) * IB, IB, full, pol);
        issue_x(k, s);
      }
      // every own item is on its way: warm L2 with the next projection's first
      // items of this CTA index while the consumers finish (the next kernel's
      // copies of them then hit L2)
      if (a.next_W && cta < a.next_workers) {
        const StreamK skn(a.next_items, a.next_workers);
        const int j0 = skn.begin(cta), nj = min(S, skn.begin(cta + 1) - j0);
        for (int k = 0; k < nj; ++k) bulk_prefetch_l2(a.next_W + (size_t)(j0 + k) * IB, IB);
      }
    }
    return;
  }

  pdl_wait();   // ss_in, the residual stream and the scratch come from earlier kernels
  uint32_t tc = 0;
  bool timed_out = false;
  if (warp == kEpilogueWarp) {
    gemv_finish<EPI, NT>(a, cta, ts, fin, rstd, tc, timed_out);
  } else {
    int slot = 0;
    uint32_t phase = 0;
    gemv_consume<QT, NT, S>(a, cta, stages, bars, ts, slot, phase, tc, timed_out);
  }
  if (timed_out && lane == 0) drain_inflight_copies();   // error path
}

}  // namespace qhl
