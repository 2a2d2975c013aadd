// Split-K GQA decode attention with QK-norm, partial RoPE, f16 KV cache and a
// sigmoid output gate (ChatTorrent README, "What it can run", lists these three
// features of the hybrid's full-attention layers; Unstable Legion, "Splitting
// the workload": a stage holds the attention cache of its own layers only).
//
// Token t of a pass sits at absolute position pos + t and attends to cache rows
// 0 .. pos + t.  The context is cut into fixed chunks of 64 rows at absolute
// multiples of 64; one CTA handles one (chunk, KV head) for a group of up to
// four tokens and every query head of the KV head, so each K/V row is read
// from HBM once per token group.  A token's partial (max, sum, weighted V) over
// a chunk depends only on the token and the chunk, and the combine walks chunks
// 0 .. in order, so a batched pass gives the same bits as running the tokens
// one at a time.
//
// New rows: every CTA whose chunk holds a position p = pos + t that its tokens
// see normalises and rotates the token's k and rounds k and v to f16 itself
// (the same operations in every CTA, so the same bits), and uses the rounded
// values -- exactly what a later pass reads back.  Only the CTA of the token's
// own group writes the row to the cache, and no CTA reads a row of this pass
// from the cache, so the CTAs of one launch never depend on one another.
//
// The two contractions of a chunk, scores = q.k and out = p.v, run on the
// warp-level tensor-core MMA (m16n8k16, f16 operands, f32 accumulation).  K and
// V are f16 already; q and p are f32, and each is split into an f16 high part
// and an f16 remainder, two MMAs per step, which keeps about 22 bits of each
// (the products themselves are exact in f32).
#pragma once

#include "qact.cuh"

namespace qhl {

constexpr int kAttDim = 256;
constexpr int kRopeDims = 64;
constexpr int kAttChunk = 64;
constexpr int kAttMaxCtx = 1 << 18;   // largest cache a stage accepts (rows per KV head)
// Tokens one attention unit serves: a 16-token pass splits its tokens into
// groups of 4, so its (chunk, KV head, group) units spread over 4x the CTAs.
constexpr int kAttGroup = 4;

struct AttnArgs {
  const float* y;          // [NT][y_stride] in-projection output: q | gate | k | v
  int y_stride;
  int Hq, Hkv;
  uint16_t* K;             // f16 bits [Hkv][max_ctx][256]
  uint16_t* V;
  int max_ctx;
  const int* kv_len;       // device: position of token 0
  const float* gq;         // q-norm weight [256]
  const float* gk;         // k-norm weight [256]
  const float2* rope;      // [max_ctx][32] (cos, sin)
  float eps;
  float* pm;               // [NT][Hq][nchunk]: chunk max score
  float* pl;               // [NT][Hq][nchunk]: chunk sum of exp
  float* po;               // [NT][Hq][nchunk][256]: chunk sum of exp * v
  int nchunk;
  float* out;              // optional f32 gated output [NT][out_stride]
  int out_stride;
  uint8_t* qout;           // gated output in block fixed point (the out-projection's input)
  int qout_stride;
};

// Shared memory of one attention unit with jobs = tokens x query heads of the
// KV head, in MT = ceil(jobs / 16) row tiles of 16 jobs:
//   [0, MT * 16 KB): first the new K and V rows (16 x 512 B each), then the
//     queries' f16 high and low parts ([MT*16][256] each), then the score
//     partials of the two dimension halves ([2][MT*16][64] f32) followed by the
//     probabilities' high and low parts ([2][MT*16][72] f16);
//   [MT * 16 KB, + 8 KB): one 256-float vector per warp.
__host__ __device__ constexpr int attn_mtiles(int nt, int rep) { return (nt * rep + 15) / 16; }
__host__ __device__ constexpr int attn_smem_bytes(int nt, int rep) {
  return attn_mtiles(nt, rep) * 16384 + 8 * kAttDim * 4;
}
template <int NT>
constexpr int attn_smem_bytes(int rep) {
  return attn_smem_bytes(NT < kAttGroup ? NT : kAttGroup, rep);
}

// RMSNorm over one 256-wide head vector held as 8 values per lane (dims 8l..8l+7)
// followed by rotate-half RoPE on dims [0, 64) at position p; result in vec[256].
QHL_DEV void norm_rope(const float (&x)[8], const float* gamma, float eps, const float2* rope_row,
                       float* vec, int lane) {
  float ss = __fmul_rn(x[0], x[0]);
#pragma unroll
  for (int i = 1; i < 8; ++i) ss = __fmaf_rn(x[i], x[i], ss);
  ss = warp_sum(ss);
  const float r = __frcp_rn(__fsqrt_rn(__fadd_rn(__fmul_rn(ss, 1.f / kAttDim), eps)));
#pragma unroll
  for (int i = 0; i < 8; ++i) vec[8 * lane + i] = __fmul_rn(__fmul_rn(x[i], r), gamma[8 * lane + i]);
  __syncwarp();
  {
    const int i = lane;   // pair (i, i + 32), i < kRopeDims / 2
    const float2 cs = rope_row[i];
    const float x1 = vec[i], x2 = vec[i + kRopeDims / 2];
    vec[i] = __fsub_rn(__fmul_rn(x1, cs.x), __fmul_rn(x2, cs.y));
    vec[i + kRopeDims / 2] = __fadd_rn(__fmul_rn(x2, cs.x), __fmul_rn(x1, cs.y));
  }
  __syncwarp();
}

// 8 consecutive f32 through L2 (the data may have been written earlier in the
// same kernel by another CTA, so L1 must not serve it).
QHL_DEV void load8_cg(const float* p, float (&x)[8]) {
  const float4 a = __ldcg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldcg(reinterpret_cast<const float4*>(p) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// One m16n8k16 MMA, f16 operands, f32 accumulators: d += A(16x16) * B(16x8).
// Fragments (g = lane / 4, t = lane % 4): a0 = A[g][2t..2t+1],
// a1 = A[g+8][2t..], a2 = A[g][2t+8..], a3 = A[g+8][2t+8..];
// b0 = B[2t..2t+1][g], b1 = B[2t+8..2t+9][g]; d = {D[g][2t], D[g][2t+1],
// D[g+8][2t], D[g+8][2t+1]}.
QHL_DEV void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                           uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// f32 pair -> f16 high parts and f16 remainders, each packed low | high << 16.
QHL_DEV void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
  const __half l0 = __float2half_rn(__fsub_rn(x0, __half2float(h0)));
  const __half l1 = __float2half_rn(__fsub_rn(x1, __half2float(h1)));
  hi = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
  lo = (uint32_t)__half_as_ushort(l0) | ((uint32_t)__half_as_ushort(l1) << 16);
}

// The K and V fragments of one attention unit, held in registers (lane =
// 4g + t).  For the scores warp w takes keys 16 (w % 4) .. +15 and dimensions
// 128 (w / 4) .. +127: k[i] (k[4 + i]) holds the 8 dimensions
// 32 (4 (w / 4) + i) + 8t .. +7 of key 16 (w % 4) + g (+ 8).  For the weighted
// sum it takes dimensions 32w .. 32w + 31: v[(qq * 4 + j) * 4 + e] holds the
// dimension pair 16 (2w + qq) + 2g, +1 of key 16j + 2t + (e % 2) + 8 (e / 2).
struct AttnRegs {
  uint4 k[8];
  uint32_t v[32];
};

// Fill the fragments from cache rows of earlier passes (rows < pos) and zero
// the others; attn_compute then fills in this pass's rows that the unit's
// tokens see.  Needs nothing written by this pass, so a kernel issues it
// before waiting for the in-projection.
QHL_DEV void attn_load_old(const AttnArgs& a, int c, int g, int pos, int ctx_end, AttnRegs& R) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, gl = lane >> 2, tl = lane & 3;
  const int k0 = c * kAttChunk;
  const int n_old = min(kAttChunk, pos - k0);   // rows of earlier passes in the chunk (may be <= 0)
  const size_t head_base = (size_t)g * a.max_ctx;
  const int kq = warp & 3, dh = warp >> 2;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int key = 16 * kq + gl + 8 * r;
    const uint4* row = reinterpret_cast<const uint4*>(a.K + (head_base + k0 + key) * kAttDim);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      R.k[4 * r + i] = key < n_old ? ld_cg_once(row + 4 * (4 * dh + i) + tl) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int qq = 0; qq < 2; ++qq)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = 16 * j + 2 * tl + (e & 1) + 8 * (e >> 1);
        R.v[(qq * 4 + j) * 4 + e] =
            key < n_old ? ld_cg_once(reinterpret_cast<const uint32_t*>(a.V + (head_base + k0 + key) * kAttDim) +
                                     8 * (2 * warp + qq) + gl)
                        : 0u;
      }
  (void)ctx_end;   // the unit's last visible row + 1 (rows from pos on come later)
}

// Byte offset of the 8-byte unit u of query row r in a [rows][256] f16 plane:
// units are XOR-swizzled with (r & 1) | (r & 2) << 2 so that the 16 lanes of a
// half-warp reading B fragments hit 16 distinct bank pairs.
QHL_DEV int q_unit_off(int r, int u) { return r * 512 + ((u ^ ((r & 1) | ((r & 2) << 2))) << 3); }

// One attention unit: KV head g, context chunk c (rows 64c .. 64c+63), tokens
// t0 .. t0 + min(kAttGroup, NT - t0) - 1 and the group's query heads (jobs).
// Writes per (token, head, chunk) the max score, the sum of exp and the
// exp-weighted V sum.  All 256 threads of the CTA take part; `pos` is the
// position of token 0.  A token's results depend only on the token and the
// chunk, whatever its group and its row in the MMA tiles.  At most 7 query
// heads per KV head (stage_load refuses more): up to 28 jobs, two row tiles of
// 16 and four column tiles of 8.
template <int NT>
QHL_DEV void attn_compute(const AttnArgs& a, int c, int g, int pos, int t0, uint8_t* smem, AttnRegs& R) {
  const int rep = a.Hq / a.Hkv;
  const int ntk = min(kAttGroup, NT - t0);
  const int njobs = ntk * rep;
  const int MT = (njobs + 15) / 16, rows = 16 * MT;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gl = lane >> 2, tl = lane & 3;
  const int k0 = c * kAttChunk;
  const int ctx_end = pos + t0 + ntk;                          // rows the unit's tokens see
  const int nkeys = min(kAttChunk, ctx_end - k0);             // > 0 by the caller
  float* vec = reinterpret_cast<float*>(smem + MT * 16384) + warp * kAttDim;
  const int q_off = 0, k_off = 2 * a.Hq * kAttDim, v_off = k_off + a.Hkv * kAttDim;
  const size_t head_base = (size_t)g * a.max_ctx;

  // 1. this pass's rows in the chunk that the unit's tokens see: QK-norm +
  //    RoPE k, round k and v to f16, keep them in shared memory; the rows of
  //    the unit's own tokens also go to the cache
  const int pn0 = max(k0, pos), p_hi = min(k0 + kAttChunk, ctx_end);
  uint8_t* newk = smem;               // [16][256] f16
  uint8_t* newv = smem + 16 * 512;    // [16][256] f16
  for (int p = pn0 + warp; p < p_hi; p += 8) {
    const int t = p - pos;
    const float* yt = a.y + (size_t)t * a.y_stride;
    float x[8];
    load8_cg(yt + k_off + g * kAttDim + 8 * lane, x);
    norm_rope(x, a.gk, a.eps, a.rope + (size_t)p * (kRopeDims / 2), vec, lane);
    float vv[8];
    load8_cg(yt + v_off + g * kAttDim + 8 * lane, vv);
    uint16_t kh[8], vh[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      kh[i] = __half_as_ushort(__float2half_rn(vec[8 * lane + i]));
      vh[i] = __half_as_ushort(__float2half_rn(vv[i]));
    }
    const uint4 kr = make_uint4(kh[0] | (kh[1] << 16), kh[2] | (kh[3] << 16), kh[4] | (kh[5] << 16), kh[6] | (kh[7] << 16));
    const uint4 vr = make_uint4(vh[0] | (vh[1] << 16), vh[2] | (vh[3] << 16), vh[4] | (vh[5] << 16), vh[6] | (vh[7] << 16));
    reinterpret_cast<uint4*>(newk + (p - pn0) * 512)[lane] = kr;
    reinterpret_cast<uint4*>(newv + (p - pn0) * 512)[lane] = vr;
    if (p >= pos + t0) {
      reinterpret_cast<uint4*>(a.K + (head_base + p) * kAttDim)[lane] = kr;
      reinterpret_cast<uint4*>(a.V + (head_base + p) * kAttDim)[lane] = vr;
    }
    __syncwarp();
  }
  if (p_hi > pn0) {   // uniform over the CTA
    named_sync(kBarMix, 256);
    const int kq = warp & 3, dh = warp >> 2;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int p = k0 + 16 * kq + gl + 8 * r;
      if (p >= pn0 && p < p_hi)
#pragma unroll
        for (int i = 0; i < 4; ++i) R.k[4 * r + i] = reinterpret_cast<const uint4*>(newk + (p - pn0) * 512)[4 * (4 * dh + i) + tl];
    }
#pragma unroll
    for (int qq = 0; qq < 2; ++qq)
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int p = k0 + 16 * j + 2 * tl + (e & 1) + 8 * (e >> 1);
          if (p >= pn0 && p < p_hi)
            R.v[(qq * 4 + j) * 4 + e] = reinterpret_cast<const uint32_t*>(newv + (p - pn0) * 512)[8 * (2 * warp + qq) + gl];
        }
    named_sync(kBarMix, 256);   // the new rows' space is reused below
  }

  // 2. queries of every token that sees this chunk, normalised and rotated,
  //    as f16 high and low planes; rows of other tokens and padding are zero
  uint8_t* qhi = smem;
  uint8_t* qlo = smem + rows * 512;
  for (int job = warp; job < rows; job += 8) {
    const int tj = job / rep, j = job - tj * rep, t = t0 + tj;
    uint32_t h[4] = {0u, 0u, 0u, 0u}, l[4] = {0u, 0u, 0u, 0u};
    if (job < njobs && pos + t >= k0) {
      const float* yt = a.y + (size_t)t * a.y_stride;
      float x[8];
      load8_cg(yt + q_off + (g * rep + j) * kAttDim + 8 * lane, x);
      norm_rope(x, a.gq, a.eps, a.rope + (size_t)(pos + t) * (kRopeDims / 2), vec, lane);
#pragma unroll
      for (int i = 0; i < 4; ++i) split2(vec[8 * lane + 2 * i], vec[8 * lane + 2 * i + 1], h[i], l[i]);
    }
    // lane's dims 8 lane .. +7 = 8-byte units 2 lane, 2 lane + 1
    *reinterpret_cast<uint2*>(qhi + q_unit_off(job, 2 * lane)) = make_uint2(h[0], h[1]);
    *reinterpret_cast<uint2*>(qhi + q_unit_off(job, 2 * lane + 1)) = make_uint2(h[2], h[3]);
    *reinterpret_cast<uint2*>(qlo + q_unit_off(job, 2 * lane)) = make_uint2(l[0], l[1]);
    *reinterpret_cast<uint2*>(qlo + q_unit_off(job, 2 * lane + 1)) = make_uint2(l[2], l[3]);
  }
  named_sync(kBarMix, 256);

  // 3. score partials S^T[key][job] over the warp's 128 dimensions: A = K
  //    (keys 16 (w % 4) ..), B = q (jobs 8 nn ..); each 16-wide MMA step takes
  //    dimensions 32 s + 8t + 4h + {0, 1 | 2, 3} (s = 4 (w / 4) + i), the
  //    order in which a lane holds K; high part, then remainder
  const int kq = warp & 3, dh = warp >> 2;
  const int nnt = (njobs + 7) / 8;
  float sacc[4][4];
#pragma unroll
  for (int nn = 0; nn < 4; ++nn)
#pragma unroll
    for (int e = 0; e < 4; ++e) sacc[nn][e] = 0.f;
#pragma unroll
  for (int nn = 0; nn < 4; ++nn) {
    if (nn < nnt) {
      const int qr = 8 * nn + gl;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int s8 = 4 * dh + i;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t a0 = h ? R.k[i].z : R.k[i].x, a2 = h ? R.k[i].w : R.k[i].y;
          const uint32_t a1 = h ? R.k[4 + i].z : R.k[4 + i].x, a3 = h ? R.k[4 + i].w : R.k[4 + i].y;
          const int u = 8 * s8 + 2 * tl + h;
          const uint2 bh = *reinterpret_cast<const uint2*>(qhi + q_unit_off(qr, u));
          const uint2 bl = *reinterpret_cast<const uint2*>(qlo + q_unit_off(qr, u));
          mma_f16_16816(sacc[nn], a0, a1, a2, a3, bh.x, bh.y);
          mma_f16_16816(sacc[nn], a0, a1, a2, a3, bl.x, bl.y);
        }
      }
    }
  }
  named_sync(kBarMix, 256);   // every query read: the space takes the partials
  float* sc = reinterpret_cast<float*>(smem);   // [2][rows][64]
#pragma unroll
  for (int nn = 0; nn < 4; ++nn) {
    if (nn < nnt) {
      const int key = 16 * kq + gl, job = 8 * nn + 2 * tl;
      float* d = sc + ((size_t)dh * rows + job) * kAttChunk + key;
      d[0] = sacc[nn][0];
      d[kAttChunk] = sacc[nn][1];
      d[8] = sacc[nn][2];
      d[kAttChunk + 8] = sacc[nn][3];
    }
  }
  named_sync(kBarMix, 256);

  // 4. chunk softmax statistics, one warp per job: score = (half 0 + half 1) / 16;
  //    probabilities as f16 high and low planes [rows][72]
  uint16_t* phi = reinterpret_cast<uint16_t*>(smem + (size_t)2 * rows * kAttChunk * 4);
  uint16_t* plo = phi + rows * 72;
  for (int job = warp; job < rows; job += 8) {
    const int tj = job / rep, j = job - tj * rep, t = t0 + tj;
    const int nk = job < njobs ? min(kAttChunk, pos + t + 1 - k0) : 0;
    float e0 = 0.f, e1 = 0.f;
    if (nk > 0) {
      const bool v0 = lane < nk, v1 = lane + 32 < nk;
      const float* s0p = sc + (size_t)job * kAttChunk;
      const float* s1p = sc + ((size_t)rows + job) * kAttChunk;
      const float s0 = v0 ? __fmul_rn(__fadd_rn(s0p[lane], s1p[lane]), 1.f / 16.f) : -INFINITY;
      const float s1 = v1 ? __fmul_rn(__fadd_rn(s0p[lane + 32], s1p[lane + 32]), 1.f / 16.f) : -INFINITY;
      const float m = warp_max(fmaxf(s0, s1));
      e0 = v0 ? expf(__fsub_rn(s0, m)) : 0.f;
      e1 = v1 ? expf(__fsub_rn(s1, m)) : 0.f;
      const float l = warp_sum(__fadd_rn(e0, e1));
      if (lane == 0) {
        const size_t idx = ((size_t)t * a.Hq + g * rep + j) * a.nchunk + c;
        a.pm[idx] = m;
        a.pl[idx] = l;
      }
    }
    const __half h0 = __float2half_rn(e0), h1 = __float2half_rn(e1);
    phi[job * 72 + lane] = __half_as_ushort(h0);
    phi[job * 72 + lane + 32] = __half_as_ushort(h1);
    plo[job * 72 + lane] = __half_as_ushort(__float2half_rn(__fsub_rn(e0, __half2float(h0))));
    plo[job * 72 + lane + 32] = __half_as_ushort(__float2half_rn(__fsub_rn(e1, __half2float(h1))));
  }
  named_sync(kBarMix, 256);

  // 5. exp-weighted V: O[job][dim] over the chunk's 64 keys, A = p (jobs
  //    16 m ..), B = V (warp w: dims 32w .. +31 as an even-dimension and an
  //    odd-dimension tile per 16 dims); high part, then remainder
  float oacc[2][2][2][4];   // [m][qq][even / odd][4]
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int qq = 0; qq < 2; ++qq)
#pragma unroll
      for (int o = 0; o < 2; ++o)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[m][qq][o][e] = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      if (m < MT) {
        const uint16_t* rh0 = phi + (16 * m + gl) * 72 + 16 * j + 2 * tl;
        const uint16_t* rl0 = plo + (16 * m + gl) * 72 + 16 * j + 2 * tl;
        const uint32_t ah0 = *reinterpret_cast<const uint32_t*>(rh0);
        const uint32_t ah1 = *reinterpret_cast<const uint32_t*>(rh0 + 8 * 72);
        const uint32_t ah2 = *reinterpret_cast<const uint32_t*>(rh0 + 8);
        const uint32_t ah3 = *reinterpret_cast<const uint32_t*>(rh0 + 8 * 72 + 8);
        const uint32_t al0 = *reinterpret_cast<const uint32_t*>(rl0);
        const uint32_t al1 = *reinterpret_cast<const uint32_t*>(rl0 + 8 * 72);
        const uint32_t al2 = *reinterpret_cast<const uint32_t*>(rl0 + 8);
        const uint32_t al3 = *reinterpret_cast<const uint32_t*>(rl0 + 8 * 72 + 8);
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
          const uint32_t* x = R.v + (qq * 4 + j) * 4;
          const uint32_t be0 = __byte_perm(x[0], x[1], 0x5410), be1 = __byte_perm(x[2], x[3], 0x5410);
          const uint32_t bo0 = __byte_perm(x[0], x[1], 0x7632), bo1 = __byte_perm(x[2], x[3], 0x7632);
          mma_f16_16816(oacc[m][qq][0], ah0, ah1, ah2, ah3, be0, be1);
          mma_f16_16816(oacc[m][qq][0], al0, al1, al2, al3, be0, be1);
          mma_f16_16816(oacc[m][qq][1], ah0, ah1, ah2, ah3, bo0, bo1);
          mma_f16_16816(oacc[m][qq][1], al0, al1, al2, al3, bo0, bo1);
        }
      }
    }
  }
  // lane holds, per tile and 16 dims, dims 16 (2w + qq) + 4t .. +3 of jobs
  // 16m + g and 16m + g + 8
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    if (m < MT) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int job = 16 * m + gl + 8 * half;
        const int tj = job / rep, j = job - tj * rep, t = t0 + tj;
        if (job < njobs && pos + t + 1 - k0 > 0) {
          float* dst = a.po + (((size_t)t * a.Hq + g * rep + j) * a.nchunk + c) * kAttDim;
#pragma unroll
          for (int qq = 0; qq < 2; ++qq) {
            const float* ev = oacc[m][qq][0];
            const float* od = oacc[m][qq][1];
            reinterpret_cast<float4*>(dst + 16 * (2 * warp + qq) + 4 * tl)[0] =
                make_float4(ev[2 * half], od[2 * half], ev[2 * half + 1], od[2 * half + 1]);
          }
        }
      }
    }
  }
  named_sync(kBarMix, 256);   // shared memory reusable by the caller
  (void)nkeys;
}

template <int NT>
QHL_DEV void attn_unit(const AttnArgs& a, int c, int g, int pos, int t0, uint8_t* smem) {
  AttnRegs R;
  attn_load_old(a, c, g, pos, pos + t0 + min(kAttGroup, NT - t0), R);
  attn_compute<NT>(a, c, g, pos, t0, smem, R);
}

template <int NT>
__global__ void __launch_bounds__(256) attn_partial_kernel(const AttnArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  if (threadIdx.x == 0) pdl_launch();
  const int pos = *a.kv_len;
  const int t0 = blockIdx.z * kAttGroup, ntk = min(kAttGroup, NT - t0);
  if ((int)blockIdx.x * kAttChunk >= pos + t0 + ntk) return;   // no token of the group sees the chunk
  AttnRegs R;
  attn_load_old(a, blockIdx.x, blockIdx.y, pos, pos + t0 + ntk, R);   // overlaps the in-projection's end
  pdl_wait();
  attn_compute<NT>(a, blockIdx.x, blockIdx.y, pos, t0, smem, R);
}

// Combine the chunk partials of one (token, query head) and apply the sigmoid
// output gate, for 64 of the head's dimensions (quarter qd: 64 qd .. +63), so
// a (token, head) takes four CTAs.  Thread (cq = tid / 64, d = tid % 64) sums
// dimension 64 qd + d over chunks cq, cq + 4, cq + 8, .. in order; the four
// sums are added as (0 + 1) + (2 + 3).  Its first 32 chunks' partials are
// requested together with the chunk statistics (staged in shared memory: cs
// holds [nchunk] max, [nchunk] weight, [nchunk] sum, then [4][64] partial
// sums), so a context up to 8192 rows costs one memory round trip.  The global
// max is exact in any order; the normaliser is summed with a fixed structure
// (lane l takes chunks l, l + 32, .. in order, then a butterfly).  The result
// depends only on the token's position, never on NT.
constexpr int kCombineParts = 4;
__host__ __device__ constexpr int combine_smem_bytes(int nchunk) { return (3 * nchunk + kCombineParts * 64) * 4; }

template <int NT>
QHL_DEV void combine_unit(const AttnArgs& a, int t, int head, int qd, int pos, float* cs) {
  const int tid = threadIdx.x, lane = tid & 31, cq = tid >> 6, d = tid & 63;
  const int dim = 64 * qd + d;
  const int nc = (pos + t + 1 + kAttChunk - 1) / kAttChunk;
  const size_t base = ((size_t)t * a.Hq + head) * a.nchunk;
  float* cm = cs;
  float* cw = cs + a.nchunk;
  float* cl = cs + 2 * a.nchunk;
  float* part = cs + 3 * a.nchunk;
  constexpr int B = 32;
  const float* po = a.po + base * kAttDim + dim;
  float v[B];
#pragma unroll
  for (int j = 0; j < B; ++j) {
    const int c = cq + kCombineParts * j;
    v[j] = c < nc ? ld_cg_once(po + (size_t)c * kAttDim) : 0.f;
  }
  const float gate = cq == 0 ? __ldcg(a.y + (size_t)t * a.y_stride + a.Hq * kAttDim + head * kAttDim + dim) : 0.f;
  for (int c = tid; c < nc; c += 256) {
    cm[c] = __ldcg(a.pm + base + c);
    cl[c] = __ldcg(a.pl + base + c);
  }
  named_sync(kBarMix, 256);
  float M = -INFINITY;
  for (int c = lane; c < nc; c += 32) M = fmaxf(M, cm[c]);
  M = warp_max(M);
  for (int c = tid; c < nc; c += 256) cw[c] = expf(__fsub_rn(cm[c], M));
  named_sync(kBarMix, 256);
  float L = 0.f;
  for (int c = lane; c < nc; c += 32) L = __fmaf_rn(cl[c], cw[c], L);
  L = warp_sum(L);
  float O = 0.f;
#pragma unroll
  for (int j = 0; j < B; ++j) {
    const int c = cq + kCombineParts * j;
    if (c < nc) O = __fmaf_rn(v[j], cw[c], O);
  }
  for (int c0 = kCombineParts * B; c0 < nc; c0 += kCombineParts * B) {
#pragma unroll
    for (int j = 0; j < B; ++j) {
      const int c = c0 + cq + kCombineParts * j;
      v[j] = c < nc ? ld_cg_once(po + (size_t)c * kAttDim) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < B; ++j) {
      const int c = c0 + cq + kCombineParts * j;
      if (c < nc) O = __fmaf_rn(v[j], cw[c], O);
    }
  }
  part[cq * 64 + d] = O;
  named_sync(kBarMix, 256);
  if (cq == 0) {   // warps 0 and 1: dims 64 qd .. +31 and +32 .. +63, one block each
    const float o = __fadd_rn(__fadd_rn(part[d], part[64 + d]), __fadd_rn(part[128 + d], part[192 + d]));
    const float r = __fmul_rn(__fdiv_rn(o, L), sigmoidf_(gate));
    if (a.out) a.out[(size_t)t * a.out_stride + head * kAttDim + dim] = r;
    if (a.qout)
      qact_store_block(r, a.qout + (size_t)t * a.qout_stride, head * (kAttDim / 32) + (dim >> 5), dim & 31);
  }
  named_sync(kBarMix, 256);   // cs reusable by the caller
}

template <int NT>
__global__ void __launch_bounds__(256) attn_combine_kernel(const AttnArgs a) {
  extern __shared__ float cs[];
  if (threadIdx.x == 0) pdl_launch();
  const int pos = *a.kv_len;
  pdl_wait();
  const int u = blockIdx.x;   // (token, head, quarter)
  combine_unit<NT>(a, u / (kCombineParts * a.Hq), (u / kCombineParts) % a.Hq, u % kCombineParts, pos, cs);
}

}  // namespace qhl
