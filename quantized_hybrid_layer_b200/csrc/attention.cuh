// Split-K GQA decode attention with QK-norm, partial RoPE, f16 KV cache and a
// sigmoid output gate (ChatTorrent README, "What it can run", lists these three
// features of the hybrid's full-attention layers; Unstable Legion, "Splitting
// the workload": a stage holds the attention cache of its own layers only).
//
// Token t of a pass sits at absolute position pos + t and attends to cache rows
// 0 .. pos + t.  The context is cut into fixed chunks of 64 rows at absolute
// multiples of 64; one CTA handles one (chunk, KV head) for every token and
// every query head of the group, so each K/V row is read from HBM once per pass.
// A token's partial (max, sum, weighted V) over a chunk depends only on the
// token and the chunk, and the combine walks chunks 0 .. in order, so a batched
// pass gives the same bits as running the tokens one at a time.
//
// New rows: the CTA whose chunk holds position p = pos + t normalises and
// rotates the token's k, rounds k and v to f16, writes them to the cache and
// uses the rounded values, exactly what a later pass reads back.
#pragma once

#include "qact.cuh"

namespace qhl {

constexpr int kAttDim = 256;
constexpr int kRopeDims = 64;
constexpr int kAttChunk = 64;
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

// Shared memory of one attention unit: normalised, rotated queries
// [jobs][256], scores / probabilities [jobs][64], a per-warp vector [8][256];
// jobs = NT * (query heads per KV head).
__host__ __device__ constexpr int attn_smem_bytes(int nt, int rep) {
  return nt * rep * kAttDim * 4 + nt * rep * kAttChunk * 4 + 8 * kAttDim * 4;
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

QHL_DEV void half8(uint4 w, float (&f)[8]) {
  const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __half2float(__ushort_as_half(static_cast<unsigned short>(w4[i] & 0xFFFFu)));
    f[2 * i + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(w4[i] >> 16)));
  }
}

// One attention unit: KV head g, context chunk c (rows 64c .. 64c+63), tokens
// t0 .. t0 + min(kAttGroup, NT - t0) - 1 and the group's query heads.  Writes
// per (token, head, chunk) the max score, the sum of exp and the exp-weighted
// V sum.  The unit's tokens' own rows in the chunk are written first; then the
// chunk's K and V rows are loaded into registers through L2.  All 256 threads
// of the CTA take part; `pos` is the position of token 0.  A token's results
// depend only on the token and the chunk, whatever its group.
template <int NT>
QHL_DEV void attn_unit(const AttnArgs& a, int c, int g, int pos, int t0, uint8_t* smem) {
  const int rep = a.Hq / a.Hkv;
  const int ntk = min(kAttGroup, NT - t0);
  const int njobs = ntk * rep;
  float* qs = reinterpret_cast<float*>(smem);                 // [njobs][256]
  float* sc = qs + njobs * kAttDim;                            // [njobs][64]
  float* vec_all = sc + njobs * kAttChunk;                     // [8][256]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k0 = c * kAttChunk;
  const int ctx_end = pos + t0 + ntk;                          // rows the unit's tokens see
  const int nkeys = min(kAttChunk, ctx_end - k0);             // > 0 by the caller
  float* vec = vec_all + warp * kAttDim;
  const int q_off = 0, k_off = 2 * a.Hq * kAttDim, v_off = k_off + a.Hkv * kAttDim;
  const size_t head_base = (size_t)g * a.max_ctx;

  // this pass's own rows that fall in the chunk: QK-norm + RoPE k, round k and v to f16, store
  const int p_lo = max(k0, pos + t0), p_hi = min(k0 + kAttChunk, ctx_end);
  for (int p = p_lo + warp; p < p_hi; p += 8) {
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
    reinterpret_cast<uint4*>(a.K + (head_base + p) * kAttDim)[lane] =
        make_uint4(kh[0] | (kh[1] << 16), kh[2] | (kh[3] << 16), kh[4] | (kh[5] << 16), kh[6] | (kh[7] << 16));
    reinterpret_cast<uint4*>(a.V + (head_base + p) * kAttDim)[lane] =
        make_uint4(vh[0] | (vh[1] << 16), vh[2] | (vh[3] << 16), vh[4] | (vh[5] << 16), vh[6] | (vh[7] << 16));
    __syncwarp();
  }
  // queries of every token that sees this chunk
  for (int job = warp; job < njobs; job += 8) {
    const int tj = job / rep, j = job - tj * rep, t = t0 + tj;
    if (pos + t < k0) continue;
    const float* yt = a.y + (size_t)t * a.y_stride;
    float x[8];
    load8_cg(yt + q_off + (g * rep + j) * kAttDim + 8 * lane, x);
    norm_rope(x, a.gq, a.eps, a.rope + (size_t)(pos + t) * (kRopeDims / 2), vec, lane);
    reinterpret_cast<float4*>(qs + job * kAttDim)[2 * lane] = reinterpret_cast<const float4*>(vec)[2 * lane];
    reinterpret_cast<float4*>(qs + job * kAttDim)[2 * lane + 1] = reinterpret_cast<const float4*>(vec)[2 * lane + 1];
    __syncwarp();
  }
  named_sync(kBarMix, 256);   // new cache rows and queries visible to all 256 threads

  // K rows are loaded up front and V rows right after the scores (through L2,
  // each in one round), so the unit pays the memory latency about twice.  Scores: lane quad (lane >> 2) of warp w owns key
  // 8w + (lane >> 2); the quad's 4 lanes split its 256 dims into interleaved
  // 8-dim groups (group 4i + r for lane r), so q is read from shared memory
  // as conflict-free broadcasts and a score needs two shuffles.  PV: thread
  // (pair p = tid & 127, half = tid >> 7) owns dims 2p, 2p+1 over keys
  // 32 half .. 32 half + 31.
  const int r4 = lane & 3, key = warp * 8 + (lane >> 2);
  uint4 kw[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    kw[i] = key < nkeys ? ld_cg_once(reinterpret_cast<const uint4*>(a.K + (head_base + k0 + key) * kAttDim) + 4 * i + r4)
                        : make_uint4(0u, 0u, 0u, 0u);

  // scores q.k / 16 (1 / sqrt(256)); per (query, key): each lane's 64 dims in
  // group order, then the quad butterfly -- the same operations for any NT
  for (int j0 = 0; j0 < njobs; j0 += 8) {
    float acc[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) acc[jj] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float kf[8];
      half8(kw[i], kf);
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        if (j0 + jj < njobs) {
          const float4* qp = reinterpret_cast<const float4*>(qs + (j0 + jj) * kAttDim + 8 * (4 * i + r4));
          const float4 qa = qp[0], qb = qp[1];
          float s = acc[jj];
          s = __fmaf_rn(qa.x, kf[0], s);
          s = __fmaf_rn(qa.y, kf[1], s);
          s = __fmaf_rn(qa.z, kf[2], s);
          s = __fmaf_rn(qa.w, kf[3], s);
          s = __fmaf_rn(qb.x, kf[4], s);
          s = __fmaf_rn(qb.y, kf[5], s);
          s = __fmaf_rn(qb.z, kf[6], s);
          s = __fmaf_rn(qb.w, kf[7], s);
          acc[jj] = s;
        }
      }
    }
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      float s = acc[jj];
      s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, 1));
      s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, 2));
      if (j0 + jj < njobs && r4 == 0 && key < nkeys) sc[(j0 + jj) * kAttChunk + key] = __fmul_rn(s, 1.f / 16.f);
    }
  }
  // V rows, issued before the softmax so their latency overlaps it (volatile
  // loads: the compiler may neither repeat them later nor move them)
  const int pair = tid & 127, half = tid >> 7;
  uint32_t vr[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int kk = half * 32 + i;
    vr[i] = kk < nkeys ? ld_cg_once(reinterpret_cast<const uint32_t*>(a.V + (head_base + k0 + kk) * kAttDim) + pair) : 0u;
  }
  named_sync(kBarMix, 256);

  // chunk softmax statistics, one warp per query
  for (int job = warp; job < njobs; job += 8) {
    const int tj = job / rep, j = job - tj * rep, t = t0 + tj;
    const int nk = min(kAttChunk, pos + t + 1 - k0);
    if (nk <= 0) continue;
    const bool v0 = lane < nk, v1 = lane + 32 < nk;
    const float s0 = v0 ? sc[job * kAttChunk + lane] : -INFINITY;
    const float s1 = v1 ? sc[job * kAttChunk + lane + 32] : -INFINITY;
    const float m = warp_max(fmaxf(s0, s1));
    const float e0 = v0 ? expf(__fsub_rn(s0, m)) : 0.f;
    const float e1 = v1 ? expf(__fsub_rn(s1, m)) : 0.f;
    const float l = warp_sum(__fadd_rn(e0, e1));
    sc[job * kAttChunk + lane] = e0;
    sc[job * kAttChunk + lane + 32] = e1;
    if (lane == 0) {
      const size_t idx = ((size_t)t * a.Hq + g * rep + j) * a.nchunk + c;
      a.pm[idx] = m;
      a.pl[idx] = l;
    }
  }
  named_sync(kBarMix, 256);

  // exp-weighted V: per (query, dim) the keys of each half in order, then
  // half 0 + half 1; 4 queries at a time (vec_all holds half 1's sums), so
  // the V rows stay in registers across the batches
  constexpr int JB = 4;
  float* part = vec_all;   // [JB][256]
  for (int j0 = 0; j0 < njobs; j0 += JB) {
    float o0[JB], o1[JB];
    int nk[JB];
#pragma unroll
    for (int jj = 0; jj < JB; ++jj) {
      o0[jj] = 0.f;
      o1[jj] = 0.f;
      nk[jj] = j0 + jj < njobs ? min(kAttChunk, pos + t0 + (j0 + jj) / rep + 1 - k0) : 0;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int kk = half * 32 + i;
      const float vlo = __half2float(__ushort_as_half(static_cast<unsigned short>(vr[i] & 0xFFFFu)));
      const float vhi = __half2float(__ushort_as_half(static_cast<unsigned short>(vr[i] >> 16)));
#pragma unroll
      for (int jj = 0; jj < JB; ++jj) {
        if (kk < nk[jj]) {
          const float pr = sc[(j0 + jj) * kAttChunk + kk];
          o0[jj] = __fmaf_rn(pr, vlo, o0[jj]);
          o1[jj] = __fmaf_rn(pr, vhi, o1[jj]);
        }
      }
    }
    if (half == 1) {
#pragma unroll
      for (int jj = 0; jj < JB; ++jj)
        reinterpret_cast<float2*>(part + jj * kAttDim)[pair] = make_float2(o0[jj], o1[jj]);
    }
    named_sync(kBarMix, 256);
    if (half == 0) {
#pragma unroll
      for (int jj = 0; jj < JB; ++jj) {
        const int job = j0 + jj;
        if (job < njobs && nk[jj] > 0) {
          const int tj = job / rep, j = job - tj * rep, t = t0 + tj;
          const float2 h1 = reinterpret_cast<const float2*>(part + jj * kAttDim)[pair];
          float2* dst = reinterpret_cast<float2*>(a.po + (((size_t)t * a.Hq + g * rep + j) * a.nchunk + c) * kAttDim);
          dst[pair] = make_float2(__fadd_rn(o0[jj], h1.x), __fadd_rn(o1[jj], h1.y));
        }
      }
    }
    named_sync(kBarMix, 256);
  }
}

template <int NT>
__global__ void __launch_bounds__(256) attn_partial_kernel(const AttnArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  if (threadIdx.x == 0) pdl_launch();
  const int pos = *a.kv_len;
  const int t0 = blockIdx.z * kAttGroup, ntk = min(kAttGroup, NT - t0);
  if ((int)blockIdx.x * kAttChunk >= pos + t0 + ntk) return;   // no token of the group sees the chunk
  pdl_wait();
  attn_unit<NT>(a, blockIdx.x, blockIdx.y, pos, t0, smem);
}

// Combine the chunk partials of one (token, query head) and apply the sigmoid
// output gate.  Thread = dim.  The chunk statistics are staged in shared
// memory (cs: 3 * nchunk floats); the global max is exact in any order; the
// normaliser is summed with a fixed structure (lane l takes chunks l, l + 32,
// .. in order, then a butterfly) and the weighted V sums chunk by chunk in
// order, with the loads issued in batches ahead of the accumulation.  The
// result depends only on the token's position, never on NT.
template <int NT>
QHL_DEV void combine_unit(const AttnArgs& a, int t, int head, int pos, float* cs) {
  const int dim = threadIdx.x, lane = dim & 31;
  const int nc = (pos + t + 1 + kAttChunk - 1) / kAttChunk;
  const size_t base = ((size_t)t * a.Hq + head) * a.nchunk;
  float* cm = cs;
  float* cw = cs + a.nchunk;
  float* cl = cs + 2 * a.nchunk;
  for (int c = dim; c < nc; c += 256) {
    cm[c] = __ldcg(a.pm + base + c);
    cl[c] = __ldcg(a.pl + base + c);
  }
  named_sync(kBarMix, 256);
  float M = -INFINITY;
  for (int c = lane; c < nc; c += 32) M = fmaxf(M, cm[c]);
  M = warp_max(M);
  for (int c = dim; c < nc; c += 256) cw[c] = expf(__fsub_rn(cm[c], M));
  named_sync(kBarMix, 256);
  float L = 0.f;
  for (int c = lane; c < nc; c += 32) L = __fmaf_rn(cl[c], cw[c], L);
  L = warp_sum(L);
  float O = 0.f;
  constexpr int B = 32;
  const float* po = a.po + base * kAttDim + dim;
  for (int c0 = 0; c0 < nc; c0 += B) {
    float v[B];
#pragma unroll
    for (int j = 0; j < B; ++j) v[j] = c0 + j < nc ? ld_cg_once(po + (size_t)(c0 + j) * kAttDim) : 0.f;
#pragma unroll
    for (int j = 0; j < B; ++j)
      if (c0 + j < nc) O = __fmaf_rn(v[j], cw[c0 + j], O);
  }
  const float gate = __ldcg(a.y + (size_t)t * a.y_stride + a.Hq * kAttDim + head * kAttDim + dim);
  const float r = __fmul_rn(__fdiv_rn(O, L), sigmoidf_(gate));
  if (a.out) a.out[(size_t)t * a.out_stride + head * kAttDim + dim] = r;
  if (a.qout)   // warp w holds dims 32w..32w+31: one block
    qact_store_block(r, a.qout + (size_t)t * a.qout_stride, head * (kAttDim / 32) + (dim >> 5), dim & 31);
  named_sync(kBarMix, 256);   // cs reusable by the caller
}

template <int NT>
__global__ void __launch_bounds__(256) attn_combine_kernel(const AttnArgs a) {
  extern __shared__ float cs[];                  // [nchunk] max, [nchunk] weight, [nchunk] sum
  if (threadIdx.x == 0) pdl_launch();
  const int pos = *a.kv_len;
  pdl_wait();
  combine_unit<NT>(a, blockIdx.x / a.Hq, blockIdx.x % a.Hq, pos, cs);
}

}  // namespace qhl
