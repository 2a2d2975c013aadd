// Split-K GQA decode attention with QK-norm, partial RoPE, f16 KV cache and a
// sigmoid output gate (ChatTorrent README, "What it can run": full-attention
// layers "that have partial RoPE, QK-norm and an attention output gate"; each
// stage "keeps its own attention cache": Unstable Legion, "Splitting the
// workload").
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

template <int NT>
constexpr int attn_smem_bytes(int rep) {
  return 2 * kAttChunk * kAttDim * 2            // K, V chunk (f16)
         + NT * rep * kAttDim * 4               // normalised, rotated queries
         + NT * rep * kAttChunk * 4             // scores / probabilities
         + 8 * kAttDim * 4                      // per-warp scratch vector
         + 16;                                  // mbarrier
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

QHL_DEV void load8(const float* p, float (&x)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0];
  const float4 b = reinterpret_cast<const float4*>(p)[1];
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

template <int NT>
__global__ void __launch_bounds__(256) attn_partial_kernel(const AttnArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int rep = a.Hq / a.Hkv;
  uint16_t* Ks = reinterpret_cast<uint16_t*>(smem);
  uint16_t* Vs = Ks + kAttChunk * kAttDim;
  float* qs = reinterpret_cast<float*>(Vs + kAttChunk * kAttDim);   // [NT*rep][256]
  float* sc = qs + NT * rep * kAttDim;                                 // [NT*rep][64]
  float* scratch = sc + NT * rep * kAttChunk;                          // [8][256]
  uint64_t* kvbar = reinterpret_cast<uint64_t*>(scratch + 8 * kAttDim);

  const int c = blockIdx.x, g = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) pdl_launch();
  const int pos = *a.kv_len;
  const int k0 = c * kAttChunk;
  const int ctx_end = pos + NT;
  if (k0 >= ctx_end) return;
  const int nkeys = min(kAttChunk, ctx_end - k0);           // rows this chunk covers for any token
  const int n_old = max(0, min(kAttChunk, pos - k0));        // rows already in the cache

  // cached rows do not depend on this pass: two bulk copies (rows are
  // contiguous per KV head) requested before the dependency wait
  const uint32_t bar = smem_u32(kvbar);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    if (n_old > 0) {
      const uint32_t bytes = (uint32_t)n_old * kAttDim * 2;
      mbar_arrive_expect_tx(bar, 2 * bytes);
      bulk_g2s_plain(smem_u32(Ks), a.K + ((size_t)g * a.max_ctx + k0) * kAttDim, bytes, bar);
      bulk_g2s_plain(smem_u32(Vs), a.V + ((size_t)g * a.max_ctx + k0) * kAttDim, bytes, bar);
    }
  }
  __syncthreads();   // barrier initialised before anyone waits on it
  pdl_wait();

  float* vec = scratch + warp * kAttDim;
  const int q_off = 0, k_off = 2 * a.Hq * kAttDim, v_off = k_off + a.Hkv * kAttDim;
  // this pass's own rows that fall in the chunk
  const int p_lo = max(k0, pos), p_hi = min(k0 + kAttChunk, ctx_end);
  for (int p = p_lo + warp; p < p_hi; p += 8) {
    const int t = p - pos;
    const float* yt = a.y + (size_t)t * a.y_stride;
    float x[8];
    load8(yt + k_off + g * kAttDim + 8 * lane, x);
    norm_rope(x, a.gk, a.eps, a.rope + (size_t)p * (kRopeDims / 2), vec, lane);
    float vv[8];
    load8(yt + v_off + g * kAttDim + 8 * lane, vv);
    uint16_t kh[8], vh[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      kh[i] = __half_as_ushort(__float2half_rn(vec[8 * lane + i]));
      vh[i] = __half_as_ushort(__float2half_rn(vv[i]));
    }
    const uint4 kw = make_uint4(kh[0] | (kh[1] << 16), kh[2] | (kh[3] << 16), kh[4] | (kh[5] << 16), kh[6] | (kh[7] << 16));
    const uint4 vw = make_uint4(vh[0] | (vh[1] << 16), vh[2] | (vh[3] << 16), vh[4] | (vh[5] << 16), vh[6] | (vh[7] << 16));
    const int lr = p - k0;
    reinterpret_cast<uint4*>(Ks + lr * kAttDim)[lane] = kw;
    reinterpret_cast<uint4*>(Vs + lr * kAttDim)[lane] = vw;
    reinterpret_cast<uint4*>(a.K + ((size_t)g * a.max_ctx + p) * kAttDim)[lane] = kw;
    reinterpret_cast<uint4*>(a.V + ((size_t)g * a.max_ctx + p) * kAttDim)[lane] = vw;
    __syncwarp();
  }
  // queries of every token that sees this chunk
  const int njobs = NT * rep;
  for (int job = warp; job < njobs; job += 8) {
    const int t = job / rep, j = job % rep;
    if (pos + t < k0) continue;
    const float* yt = a.y + (size_t)t * a.y_stride;
    float x[8];
    load8(yt + q_off + (g * rep + j) * kAttDim + 8 * lane, x);
    norm_rope(x, a.gq, a.eps, a.rope + (size_t)(pos + t) * (kRopeDims / 2), vec, lane);
    reinterpret_cast<float4*>(qs + job * kAttDim)[2 * lane] = reinterpret_cast<const float4*>(vec)[2 * lane];
    reinterpret_cast<float4*>(qs + job * kAttDim)[2 * lane + 1] = reinterpret_cast<const float4*>(vec)[2 * lane + 1];
    __syncwarp();
  }
  if (n_old > 0) mbar_wait(bar, 0, nullptr);
  __syncthreads();

  // scores q.k / 16: warp w takes rows 8w .. 8w+7, lanes split the 256 dims
  for (int kk = warp * 8; kk < warp * 8 + 8 && kk < nkeys; ++kk) {
    const uint4 kw = reinterpret_cast<const uint4*>(Ks + kk * kAttDim)[lane];
    float kf[8];
    {
      const uint32_t w4[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        kf[2 * i] = __half2float(__ushort_as_half(static_cast<unsigned short>(w4[i] & 0xFFFFu)));
        kf[2 * i + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(w4[i] >> 16)));
      }
    }
    for (int job = 0; job < njobs; ++job) {
      const int t = job / rep;
      if (k0 + kk > pos + t) continue;                       // causal: row beyond the token
      float q8[8];
      load8(qs + job * kAttDim + 8 * lane, q8);
      float s = __fmul_rn(q8[0], kf[0]);
#pragma unroll
      for (int i = 1; i < 8; ++i) s = __fmaf_rn(q8[i], kf[i], s);
      s = warp_sum(s);
      if (lane == 0) sc[job * kAttChunk + kk] = __fmul_rn(s, 1.f / 16.f);   // 1 / sqrt(256)
    }
  }
  __syncthreads();

  // chunk softmax statistics, one warp per query
  for (int job = warp; job < njobs; job += 8) {
    const int t = job / rep, j = job % rep;
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
  __syncthreads();

  // weighted V: thread = dim, rows in order
  const int dim = tid;
  for (int t = 0; t < NT; ++t) {
    const int nk = min(kAttChunk, pos + t + 1 - k0);
    if (nk <= 0) continue;
    float acc[16];
    for (int j0 = 0; j0 < rep; j0 += 16) {
      const int jn = min(16, rep - j0);
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] = 0.f;
      for (int kk = 0; kk < nk; ++kk) {
        const float v = __half2float(__ushort_as_half(Vs[kk * kAttDim + dim]));
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (j < jn) acc[j] = __fmaf_rn(sc[(t * rep + j0 + j) * kAttChunk + kk], v, acc[j]);
      }
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j < jn)
          a.po[(((size_t)t * a.Hq + g * rep + j0 + j) * a.nchunk + c) * kAttDim + dim] = acc[j];
    }
  }
}

// Combine the chunk partials of one (token, query head) in chunk order and
// apply the sigmoid output gate.  Thread = dim.  The per-chunk statistics are
// staged in shared memory and the weighted sums' loads are issued in batches
// ahead of the (in-order) accumulation, so the kernel is not a chain of
// dependent L2 round trips.
template <int NT>
__global__ void __launch_bounds__(256) attn_combine_kernel(const AttnArgs a) {
  extern __shared__ float cs[];                  // [nchunk] max, [nchunk] weight, [nchunk] sum
  const int t = blockIdx.x / a.Hq, head = blockIdx.x % a.Hq, dim = threadIdx.x;
  if (threadIdx.x == 0) pdl_launch();
  const int pos = *a.kv_len;
  pdl_wait();
  const int nc = (pos + t + 1 + kAttChunk - 1) / kAttChunk;
  const size_t base = ((size_t)t * a.Hq + head) * a.nchunk;
  float* cm = cs;
  float* cw = cs + a.nchunk;
  float* cl = cs + 2 * a.nchunk;
  for (int c = threadIdx.x; c < nc; c += 256) {
    cm[c] = a.pm[base + c];
    cl[c] = a.pl[base + c];
  }
  __syncthreads();
  float M = -INFINITY;
  for (int c = 0; c < nc; ++c) M = fmaxf(M, cm[c]);
  for (int c = threadIdx.x; c < nc; c += 256) cw[c] = expf(__fsub_rn(cm[c], M));
  __syncthreads();
  float L = 0.f, O = 0.f;
  for (int c = 0; c < nc; ++c) L = __fmaf_rn(cl[c], cw[c], L);
  constexpr int B = 16;
  const float* po = a.po + base * kAttDim + dim;
  for (int c0 = 0; c0 < nc; c0 += B) {
    float v[B];
#pragma unroll
    for (int j = 0; j < B; ++j) v[j] = c0 + j < nc ? __ldg(po + (size_t)(c0 + j) * kAttDim) : 0.f;
#pragma unroll
    for (int j = 0; j < B; ++j)
      if (c0 + j < nc) O = __fmaf_rn(v[j], cw[c0 + j], O);
  }
  const float gate = a.y[(size_t)t * a.y_stride + a.Hq * kAttDim + head * kAttDim + dim];
  const float r = __fmul_rn(__fdiv_rn(O, L), sigmoidf_(gate));
  if (a.out) a.out[(size_t)t * a.out_stride + head * kAttDim + dim] = r;
  if (a.qout)   // warp w holds dims 32w..32w+31: one block
    qact_store_block(r, a.qout + (size_t)t * a.qout_stride, head * (kAttDim / 32) + (dim >> 5), dim & 31);
}

}  // namespace qhl
