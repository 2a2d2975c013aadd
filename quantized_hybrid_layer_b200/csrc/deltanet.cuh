// Gated-DeltaNet state step over n_tok tokens (Gated DeltaNet: ChatTorrent
// README, "What it can run"; SwarmLLM README model table "hybrid
// Gated-DeltaNet + attention"; the gated delta rule of the Gated DeltaNet paper
// its prior-work line names).
//
// Per value head h (key head g = h / (Hv/Hk)), with q, k L2-normalised,
// beta = sigmoid(b) and alpha = exp(-softplus(a)) = 1 / (1 + e^a):
//     S <- alpha * S (I - beta k k^T) + beta v k^T,      o = S q  (updated S)
// Row i of S (value dim) changes independently of the others:
//     S_i <- alpha S_i + beta (v_i - alpha (S_i . k)) k,   o_i = S_i . q
//
// Each warp keeps 4 rows of one head's 128x128 f32 state in registers (lane l
// holds columns 4l..4l+3) for all NT tokens (8 warps = 32 rows per CTA, so a
// CTA owns whole 32-value output blocks), so the state is read from HBM once
// and written once per token as the snapshot S_t used for exact rollback
// (SwarmLLM README: drafts are verified in one batched pass and the rejected
// tail is undone exactly in the recurrent state).  The state rows are loaded before griddepcontrol.wait, overlapping
// the in-projection that produces q, k, v, b, a.  Reductions are xor
// butterflies over fixed lane partials, so every token's arithmetic is the
// same whatever NT is.
#pragma once

#include "qact.cuh"

namespace qhl {

constexpr int kDnDim = 128;

struct DnArgs {
  const float* y;          // [NT][y_stride] in-projection output: q | k | v | b | a
  int y_stride;
  int Hk, Hv;
  // state source / snapshot destinations:
  //   cur != nullptr (stage): S_0 = ring[*cur], S_t -> ring[(*cur + t) % ring_size]
  //   cur == nullptr: S_0 = s_in, S_t -> ring[t - 1]
  float* ring;
  long long state_elems;   // Hv * 128 * 128
  int ring_size;
  const int* cur;
  const float* s_in;
  float* o;                // optional f32 output [NT][o_stride], o_stride >= Hv * 128
  int o_stride;
  uint8_t* qo;             // optional output in block fixed point (the out-projection's input)
  int qo_stride;
  int mode;                // DN_SNAPSHOTS, DN_FINAL or DN_CHUNKED
};

// What a pass keeps of the recurrent state:
//   DN_SNAPSHOTS  the state after every token (a verify pass: any prefix can
//                 be committed),
//   DN_FINAL      the state after the last token only, the same sequential
//                 arithmetic (a prefill chunk, committed whole: bit-identical
//                 to DN_SNAPSHOTS followed by commit of every token),
//   DN_CHUNKED    the state after the last token by the chunked closed form of
//                 the recurrence (a prefill chunk; not bit-identical to the
//                 token-by-token steps, within rounding of them).
enum DnMode : int { DN_SNAPSHOTS = 0, DN_FINAL = 1, DN_CHUNKED = 2 };

// Sum of each of 32 per-lane values over the warp; lane l returns the total of
// value l.  Five halving steps: at each, a lane keeps the half of its values
// that its lane bit selects and adds the partner's copy of that half.
QHL_DEV float warp_transpose_sum(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool up = lane & w;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float keep = up ? v[w + i] : v[i];
      const float send = up ? v[i] : v[w + i];
      v[i] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, w));
    }
  }
  return v[0];
}

QHL_DEV float dot4(float4 a, float4 b) {
  float s = __fmul_rn(a.x, b.x);
  s = __fmaf_rn(a.y, b.y, s);
  s = __fmaf_rn(a.z, b.z, s);
  return __fmaf_rn(a.w, b.w, s);
}

// One unit: 32 rows of value head `unit / 4` (8 warps x 4 rows), all NT tokens.
// ob: shared [NT][32] for the unit's outputs.  q, k, v, b, a are read through
// L2 (they may have been written earlier in the same kernel by another CTA).
// The unit's starting state rows (they never depend on the kernel before).
template <int NT>
QHL_DEV void dn_load(const DnArgs& a, int unit, float4 (&S)[4]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = unit >> 2, row0 = (unit & 3) * 32 + warp * 4;
  const float* s_in = a.cur ? a.ring + (size_t)(*a.cur) * a.state_elems : a.s_in;
#pragma unroll
  for (int r = 0; r < 4; ++r)
    S[r] = __ldg(reinterpret_cast<const float4*>(s_in + ((size_t)h * kDnDim + row0 + r) * kDnDim) + lane);
}

// Shared memory of one unit (floats): outputs ob [NT][32], then the unit's
// inputs staged once for all tokens: q, k [NT][128] each, v [NT][32], b, a
// [NT]; then, for the chunked form, c, e^c, e^(c_n - c) [NT] and two [NT][NT]
// coefficient matrices.
constexpr int dn_smem_floats(int nt) { return nt * (32 + 2 * kDnDim + 32 + 2) + 3 * nt + 2 * nt * nt; }

template <int NT>
QHL_DEV void dn_run(const DnArgs& a, int unit, float4 (&S)[4], float* sm) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = unit >> 2;                       // 4 units of 32 rows per head
  const int row0 = (unit & 3) * 32 + warp * 4;
  const int g = h / (a.Hv / a.Hk);
  const int cur = a.cur ? *a.cur : 0;
  float (*ob)[32] = reinterpret_cast<float (*)[32]>(sm);
  float* sq = sm + NT * 32;                      // [NT][128]
  float* sk = sq + NT * kDnDim;                  // [NT][128]
  float* sv = sk + NT * kDnDim;                  // [NT][32]: value rows (unit & 3) * 32 ..
  float* sb = sv + NT * 32;                      // [NT]
  float* sa = sb + NT;                           // [NT]

  const int off_k = a.Hk * kDnDim;
  const int off_v = 2 * a.Hk * kDnDim;
  const int off_b = off_v + a.Hv * kDnDim;
  const int off_a = off_b + a.Hv;
  // every token's inputs in one round of loads (through L2: written by the
  // in-projection, possibly earlier in the same kernel)
  for (int i = tid; i < NT * 64; i += 256) {
    const int t = i >> 6, q4 = i & 63;
    const float* yt = a.y + (size_t)t * a.y_stride;
    const float4 v = __ldcg(reinterpret_cast<const float4*>(yt + (q4 < 32 ? 0 : off_k) + g * kDnDim) + (q4 & 31));
    reinterpret_cast<float4*>(q4 < 32 ? sq + t * kDnDim : sk + t * kDnDim)[q4 & 31] = v;
  }
  for (int i = tid; i < NT * 32; i += 256) {
    const int t = i >> 5, r = i & 31;
    sv[i] = __ldcg(a.y + (size_t)t * a.y_stride + off_v + h * kDnDim + (unit & 3) * 32 + r);
  }
  if (tid < NT) {
    sb[tid] = __ldcg(a.y + (size_t)tid * a.y_stride + off_b + h);
    sa[tid] = __ldcg(a.y + (size_t)tid * a.y_stride + off_a + h);
  }
  named_sync(kBarMix, 256);

  for (int t = 0; t < NT; ++t) {
    float4 q = reinterpret_cast<const float4*>(sq + t * kDnDim)[lane];
    float4 k = reinterpret_cast<const float4*>(sk + t * kDnDim)[lane];
    float v[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) v[r] = sv[t * 32 + warp * 4 + r];
    const float bb = sb[t], aa = sa[t];
    const float rq = __frcp_rn(__fsqrt_rn(__fadd_rn(warp_sum(dot4(q, q)), 1e-6f)));
    const float rk = __frcp_rn(__fsqrt_rn(__fadd_rn(warp_sum(dot4(k, k)), 1e-6f)));
    q = make_float4(__fmul_rn(q.x, rq), __fmul_rn(q.y, rq), __fmul_rn(q.z, rq), __fmul_rn(q.w, rq));
    k = make_float4(__fmul_rn(k.x, rk), __fmul_rn(k.y, rk), __fmul_rn(k.z, rk), __fmul_rn(k.w, rk));
    const float beta = sigmoidf_(bb);      // sigmoid(b)
    const float alpha = sigmoidf_(-aa);    // exp(-softplus(a)) = sigmoid(-a)
    float* dst = a.cur ? a.ring + (size_t)((cur + 1 + t) % a.ring_size) * a.state_elems
                       : a.ring + (size_t)t * a.state_elems;
    const bool keep = a.mode == DN_SNAPSHOTS || t == NT - 1;   // DN_FINAL: the last state only
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float kS = warp_sum(dot4(S[r], k));
      const float coef = __fmul_rn(beta, __fsub_rn(v[r], __fmul_rn(alpha, kS)));
      S[r].x = __fmaf_rn(coef, k.x, __fmul_rn(alpha, S[r].x));
      S[r].y = __fmaf_rn(coef, k.y, __fmul_rn(alpha, S[r].y));
      S[r].z = __fmaf_rn(coef, k.z, __fmul_rn(alpha, S[r].z));
      S[r].w = __fmaf_rn(coef, k.w, __fmul_rn(alpha, S[r].w));
      const float o = warp_sum(dot4(S[r], q));
      if (lane == 0) {
        ob[t][warp * 4 + r] = o;
        if (a.o) a.o[(size_t)t * a.o_stride + h * kDnDim + row0 + r] = o;
      }
      if (keep) reinterpret_cast<float4*>(dst + ((size_t)h * kDnDim + row0 + r) * kDnDim)[lane] = S[r];
    }
  }
  named_sync(kBarMix, 256);
  if (a.qo)
    for (int t = warp; t < NT; t += 8)
      qact_store_block(ob[t][lane], a.qo + (size_t)t * a.qo_stride, h * (kDnDim / 32) + (unit & 3), lane);
  named_sync(kBarMix, 256);   // sm reusable by the caller
}

// Chunked form of the same recurrence for a prefill chunk whose tokens are
// committed together (only the final state is kept).  With c_t = sum over
// m <= t of log alpha_m and u_t = beta_t (v_t - alpha_t S_{t-1} k_t), the state
// after token t is
//     S_t = e^{c_t} S_0 + sum_{j <= t} e^{c_t - c_j} u_j k_j^T,
// so each value row i needs only dot products against the starting state:
//     u_t[i] = beta_t (v_t[i] - e^{c_t} (S_0 k_t)[i] - sum_{j < t} e^{c_t - c_j} (k_j . k_t) u_j[i])
//     o_t[i] = e^{c_t} (S_0 q_t)[i] + sum_{j <= t} e^{c_t - c_j} (q_t . k_j) u_j[i]
//     S_n[i] = e^{c_n} S_0[i] + sum_j e^{c_n - c_j} u_j[i] k_j
// (a unit lower-triangular solve per row).  The 2 NT dot products against S_0
// are independent of one another -- no chain of token steps -- and the state is
// read once and written once.  Ratios of the decays are formed as exp of
// differences of c, which is never above 0, so nothing overflows.
template <int NT>
QHL_DEV void dn_run_chunked(const DnArgs& a, int unit, float4 (&S)[4], float* sm) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = unit >> 2;
  const int row0 = (unit & 3) * 32 + warp * 4;
  const int g = h / (a.Hv / a.Hk);
  const int cur = a.cur ? *a.cur : 0;
  float (*ob)[32] = reinterpret_cast<float (*)[32]>(sm);
  float* sq = sm + NT * 32;
  float* sk = sq + NT * kDnDim;
  float* sv = sk + NT * kDnDim;
  float* sb = sv + NT * 32;
  float* sa = sb + NT;
  float* cl = sa + NT;            // c_t
  float* eg = cl + NT;            // e^{c_t}
  float* ef = eg + NT;            // e^{c_{n-1} - c_t}
  float* Lm = ef + NT;            // [t][j]: e^{c_t - c_j} k_j . k_t, j < t
  float* Pm = Lm + NT * NT;       // [t][j]: e^{c_t - c_j} q_t . k_j, j <= t

  const int off_k = a.Hk * kDnDim;
  const int off_v = 2 * a.Hk * kDnDim;
  const int off_b = off_v + a.Hv * kDnDim;
  const int off_a = off_b + a.Hv;
  for (int i = tid; i < NT * 64; i += 256) {
    const int t = i >> 6, q4 = i & 63;
    const float* yt = a.y + (size_t)t * a.y_stride;
    const float4 v = __ldcg(reinterpret_cast<const float4*>(yt + (q4 < 32 ? 0 : off_k) + g * kDnDim) + (q4 & 31));
    reinterpret_cast<float4*>(q4 < 32 ? sq + t * kDnDim : sk + t * kDnDim)[q4 & 31] = v;
  }
  for (int i = tid; i < NT * 32; i += 256) {
    const int t = i >> 5, r = i & 31;
    sv[i] = __ldcg(a.y + (size_t)t * a.y_stride + off_v + h * kDnDim + (unit & 3) * 32 + r);
  }
  if (tid < NT) {
    sb[tid] = __ldcg(a.y + (size_t)tid * a.y_stride + off_b + h);
    sa[tid] = __ldcg(a.y + (size_t)tid * a.y_stride + off_a + h);
  }
  named_sync(kBarMix, 256);
  // q, k normalised in place (warp w: tokens w, w + 8); decays by thread 0
  for (int t = warp; t < NT; t += 8) {
    float4 q = reinterpret_cast<const float4*>(sq + t * kDnDim)[lane];
    float4 k = reinterpret_cast<const float4*>(sk + t * kDnDim)[lane];
    const float rq = __frcp_rn(__fsqrt_rn(__fadd_rn(warp_sum(dot4(q, q)), 1e-6f)));
    const float rk = __frcp_rn(__fsqrt_rn(__fadd_rn(warp_sum(dot4(k, k)), 1e-6f)));
    reinterpret_cast<float4*>(sq + t * kDnDim)[lane] =
        make_float4(__fmul_rn(q.x, rq), __fmul_rn(q.y, rq), __fmul_rn(q.z, rq), __fmul_rn(q.w, rq));
    reinterpret_cast<float4*>(sk + t * kDnDim)[lane] =
        make_float4(__fmul_rn(k.x, rk), __fmul_rn(k.y, rk), __fmul_rn(k.z, rk), __fmul_rn(k.w, rk));
  }
  if (tid == 0) {
    float c = 0.f;
    for (int t = 0; t < NT; ++t) {
      const float x = sa[t];   // log alpha = -softplus(a), computed without overflow
      const float sp = x > 0.f ? __fadd_rn(x, log1pf(expf(-x))) : log1pf(expf(x));
      c = __fsub_rn(c, sp);
      cl[t] = c;
      eg[t] = expf(c);
      sb[t] = sigmoidf_(sb[t]);   // beta
    }
    for (int t = 0; t < NT; ++t) ef[t] = expf(__fsub_rn(cl[NT - 1], cl[t]));
  }
  named_sync(kBarMix, 256);
  // token pairs, one thread each: k_j . k_t and q_t . k_j over the 128 dims,
  // float4s taken in order from float4 j (mod 32) so that the 8 lanes of a
  // shared-memory phase read distinct banks, two partial sums per product over
  // alternate float4s
  if (tid < NT * NT) {
    const int t = tid / NT, j = tid % NT;
    const float4* kj = reinterpret_cast<const float4*>(sk + j * kDnDim);
    const float4* kt = reinterpret_cast<const float4*>(sk + t * kDnDim);
    const float4* qt = reinterpret_cast<const float4*>(sq + t * kDnDim);
    float kk0 = 0.f, kk1 = 0.f, qk0 = 0.f, qk1 = 0.f;
#pragma unroll 4
    for (int i = 0; i < kDnDim / 4; i += 2) {
      const int d0 = (i + j) & 31, d1 = (i + 1 + j) & 31;
      const float4 a0 = kj[d0], a1 = kj[d1];
      kk0 = __fmaf_rn(a0.w, kt[d0].w, __fmaf_rn(a0.z, kt[d0].z, __fmaf_rn(a0.y, kt[d0].y, __fmaf_rn(a0.x, kt[d0].x, kk0))));
      kk1 = __fmaf_rn(a1.w, kt[d1].w, __fmaf_rn(a1.z, kt[d1].z, __fmaf_rn(a1.y, kt[d1].y, __fmaf_rn(a1.x, kt[d1].x, kk1))));
      qk0 = __fmaf_rn(a0.w, qt[d0].w, __fmaf_rn(a0.z, qt[d0].z, __fmaf_rn(a0.y, qt[d0].y, __fmaf_rn(a0.x, qt[d0].x, qk0))));
      qk1 = __fmaf_rn(a1.w, qt[d1].w, __fmaf_rn(a1.z, qt[d1].z, __fmaf_rn(a1.y, qt[d1].y, __fmaf_rn(a1.x, qt[d1].x, qk1))));
    }
    const float e = j <= t ? expf(__fsub_rn(cl[t], cl[j])) : 0.f;
    Lm[tid] = j < t ? __fmul_rn(e, __fadd_rn(kk0, kk1)) : 0.f;
    Pm[tid] = __fmul_rn(e, __fadd_rn(qk0, qk1));
  }
  named_sync(kBarMix, 256);

  float* dst = a.cur ? a.ring + (size_t)((cur + NT) % a.ring_size) * a.state_elems
                     : a.ring + (size_t)(NT - 1) * a.state_elems;
#pragma unroll 1
  for (int r = 0; r < 4; ++r) {
    // the row's 2 NT products with the starting state, S_0 k_t (value t) and
    // S_0 q_t (value 16 + t), reduced over the warp in one transposed
    // butterfly: lane l ends with value l
    float x32[32];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      x32[t] = t < NT ? dot4(S[r], reinterpret_cast<const float4*>(sk + t * kDnDim)[lane]) : 0.f;
      x32[16 + t] = t < NT ? dot4(S[r], reinterpret_cast<const float4*>(sq + t * kDnDim)[lane]) : 0.f;
    }
    const float mine = warp_transpose_sum(x32, lane);
    float A[NT], u[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) A[t] = __shfl_sync(0xffffffffu, mine, t);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float x = __fsub_rn(sv[t * 32 + warp * 4 + r], __fmul_rn(eg[t], A[t]));
#pragma unroll
      for (int j = 0; j < t; ++j) x = __fsub_rn(x, __fmul_rn(Lm[t * NT + j], u[j]));
      u[t] = __fmul_rn(sb[t], x);
    }
    // output of token t in lane 16 + t
    if (lane >= 16 && lane - 16 < NT) {
      const int t = lane - 16;
      float o = __fmul_rn(eg[t], mine);
#pragma unroll
      for (int j = 0; j < NT; ++j)
        if (j <= t) o = __fmaf_rn(Pm[t * NT + j], u[j], o);
      ob[t][warp * 4 + r] = o;
      if (a.o) a.o[(size_t)t * a.o_stride + h * kDnDim + row0 + r] = o;
    }
    const float e = eg[NT - 1];
    float4 sn = make_float4(__fmul_rn(e, S[r].x), __fmul_rn(e, S[r].y), __fmul_rn(e, S[r].z), __fmul_rn(e, S[r].w));
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const float w = __fmul_rn(ef[j], u[j]);
      const float4 kj = reinterpret_cast<const float4*>(sk + j * kDnDim)[lane];
      sn.x = __fmaf_rn(w, kj.x, sn.x);
      sn.y = __fmaf_rn(w, kj.y, sn.y);
      sn.z = __fmaf_rn(w, kj.z, sn.z);
      sn.w = __fmaf_rn(w, kj.w, sn.w);
    }
    reinterpret_cast<float4*>(dst + ((size_t)h * kDnDim + row0 + r) * kDnDim)[lane] = sn;
  }
  named_sync(kBarMix, 256);
  if (a.qo)
    for (int t = warp; t < NT; t += 8)
      qact_store_block(ob[t][lane], a.qo + (size_t)t * a.qo_stride, h * (kDnDim / 32) + (unit & 3), lane);
  named_sync(kBarMix, 256);
}

template <int NT>
QHL_DEV void dn_unit(const DnArgs& a, int unit, float* sm) {
  float4 S[4];
  dn_load<NT>(a, unit, S);
  dn_run<NT>(a, unit, S, sm);
}

template <int NT>
__global__ void __launch_bounds__(256) dn_step_kernel(const DnArgs a) {
  __shared__ __align__(16) float sm[dn_smem_floats(NT)];
  if (threadIdx.x == 0) pdl_launch();
  float4 S[4];
  dn_load<NT>(a, blockIdx.x, S);   // overlaps the in-projection's last tiles
  pdl_wait();                      // q, k, v, b, a come from it
  if (a.mode == DN_CHUNKED)
    dn_run_chunked<NT>(a, blockIdx.x, S, sm);
  else
    dn_run<NT>(a, blockIdx.x, S, sm);
}

}  // namespace qhl
