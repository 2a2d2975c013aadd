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
};

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
// inputs staged once for all tokens: q, k [NT][128] each, v [NT][32], b, a [NT].
constexpr int dn_smem_floats(int nt) { return nt * (32 + 2 * kDnDim + 32 + 2); }

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
  named_sync(1, 256);

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
      reinterpret_cast<float4*>(dst + ((size_t)h * kDnDim + row0 + r) * kDnDim)[lane] = S[r];
    }
  }
  named_sync(1, 256);
  if (a.qo)
    for (int t = warp; t < NT; t += 8)
      qact_store_block(ob[t][lane], a.qo + (size_t)t * a.qo_stride, h * (kDnDim / 32) + (unit & 3), lane);
  named_sync(1, 256);   // sm reusable by the caller
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
  dn_run<NT>(a, blockIdx.x, S, sm);
}

}  // namespace qhl
