// Device helpers shared by the stage kernels (sm_100a only).
//
// Inline PTX for: packed f32x2 FMA, mbarrier phases, non-tensor bulk copies
// global -> shared (no cluster multicast), L2 eviction hints and programmatic
// dependent launch.  Every wait here is bounded: on timeout it records an error
// bit in a device word the host reads, and returns.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define QHL_DEV __device__ __forceinline__

namespace qhl {

// Bits of the device error word.
enum : unsigned {
  ERR_WAIT_TIMEOUT = 1u,   // an mbarrier wait ran out of iterations
  ERR_BAD_SHAPE = 2u,      // a kernel saw parameters it cannot handle
};

// Iteration cap of every mbarrier wait (each try_wait blocks for a short
// hardware-defined time, so this bounds a stuck wait to well under a minute).
constexpr uint32_t kWaitLimit = 1u << 24;

QHL_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// d = a * b + c on two f32 lanes, each rounded to nearest (packed FFMA2).
QHL_DEV float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// ---- mbarrier -------------------------------------------------------------
QHL_DEV void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
QHL_DEV void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
QHL_DEV void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
QHL_DEV void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
QHL_DEV bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// The iteration cap of a wait: `limit`, or kWaitLimit when it is 0 (tests of
// the error path pass a small cap so that an injected stall ends quickly).
QHL_DEV uint32_t wait_limit(uint32_t limit) { return limit ? limit : kWaitLimit; }

// Wait for the phase with the given parity to complete; false (and an error
// bit) if it did not within wait_limit(limit) tries.
QHL_DEV bool mbar_wait(uint32_t bar, uint32_t parity, unsigned* err, uint32_t limit = 0) {
  const uint32_t n = wait_limit(limit);
  for (uint32_t i = 0; i < n; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  if (err) atomicOr(err, ERR_WAIT_TIMEOUT);
  return false;
}

// Loads through L2 that the compiler issues exactly where written, once: a
// batch of them stays a batch (one memory round trip) instead of being sunk to
// each value's first use, as register pressure can otherwise make it do.
QHL_DEV uint32_t ld_cg_once(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.global.cg.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
QHL_DEV uint4 ld_cg_once(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

QHL_DEV float ld_cg_once(const float* p) {
  float v;
  asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}
QHL_DEV float2 ld_cg_once(const float2* p) {
  float2 v;
  asm volatile("ld.global.cg.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(p));
  return v;
}

// Error path of a kernel that gave up waiting: idle ~200 us so that bulk copies
// already issued into this CTA's shared memory land before the CTA leaves.
QHL_DEV void drain_inflight_copies() {
  for (int i = 0; i < 200; ++i) __nanosleep(1000);
}

// ---- bulk copies (non-tensor TMA) -----------------------------------------
QHL_DEV uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
// Copy `bytes` (multiple of 16, both addresses 16-byte aligned) from global to
// this CTA's shared memory; completion is signalled on `bar` as tx bytes.
QHL_DEV void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}
QHL_DEV void bulk_g2s_plain(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
// Fetch `bytes` (multiple of 16, 16-byte aligned) from global memory into L2,
// without a destination in shared memory.
QHL_DEV void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) writes to the same memory.
QHL_DEV void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- programmatic dependent launch ---------------------------------------
// Block until every grid this one depends on has completed and its memory is
// visible (no-op when launched without a programmatic dependency).
QHL_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the dependent grid to be scheduled.
QHL_DEV void pdl_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- named barrier among a subset of warps ---------------------------------
// Barrier 0 is __syncthreads.  The mixer units (DeltaNet step, attention,
// stage input) synchronise their 256 (or 128) threads on kBarMix, so they can
// run beside warps that use other named barriers.
constexpr int kBarMix = 5;
QHL_DEV void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Arrive on a named barrier without waiting for it (the other participants
// use named_sync with the same count).
QHL_DEV void named_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Named barrier that also ANDs a predicate over the participating threads:
// every thread gets the same answer.
QHL_DEV bool bar_and(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// ---- warp reductions: xor butterflies give every lane the same bits --------
QHL_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
QHL_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// 1 / sqrt(mean + eps) from per-tile partial sums, computed by one warp: lane
// l sums tiles l, l + 32, .. in order, then an xor butterfly (every lane gets
// the same bits).  One round of loads instead of a chain; the summation order
// is fixed by ntiles alone.
QHL_DEV float rstd_warp(const float* ss, int ntiles, float inv_dim, float eps, int lane) {
  constexpr int B = 8;   // up to 256 tiles in one round of loads
  float v[B];
#pragma unroll
  for (int j = 0; j < B; ++j) v[j] = lane + 32 * j < ntiles ? ld_cg_once(ss + lane + 32 * j) : 0.f;
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < B; ++j)
    if (lane + 32 * j < ntiles) s = __fadd_rn(s, v[j]);
  for (int i = lane + 32 * B; i < ntiles; i += 32) s = __fadd_rn(s, __ldcg(ss + i));
  s = warp_sum(s);
  return __frcp_rn(__fsqrt_rn(__fadd_rn(__fmul_rn(s, inv_dim), eps)));
}

// 1 / (1 + e^-x) without overflow: e^-|x| <= 1 always, so the result only
// underflows where the true value is below the f32 range.
QHL_DEV float sigmoidf_(float x) {
  const float e = expf(-fabsf(x));
  const float d = __fadd_rn(1.f, e);
  return x >= 0.f ? __frcp_rn(d) : __fdiv_rn(e, d);
}

}  // namespace qhl
